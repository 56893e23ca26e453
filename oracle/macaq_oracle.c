/*
 * macaq_oracle.c -- plain, slow CPU oracle for the MACaQ W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * What it computes follows "MACaQ: Fast, Model Agnostic Calibrated Quantization for
 * Low-Precision Weights and Activations" (arXiv 2611.10649), Abstract: at inference the
 * activations of each layer are scaled channel by channel and rotated by a block
 * Hadamard, the inverse of both is folded into that layer's weights, and both operands
 * are MXFP4 (W4A4), the weights rounded to nearest.  The pages fix
 * neither the block size, the Hadamard normalisation, the scale direction, nor the MX
 * bit layout; the readings used here are:
 *
 *   - block size b = 32, equal to the MX block, so each Hadamard block has one scale;
 *   - H is the Sylvester (natural-order) 32x32 Hadamard matrix, H[i][j] =
 *     (-1)^popcount(i & j), applied unnormalised; its 1/sqrt(32) normalisation is folded
 *     into one fp32 multiplier per input channel together with the channel scale:
 *         activations:  a_k = fl32(c / s_k),   weights:  w_k = fl32(s_k * c),
 *     with c = 1/sqrt(32) in IEEE double (activations are divided by s, weights
 *     multiplied by s, the SmoothQuant direction that the calibration rule
 *     s = sqrt(max|x| / max|W|) is built for);
 *   - the transform is done in fp32 in one canonical order: u_k = fl32(x_k * a_k), then
 *     butterfly stages h = 1, 2, 4, 8, 16, each replacing (u_i, u_{i+h}) by
 *     (fl32(u_i + u_{i+h}), fl32(u_i - u_{i+h})) for every i with (i & h) == 0;
 *   - MXFP4 follows the OCP Microscaling v1.0 format: one E8M0 scale per 32 elements,
 *     shared exponent floor(log2(amax)) - 2 (2 = largest E2M1 exponent), clamped at the
 *     format minimum; elements are v / 2^(e-127) rounded to the nearest E2M1 value, ties
 *     to the even code, saturating at 6;
 *   - an E2M1 code is (sign << 3) | index, index into {0, .5, 1, 1.5, 2, 3, 4, 6}; the
 *     IEEE sign of v is kept, so a negative value that rounds to zero gives 0x8;
 *   - two codes per byte, element 2j in the low nibble; scales are row-major [rows][K/32].
 *
 * The GEMM is the exact contraction of decoded values in fp64.
 *
 * Calibration of s (the step before the fold; the pages name calibration but give no rule):
 * s_j = fl32(sqrt(max_r |xcal_rj| / max_n |W_nj|)) with the maxima, the quotient and the root
 * in IEEE double -- the SmoothQuant alpha = 1/2 balance, after which max|x_j / s_j| and
 * max|W_nj * s_j| agree; s_j = 1 when either maximum is zero (nothing to balance).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no -ffast-math, no -march):
 * every fp32 operation above must be one IEEE round-to-nearest operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitudes, by code index (OCP MX v1.0, FP4 E2M1 element format). */
static const double kE2M1Magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* c = 1/sqrt(32), correctly rounded: sqrt and division are IEEE-exact operations. */
static double hadamard_norm(void) { return 1.0 / sqrt(32.0); }

/* Per-channel multipliers (Abstract: "per-channel scale"; normalisation folded in).
 * act_mult[k] = fl32(c / s_k), w_mult[k] = fl32(s_k * c). */
void oracle_multipliers(const float* s, int64_t K, float* act_mult, float* w_mult) {
    const double c = hadamard_norm();
    for (int64_t k = 0; k < K; ++k) {
        if (act_mult) act_mult[k] = (float)(c / (double)s[k]);
        if (w_mult) w_mult[k] = (float)((double)s[k] * c);
    }
}

/* Unnormalised Sylvester Walsh-Hadamard transform of one 32-block, fp32, canonical
 * stage order h = 1, 2, 4, 8, 16 (block-Hadamard of the Abstract, b = 32). */
static void fwht32_f32(float u[32]) {
    for (int h = 1; h < 32; h <<= 1) {
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                float a = u[i];
                float b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
            }
        }
    }
}

/* Scale then block-Hadamard, fp32 canonical order: V[r][k] for every row.
 * X is [R][K] fp32 (bf16 activations widen to fp32 exactly), mult is [K]. */
void oracle_transform_f32(const float* X, int64_t R, int64_t K, const float* mult, float* V) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            float u[32];
            for (int i = 0; i < 32; ++i) {
                const int64_t k = 32 * b + i;
                u[i] = X[r * K + k] * mult[k];
            }
            fwht32_f32(u);
            for (int i = 0; i < 32; ++i) V[r * K + 32 * b + i] = u[i];
        }
    }
}

/* The same transform in fp64 with fp64 multipliers (used only to check the algebra:
 * with no rounding, transform-then-fold reproduces x W^T). */
void oracle_transform_f64(const double* X, int64_t R, int64_t K, const double* mult, double* V) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            double u[32];
            for (int i = 0; i < 32; ++i) u[i] = X[r * K + 32 * b + i] * mult[32 * b + i];
            for (int h = 1; h < 32; h <<= 1)
                for (int i = 0; i < 32; ++i)
                    if ((i & h) == 0) {
                        double a = u[i], c = u[i + h];
                        u[i] = a + c;
                        u[i + h] = a - c;
                    }
            for (int i = 0; i < 32; ++i) V[r * K + 32 * b + i] = u[i];
        }
    }
}

/* E8M0 shared-scale byte of one block from its largest magnitude (OCP MX v1.0):
 * floor(log2(amax)) - 2, biased by 127, clamped below at 0.  floor(log2(amax)) is the
 * unbiased exponent field of the fp32 amax; zero and subnormal amax give byte 0. */
int oracle_e8m0_from_amax(float amax) {
    uint32_t bits;
    memcpy(&bits, &amax, sizeof bits);
    const int E = (int)((bits >> 23) & 0xFFu);
    return E >= 3 ? E - 2 : 0;
}

/* Index of the E2M1 magnitude nearest to t >= 0; on a tie the even index wins
 * (round half to even on the code); values above 6 land on 6 (saturation). */
int oracle_e2m1_index(double t) {
    int best = 0;
    double best_d = fabs(t - kE2M1Magnitude[0]);
    for (int i = 1; i < 8; ++i) {
        const double d = fabs(t - kE2M1Magnitude[i]);
        if (d < best_d || (d == best_d && (i % 2) == 0)) {
            best = i;
            best_d = d;
        }
    }
    return best;
}

/* 4-bit E2M1 code of v under shared scale byte e: sign bit of v, magnitude of
 * v * 2^(127 - e) (exact in fp64) rounded to the nearest E2M1 value. */
int oracle_e2m1_code(float v, int e) {
    const double q = (double)v * ldexp(1.0, 127 - e);
    const int sign = signbit(v) ? 1 : 0;
    return (sign << 3) | oracle_e2m1_index(fabs(q));
}

/* MXFP4 quantisation of V [R][K] along K: codes [R][K/2] (element 2j low nibble),
 * scales [R][K/32] row-major. */
void oracle_quantize_mx(const float* V, int64_t R, int64_t K, uint8_t* codes, uint8_t* scales) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* v = V + r * K + 32 * b;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                const float m = fabsf(v[i]);
                if (m > amax) amax = m;
            }
            const int e = oracle_e8m0_from_amax(amax);
            scales[r * nb + b] = (uint8_t)e;
            for (int j = 0; j < 16; ++j) {
                const int lo = oracle_e2m1_code(v[2 * j], e);
                const int hi = oracle_e2m1_code(v[2 * j + 1], e);
                codes[r * (K / 2) + 16 * b + j] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* Activation path: scale by a_k, block-Hadamard, MXFP4 (steps a1-a4). */
void oracle_act_transform_quant(const float* X, int64_t R, int64_t K, const float* act_mult,
                                uint8_t* codes, uint8_t* scales) {
    float* V = (float*)malloc((size_t)(R * K) * sizeof(float));
    oracle_transform_f32(X, R, K, act_mult, V);
    oracle_quantize_mx(V, R, K, codes, scales);
    free(V);
}

/* Weight fold (Abstract: inverse transforms absorbed into the weights) then RTN MXFP4:
 * W' = W diag(s) H_bd / sqrt(32) quantised along K.  Also returns act_mult. */
void oracle_fold_weights(const float* W, int64_t N, int64_t K, const float* s, uint8_t* codes,
                         uint8_t* scales, float* act_mult) {
    float* w_mult = (float*)malloc((size_t)K * sizeof(float));
    oracle_multipliers(s, K, act_mult, w_mult);
    float* V = (float*)malloc((size_t)(N * K) * sizeof(float));
    oracle_transform_f32(W, N, K, w_mult, V);
    oracle_quantize_mx(V, N, K, codes, scales);
    free(V);
    free(w_mult);
}

/* Value of element k of an MXFP4 row: +-E2M1 magnitude times 2^(e-127). */
static double mx_decode(const uint8_t* codes_row, const uint8_t* scales_row, int64_t k) {
    const uint8_t byte = codes_row[k / 2];
    const int code = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    const double mag = kE2M1Magnitude[code & 7];
    const double val = (code & 8) ? -mag : mag;
    return ldexp(val, (int)scales_row[k / 32] - 127);
}

/* Decode R rows of an MXFP4 matrix to fp64 [R][K]. */
void oracle_mx_decode(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t K, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = mx_decode(codes + r * (K / 2), scales + r * (K / 32), k);
}

/* Block-scaled GEMM, exact contraction in fp64:
 *   y[i][n] = sum_k dec(A)[rows[i]][k] * dec(W)[n][k]
 * for the n_rows selected activation rows (rows == NULL selects 0..n_rows-1). */
void oracle_mx_gemm(const uint8_t* Aq, const uint8_t* As, const int64_t* rows, int64_t n_rows,
                    const uint8_t* Wq, const uint8_t* Ws, int64_t N, int64_t K, double* y) {
    double* a = (double*)malloc((size_t)(n_rows * K) * sizeof(double));
    for (int64_t i = 0; i < n_rows; ++i) {
        const int64_t m = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; ++k) a[i * K + k] = mx_decode(Aq + m * (K / 2), As + m * (K / 32), k);
    }
#pragma omp parallel
    {
        double* w = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) w[k] = mx_decode(Wq + n * (K / 2), Ws + n * (K / 32), k);
            for (int64_t i = 0; i < n_rows; ++i) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += a[i * K + k] * w[k];
                y[i * N + n] = acc;
            }
        }
        free(w);
    }
    free(a);
}

/* ------------------------------------------------------------------ Flip-Refinement
 *
 * "MACaQ ...", Abstract: Flip-Refinement starts from the round-to-nearest codes and runs a greedy
 * coordinate descent, weighted by the Hessian, in which a step shifts one FP4 code to a
 * neighbouring grid value (the French news page sets it against GPTQ-style updates).  The pages
 * give no more; the readings used here:
 *   - it refines one layer's folded weight codes W' = MXFP4(W diag(w) H_bd), starting from the
 *     round-to-nearest codes, with every E8M0 block scale kept (only codes move);
 *   - the objective of output row n is the layer's output error on the calibration batch,
 *       L_n = (q_n - v_n) Hs (q_n - v_n)^T,   Hs = Xt^T Xt,
 *     q_n the decoded refined row, v_n the fp32 folded row before quantisation, and Xt the
 *     calibration activations after the online transform (fp32, before their quantisation);
 *   - "adjacent representable values": the 15 distinct E2M1 values -6 .. 6 in order; a move
 *     takes one code one step up or down that line (at +-6 only inwards); a code that moves to
 *     zero keeps its sign bit;
 *   - "greedily": each step applies, in one row, the single move with the most negative change
 *     dL = d (2 g_k + d Hs_kk) (g = Hs r, r = q - v, d the value step times the block scale);
 *     ties go to the smaller k, then to the downward move; a row stops when no move lowers L or
 *     after max_moves moves.
 * Arithmetic (fp64, one order, so another implementation can reproduce every decision):
 *   Hs[j][k] = sum over calibration rows c ascending of Xt[c][j] Xt[c][k], as fma(Xt, Xt, acc)
 *   from +0; r_k = q_k - v_k; g_j = sum over k ascending of Hs[j][k] r_k as fma from +0;
 *   dL = d * fma(d, Hs[k][k], 2 g_k); after a move of coordinate k by d:
 *   g_j = fma(d, Hs[j][k], g_j) for every j, r_k = r_k + d. */

/* Hs = Xt^T Xt for transformed calibration activations Xt [C][K] (fp32), fp64 [K][K]. */
void oracle_hessian(const float* Xt, int64_t C, int64_t K, double* Hs) {
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t j = 0; j < K; ++j) {
        for (int64_t k = 0; k < K; ++k) {
            double acc = 0.0;
            for (int64_t c = 0; c < C; ++c) acc = fma((double)Xt[c * K + j], (double)Xt[c * K + k], acc);
            Hs[j * K + k] = acc;
        }
    }
}

/* The 15 E2M1 values in increasing order; position 7 is zero. */
static const double kE2M1Line[15] = {-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0,
                                     0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0};

/* Position of a 4-bit code on that line (both zero codes sit at 7). */
static int e2m1_line_pos(int code) {
    const int m = code & 7;
    return (code & 8) ? 7 - m : 7 + m;
}

/* Code of line position p; a zero keeps the sign bit of `old`. */
static int e2m1_code_at(int p, int old) {
    if (p == 7) return old & 8;
    return p > 7 ? p - 7 : 8 | (7 - p);
}

/* Flip-Refinement of weight codes in place.  V [N][K] fp32 folded weights before quantisation,
 * codes [N][K/2] (their round-to-nearest codes on entry), scales [N][K/32] E8M0 (unchanged),
 * Hs [K][K].  moves[n] = the moves applied to row n. */
void oracle_flip_refine(const float* V, int64_t N, int64_t K, const double* Hs, uint8_t* codes,
                        const uint8_t* scales, int64_t max_moves, int64_t* moves) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < N; ++n) {
        int* c = (int*)malloc(sizeof(int) * K);
        double* unit = (double*)malloc(sizeof(double) * K);
        double* r = (double*)malloc(sizeof(double) * K);
        double* g = (double*)malloc(sizeof(double) * K);
        for (int64_t k = 0; k < K; ++k) {
            const uint8_t byte = codes[n * (K / 2) + k / 2];
            c[k] = (k & 1) ? byte >> 4 : byte & 15;
            unit[k] = ldexp(1.0, (int)scales[n * (K / 32) + k / 32] - 127);
            r[k] = kE2M1Line[e2m1_line_pos(c[k])] * unit[k] - (double)V[n * K + k];
        }
        for (int64_t j = 0; j < K; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc = fma(Hs[j * K + k], r[k], acc);
            g[j] = acc;
        }
        int64_t done = 0;
        while (done < max_moves) {
            double best = 0.0;
            int64_t bk = -1;
            int bp = 0;
            for (int64_t k = 0; k < K; ++k) {
                const int p = e2m1_line_pos(c[k]);
                for (int dir = -1; dir <= 1; dir += 2) {
                    const int q = p + dir;
                    if (q < 0 || q > 14) continue;
                    const double d = (kE2M1Line[q] - kE2M1Line[p]) * unit[k];
                    const double dl = d * fma(d, Hs[k * K + k], 2.0 * g[k]);
                    if (dl < best) {  /* strictly: ties keep the earlier candidate */
                        best = dl;
                        bk = k;
                        bp = q;
                    }
                }
            }
            if (bk < 0) break;  /* no move lowers the objective */
            const double d = (kE2M1Line[bp] - kE2M1Line[e2m1_line_pos(c[bk])]) * unit[bk];
            c[bk] = e2m1_code_at(bp, c[bk]);
            r[bk] = r[bk] + d;
            for (int64_t j = 0; j < K; ++j) g[j] = fma(d, Hs[j * K + bk], g[j]);
            ++done;
        }
        for (int64_t k = 0; k < K; k += 2) codes[n * (K / 2) + k / 2] = (uint8_t)(c[k] | (c[k + 1] << 4));
        moves[n] = done;
        free(c);
        free(unit);
        free(r);
        free(g);
    }
}

/* Per-channel scale from a calibration batch xcal [C][K] (bf16 values held in fp32) and the
 * weights W [N][K]: column maxima of |.|, then sqrt of their quotient in double, rounded once to
 * fp32; 1 for a column whose activation or weight maximum is zero. */
void oracle_calibrate_scale(const float* xcal, int64_t C, const float* W, int64_t N, int64_t K, float* s) {
    for (int64_t j = 0; j < K; ++j) {
        double ax = 0.0, aw = 0.0;
        for (int64_t r = 0; r < C; ++r) ax = fmax(ax, fabs((double)xcal[r * K + j]));
        for (int64_t n = 0; n < N; ++n) aw = fmax(aw, fabs((double)W[n * K + j]));
        s[j] = (ax == 0.0 || aw == 0.0) ? 1.0f : (float)sqrt(ax / aw);
    }
}

/* Number of OpenMP threads the oracle runs with (reported beside its timings). */
int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
