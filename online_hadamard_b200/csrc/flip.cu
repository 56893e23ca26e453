// flip.cu -- Flip-Refinement of the folded MXFP4 weight codes, and the calibration Hessian it uses.
//
// "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
// Activations", Abstract: Flip-Refinement starts from the round-to-nearest codes and runs a greedy
// coordinate descent, weighted by the Hessian, in which a step shifts one FP4 code to a
// neighbouring grid value.  The pages say no more; this library reads it as follows.
//   - It refines one layer's folded weight codes (macaq_fold_weights: round to nearest), keeping
//     every E8M0 block scale: only code nibbles change.
//   - Objective of output row n: L_n = (q_n - v_n) Hs (q_n - v_n)^T, the layer's output error on a
//     calibration batch, with q_n the decoded row, v_n the fp32 folded row before quantisation
//     (W diag(s) H_bd / sqrt(32), the fold's canonical fp32 transform), Hs = Xt^T Xt and Xt the
//     calibration activations after the online transform (fp32, before their quantisation).
//   - A move takes one code one step along the ordered line of the 15 E2M1 values -6 .. 6 (at
//     +-6 only inwards); a code that reaches zero keeps its sign bit.  Each step applies, in one
//     row, the move with the most negative dL = d (2 g_k + d Hs_kk) (g = Hs r, r = q - v, d the
//     value step times the block scale); ties go to the smaller k, then to the downward move.  A
//     row stops when no move lowers L, or after max_moves moves.
//   - fp64 in one fixed order, so every decision is reproducible: Hs[j][k] = fma chain over the
//     calibration rows in order; r_k = q_k - v_k; g_j = fma chain of Hs[j][k] r_k over k in
//     order; dL = d * fma(d, Hs_kk, 2 g_k); a move of code k by d updates g_j = fma(d, Hs[j][k], g_j).
//
// Kernels (offline; one layer at a time):
//   transform_f32_kernel   the online transform (activations) or the fold's (weights) in fp32,
//                          values kept: one thread per 32-element block, the quantiser's arithmetic
//   hessian_kernel         Hs = Xt^T Xt: 32 x 32 output tiles, the calibration rows streamed through
//                          shared memory, each output one fma chain in row order
//   flip_g_kernel          g for 8 weight rows x 256 outputs per CTA: each thread one output column
//                          for 8 rows, Hs read once per 8 rows, r computed while staging
//   flip_greedy_kernel     one CTA per weight row: g, codes and Hs's diagonal in shared memory; per
//                          step every thread scores its codes' two moves, a block-wide argmin picks
//                          the move, and the row of Hs updates g
#include <cstdint>
#include <cmath>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

constexpr int kFlipThreads = 256;
constexpr int64_t kFlipMaxK = 12288;   // g, the diagonal and the codes of one row fit in shared memory
constexpr int64_t kFlipChunkRows = 2048;

__device__ __constant__ double kLine[15] = {-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0,
                                            0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0};

__device__ __forceinline__ int line_pos(int code) {
    const int m = code & 7;
    return (code & 8) ? 7 - m : 7 + m;
}

__device__ __forceinline__ int code_at(int p, int old) {
    if (p == 7) return old & 8;
    return p > 7 ? p - 7 : 8 | (7 - p);
}

// 2^(e - 127) for an E8M0 byte (e <= 254: a normal double).
__device__ __forceinline__ double e8m0_unit(uint32_t e) {
    return __longlong_as_double(static_cast<long long>(static_cast<int64_t>(e) - 127 + 1023) << 52);
}

// Xt[r][k] for every row: activations (bf16, act_mult) or weights (fp32, multipliers fl32(s_k c)
// as in the fold), scale then the unnormalised FWHT-32, fp32 in the canonical order.
template <QuantMode MODE>
__global__ void __launch_bounds__(128) transform_f32_kernel(const void* __restrict__ in, int64_t R, int64_t K,
                                                            const float* __restrict__ mult,
                                                            const float* __restrict__ s, double c,
                                                            float* __restrict__ out) {
    const int64_t kb_real = K / 32;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (item >= R * kb_real) return;
    const int64_t r = item / kb_real, kb = item % kb_real, k0 = kb * 32;
    float2 m[16];
    if constexpr (MODE == QuantMode::kWeightFold) {
#pragma unroll
        for (int p = 0; p < 16; ++p)
            m[p] = make_float2(__double2float_rn(__dmul_rn(static_cast<double>(s[k0 + 2 * p]), c)),
                               __double2float_rn(__dmul_rn(static_cast<double>(s[k0 + 2 * p + 1]), c)));
    } else {
        const float4* mp = reinterpret_cast<const float4*>(mult + k0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = __ldg(mp + j);
            m[2 * j] = make_float2(t.x, t.y);
            m[2 * j + 1] = make_float2(t.z, t.w);
        }
    }
    RawBlock<MODE> raw;
    load_block<MODE>(in, r * K + k0, raw);
    float2 u[16];
    widen<MODE>(raw, u);
    scale_fwht32(u, m);
    float4* o = reinterpret_cast<float4*>(out + r * K + k0);
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = make_float4(u[2 * j].x, u[2 * j].y, u[2 * j + 1].x, u[2 * j + 1].y);
}

// Hs[j][k] = sum over c of Xt[c][j] Xt[c][k], one fma chain per output in calibration-row order.
// CTA: a 32 x 32 output tile, 256 threads x 4 outputs; rows staged 32 at a time.
__global__ void __launch_bounds__(kFlipThreads) hessian_kernel(const float* __restrict__ Xt, int64_t C, int64_t K,
                                                               double* __restrict__ Hs) {
    __shared__ double xj[32][33], xk[32][33];
    const int64_t j0 = static_cast<int64_t>(blockIdx.y) * 32, k0 = static_cast<int64_t>(blockIdx.x) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // output column k0 + tx, rows j0 + ty + 8 i
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t c0 = 0; c0 < C; c0 += 32) {
        for (int t = threadIdx.x; t < 32 * 32; t += kFlipThreads) {
            const int cr = t >> 5, col = t & 31;
            const bool ok = c0 + cr < C;
            xj[cr][col] = ok ? static_cast<double>(Xt[(c0 + cr) * K + j0 + col]) : 0.0;
            xk[cr][col] = ok ? static_cast<double>(Xt[(c0 + cr) * K + k0 + col]) : 0.0;
        }
        __syncthreads();
        const int n = C - c0 < 32 ? static_cast<int>(C - c0) : 32;
        for (int cr = 0; cr < n; ++cr) {
            const double b = xk[cr][tx];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = __fma_rn(xj[cr][ty + 8 * i], b, acc[i]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) Hs[(j0 + ty + 8 * i) * K + k0 + tx] = acc[i];
}

// g[n][j] = sum over k of Hs[j][k] r[n][k] (fma chain over k in order) for 8 rows x 256 columns;
// Hs[k][j] is read (the same bits: Hs is symmetric bit for bit), coalesced over j.
// r[n][k] = q - v: q the decoded code (exact), v the fp32 folded value.
__global__ void __launch_bounds__(kFlipThreads) flip_g_kernel(const float* __restrict__ V, const uint8_t* __restrict__ codes,
                                                              const uint8_t* __restrict__ scales, int64_t row0,
                                                              int64_t rows, int64_t K, const double* __restrict__ Hs,
                                                              double* __restrict__ G) {
    constexpr int kRows = 8, kChunk = 64;
    __shared__ double rs[kRows][kChunk];
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kRows;  // chunk-local first row
    const int64_t j = static_cast<int64_t>(blockIdx.x) * kFlipThreads + threadIdx.x;
    const int64_t kbp = padded_blocks(K);
    double acc[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) acc[i] = 0.0;
    for (int64_t k0 = 0; k0 < K; k0 += kChunk) {
        for (int t = threadIdx.x; t < kRows * kChunk; t += kFlipThreads) {
            const int i = t / kChunk, kk = t % kChunk;
            const int64_t n = n0 + i, k = k0 + kk;
            double r = 0.0;
            if (n < rows && k < K) {
                const int64_t gn = row0 + n;
                const uint8_t byte = codes[gn * (K / 2) + k / 2];
                const int code = (k & 1) ? byte >> 4 : byte & 15;
                const double unit = e8m0_unit(scales[scale_offset(gn, k / 32, kbp)]);
                r = __dsub_rn(__dmul_rn(kLine[line_pos(code)], unit), static_cast<double>(V[n * K + k]));
            }
            rs[i][kk] = r;
        }
        __syncthreads();
        if (j < K) {
            const int n = K - k0 < kChunk ? static_cast<int>(K - k0) : kChunk;
            for (int kk = 0; kk < n; ++kk) {
                const double h = Hs[(k0 + kk) * K + j];
#pragma unroll
                for (int i = 0; i < kRows; ++i) acc[i] = __fma_rn(h, rs[i][kk], acc[i]);
            }
        }
        __syncthreads();
    }
    if (j < K) {
#pragma unroll
        for (int i = 0; i < kRows; ++i)
            if (n0 + i < rows) G[(n0 + i) * K + j] = acc[i];
    }
}

// A candidate move: its dL, then the tie-break key 2 k + (upward ? 1 : 0).
struct Move {
    double dl;
    int key;
};

__device__ __forceinline__ bool better(const Move& a, const Move& b) {
    return a.dl < b.dl || (a.dl == b.dl && a.key < b.key);
}

// One CTA per weight row of the chunk: greedy moves until none lowers the objective or max_moves.
__global__ void __launch_bounds__(kFlipThreads) flip_greedy_kernel(const double* __restrict__ G,
                                                                   const uint8_t* __restrict__ scales, int64_t row0,
                                                                   int64_t K, const double* __restrict__ Hs,
                                                                   uint8_t* __restrict__ codes, int64_t max_moves,
                                                                   int32_t* __restrict__ moves) {
    extern __shared__ __align__(16) uint8_t fsm[];
    double* g = reinterpret_cast<double*>(fsm);
    double* diag = g + K;
    double* unit = diag + K;                              // one per 32-element block
    uint8_t* nib = reinterpret_cast<uint8_t*>(unit + K / 32);
    __shared__ Move warp_best[kFlipThreads / 32];
    __shared__ Move best_all;
    const int64_t n = blockIdx.x;
    const int64_t gn = row0 + n;
    const int64_t kbp = padded_blocks(K);
    for (int64_t k = threadIdx.x; k < K; k += kFlipThreads) {
        g[k] = G[n * K + k];
        diag[k] = Hs[k * K + k];
        const uint8_t byte = codes[gn * (K / 2) + k / 2];
        nib[k] = static_cast<uint8_t>((k & 1) ? byte >> 4 : byte & 15);
    }
    for (int64_t b = threadIdx.x; b < K / 32; b += kFlipThreads) unit[b] = e8m0_unit(scales[scale_offset(gn, b, kbp)]);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t done = 0;
    while (done < max_moves) {
        Move mine{INFINITY, 0x7FFFFFFF};
        for (int64_t k = threadIdx.x; k < K; k += kFlipThreads) {  // this thread's codes in order
            const int p = line_pos(nib[k]);
            const double gk2 = 2.0 * g[k];
#pragma unroll
            for (int dir = -1; dir <= 1; dir += 2) {
                const int q = p + dir;
                if (q < 0 || q > 14) continue;
                const double d = __dmul_rn(kLine[q] - kLine[p], unit[k >> 5]);
                const double dl = __dmul_rn(d, __fma_rn(d, diag[k], gk2));
                if (dl < mine.dl) mine = Move{dl, static_cast<int>(2 * k + (dir > 0 ? 1 : 0))};
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            Move o{__shfl_xor_sync(0xFFFFFFFFu, mine.dl, off), __shfl_xor_sync(0xFFFFFFFFu, mine.key, off)};
            if (better(o, mine)) mine = o;
        }
        if (lane == 0) warp_best[warp] = mine;
        __syncthreads();
        if (threadIdx.x == 0) {
            Move b = warp_best[0];
            for (int w = 1; w < kFlipThreads / 32; ++w)
                if (better(warp_best[w], b)) b = warp_best[w];
            best_all = b;
        }
        __syncthreads();
        const Move b = best_all;
        if (!(b.dl < 0.0)) break;  // no move lowers the objective (every thread sees the same b)
        const int64_t k = b.key >> 1;
        const int p = line_pos(nib[k]);
        const int q = p + ((b.key & 1) ? 1 : -1);
        const double d = __dmul_rn(kLine[q] - kLine[p], unit[k >> 5]);
        __syncthreads();  // every thread has read nib[k] before it changes
        if (threadIdx.x == 0) nib[k] = static_cast<uint8_t>(code_at(q, nib[k]));
        const double* hk = Hs + k * K;  // Hs[k][j] == Hs[j][k]
        for (int64_t j = threadIdx.x; j < K; j += kFlipThreads) g[j] = __fma_rn(d, hk[j], g[j]);
        ++done;
        __syncthreads();
    }
    for (int64_t k = 2 * threadIdx.x; k < K; k += 2 * kFlipThreads)
        codes[gn * (K / 2) + k / 2] = static_cast<uint8_t>(nib[k] | (nib[k + 1] << 4));
    if (threadIdx.x == 0 && moves) moves[gn] = static_cast<int32_t>(done);
}

static size_t flip_greedy_smem(int64_t K) { return static_cast<size_t>(K) * 17 + static_cast<size_t>(K / 32) * 8; }

}  // namespace macaq

using namespace macaq;

extern "C" size_t macaq_hessian_workspace_bytes(int64_t C, int64_t K) {
    if (check_shape(C, K) != MACAQ_OK) return 0;
    return static_cast<size_t>(C) * static_cast<size_t>(K) * 4;
}

extern "C" int macaq_calib_hessian(const uint16_t* xcal, int64_t C, int64_t K, const float* act_mult, double* Hs,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    if (!xcal || !act_mult || !Hs || !workspace) return MACAQ_EINVAL;
    if (int st = check_shape(C, K)) return st;
    if (!aligned16(xcal) || !aligned16(act_mult) || !aligned16(Hs) || !aligned16(workspace)) return MACAQ_EALIGN;
    if (workspace_bytes < macaq_hessian_workspace_bytes(C, K)) return MACAQ_EWORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* Xt = static_cast<float*>(workspace);
    const int64_t items = C * (K / 32);
    transform_f32_kernel<QuantMode::kActTransform><<<static_cast<unsigned>((items + 127) / 128), 128, 0, st>>>(
        xcal, C, K, act_mult, nullptr, 0.0, Xt);
    if (int rc = launch_status()) return rc;
    const dim3 grid(static_cast<unsigned>(K / 32), static_cast<unsigned>(K / 32));
    hessian_kernel<<<grid, kFlipThreads, 0, st>>>(Xt, C, K, Hs);
    return launch_status();
}

extern "C" size_t macaq_flip_refine_workspace_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K) != MACAQ_OK || K > kFlipMaxK) return 0;
    const int64_t rows = N < kFlipChunkRows ? N : kFlipChunkRows;
    return static_cast<size_t>(rows) * static_cast<size_t>(K) * 12;
}

extern "C" int macaq_flip_refine(const float* W, int64_t N, int64_t K, const float* s, const double* Hs, uint8_t* Wq,
                                 const uint8_t* Ws, int64_t max_moves, int32_t* moves, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    if (!W || !s || !Hs || !Wq || !Ws || !workspace || max_moves < 0) return MACAQ_EINVAL;
    if (int st = check_shape(N, K)) return st;
    if (K > kFlipMaxK) return MACAQ_ESHAPE;
    if (!aligned16(W) || !aligned16(s) || !aligned16(Hs) || !aligned16(Wq) || !aligned16(Ws) ||
        !aligned16(workspace) || (moves && !aligned16(moves)))
        return MACAQ_EALIGN;
    if (workspace_bytes < macaq_flip_refine_workspace_bytes(N, K)) return MACAQ_EWORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t smem = flip_greedy_smem(K);
    if (cudaFuncSetAttribute(flip_greedy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return MACAQ_ECUDA;
    const int64_t chunk = N < kFlipChunkRows ? N : kFlipChunkRows;
    float* V = static_cast<float*>(workspace);
    double* G = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + static_cast<size_t>(chunk) * K * 4);
    const double c = 1.0 / std::sqrt(32.0);  // correctly rounded, as in the fold
    for (int64_t r0 = 0; r0 < N; r0 += chunk) {
        const int64_t rows = N - r0 < chunk ? N - r0 : chunk;
        const int64_t items = rows * (K / 32);
        transform_f32_kernel<QuantMode::kWeightFold><<<static_cast<unsigned>((items + 127) / 128), 128, 0, st>>>(
            W + r0 * K, rows, K, nullptr, s, c, V);
        if (int rc = launch_status()) return rc;
        const dim3 ggrid(static_cast<unsigned>((K + kFlipThreads - 1) / kFlipThreads), static_cast<unsigned>((rows + 7) / 8));
        flip_g_kernel<<<ggrid, kFlipThreads, 0, st>>>(V, Wq, Ws, r0, rows, K, Hs, G);
        if (int rc = launch_status()) return rc;
        flip_greedy_kernel<<<static_cast<unsigned>(rows), kFlipThreads, smem, st>>>(G, Ws, r0, K, Hs, Wq, max_moves,
                                                                                     moves);
        if (int rc = launch_status()) return rc;
    }
    return MACAQ_OK;
}
