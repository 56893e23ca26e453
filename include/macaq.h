/*
 * macaq.h -- C ABI of libmacaq: the inference hot path of MACaQ's layer-local MXFP4 W4A4
 * linear layer on NVIDIA B200 (sm_100a).
 *
 * Method: "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights
 * and Activations" (arXiv 2611.10649), Abstract: no linear layer depends on another; at
 * inference the activations of a layer are scaled channel by channel and rotated by a
 * block Hadamard, and the inverse of both is folded into the same layer's weights; both
 * operands are MXFP4 (W4A4), the weights rounded to nearest.  The pages leave the details
 * open; this library fixes them as follows.
 *
 *   Notation.  x is bf16 [M][K] row-major, W is fp32 [N][K] row-major (y = x W^T, the
 *   nn.Linear layout), s is fp32 [K] with s_k > 0 finite.  c = 1/sqrt(32).
 *   Block-Hadamard: blocks of b = 32 consecutive k, Sylvester order
 *   H[i][j] = (-1)^popcount(i&j), applied unnormalised; its 1/sqrt(32) goes into one fp32
 *   multiplier per channel:  act_mult[k] = fl32(c / s_k),  w_mult[k] = fl32(s_k * c).
 *   Activations are divided by s, weights multiplied by s, so that
 *   (x diag(1/s) H/sqrt32)(W diag(s) H/sqrt32)^T = x W^T.
 *   Transform (fp32, one canonical order): u_k = fl32(x_k * mult_k), then butterfly stages
 *   h = 1, 2, 4, 8, 16 replacing (u_i, u_{i+h}) by (u_i + u_{i+h}, u_i - u_{i+h}).
 *   MXFP4 (OCP Microscaling v1.0): per 32-block, E8M0 scale byte e = max(E(amax) - 2, 0)
 *   where E(amax) is the biased fp32 exponent of the block's largest |v| (e never reaches
 *   0xFF); element code = (sign << 3) | index of v * 2^(127-e) rounded to the nearest of
 *   {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even index, saturating at 6; the IEEE sign
 *   is kept, so a negative value rounding to zero is code 0x8.
 *
 * Data layouts (all sizes in bytes, all buffers caller-allocated and caller-owned):
 *
 *   MXFP4 codes   uint8 [rows][K/2]: element k of a row sits in byte k/2, low nibble
 *                 when k is even.
 *   E8M0 scales   "MMA tile layout": uint8, macaq_scale_bytes(rows, K) bytes.  Rows are
 *                 padded to a multiple of 128 and the K/32 blocks of a row to a multiple
 *                 of 8; the byte of (row r, block kb) is at macaq_scale_offset(r, kb, K) =
 *                   ((r/128) * (KBp/4) + kb/4) * 512 + (r%32)*16 + ((r/32)%4)*4 + kb%4,
 *                 KBp = 8 * ceil(K/256).  Each 512-byte atom holds 4 blocks of 128 rows in
 *                 the order the tensor cores' scale-factor copy expects.  Writers fill the
 *                 padded blocks of real rows with 0; bytes of padded rows are never used
 *                 for a stored output and may hold anything.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers on the current CUDA device, 16-byte aligned;
 *     otherwise MACAQ_EALIGN.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - M, N >= 1, 32 <= K, K % 32 == 0, and M, N, K < 2^31; otherwise MACAQ_ESHAPE.
 *   - The calls validate, enqueue kernels on `stream` and return; the return value is the
 *     validation/launch status.  Errors of the asynchronous work surface at the next
 *     synchronisation; a device-side wait that gives up (it never should) sets a flag
 *     that macaq_device_status() reports.  No call allocates device memory: scratch is
 *     passed in by the caller, or, for macaq_w4a4_linear_noalloc, held in a static array
 *     of the library.
 *   - Non-finite activations or weights are out of scope (codes are then unspecified).
 */
#ifndef MACAQ_H_
#define MACAQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MACAQ_OK = 0,
    MACAQ_EINVAL = -1,     /* null pointer, non-finite or non-positive s, bad flag */
    MACAQ_ESHAPE = -2,     /* M, N, K out of range or K % 32 != 0 */
    MACAQ_EALIGN = -3,     /* a pointer is not 16-byte aligned */
    MACAQ_ECUDA = -4,      /* a CUDA runtime call or kernel launch failed */
    MACAQ_ETIMEOUT = -5,   /* a bounded device-side wait gave up (see macaq_device_status) */
    MACAQ_EWORKSPACE = -6, /* workspace smaller than the call needs */
    MACAQ_ETOOLARGE = -7,  /* problem needs more than the no-allocation scratch (below) */
    MACAQ_ECOUNTS = -8     /* device routing counts were corrected or capped (macaq_w4a4_grouped_linear_device) */
} macaq_status;

/* Human-readable name of a status code (static storage). */
const char* macaq_status_str(int status);

/* Bytes of an E8M0 scale buffer in the MMA tile layout for `rows` x K elements
 * (0 on invalid arguments). */
size_t macaq_scale_bytes(int64_t rows, int64_t K);

/* Offset of the scale byte of (row r, 32-block kb) in that buffer (-1 if out of range). */
int64_t macaq_scale_offset(int64_t r, int64_t kb, int64_t K);

/* Conversions between row-major E8M0 scales, uint8 [rows][K/32] (the layout most MXFP4 producers
 * write), and the MMA tile layout above (macaq_scale_bytes(rows, K) bytes), on the device, for
 * callers that quantise activations or weights elsewhere.  To the tile layout, the padded blocks of
 * real rows and the padded rows are written as 0; back, only the real rows and blocks are written.
 * Asynchronous on `stream`; MACAQ_EINVAL for a null pointer, MACAQ_ESHAPE as for the other calls. */
int macaq_scales_to_tiled(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* tiled, void* stream);
int macaq_scales_to_rowmajor(const uint8_t* tiled, int64_t rows, int64_t K, uint8_t* rowmajor, void* stream);

/* Bytes of scratch macaq_mxfp4_gemm uses for its stream-K schedule on the current device
 * (256 eight-byte flag words and a 128-row fp32 partial-sum slot per CTA of the persistent
 * grid; depends on M and the device's SM count).  The scratch needs no initialisation: a
 * flag word counts as written only when it holds the tag of the current launch, and the
 * launch clears the words it consumed, so calls captured in a CUDA graph may be replayed. */
size_t macaq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Bytes of scratch macaq_w4a4_linear (and macaq_mxfp4_linear) needs on the current device:
 * the activations' MXFP4 codes (M*K/2) and scales (macaq_scale_bytes(M, K)), each rounded
 * up to 256, then macaq_gemm_workspace_bytes(M, N, K). */
size_t macaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * macaq_calibrate_scale -- the per-channel scale s before the fold (Abstract: the method is
 * calibrated per layer; the pages give no rule).  The rule used is the SmoothQuant 1/2
 * balance: s_j = fl32(sqrt(max_r |xcal_rj| / max_n |W_nj|)), quotient and root in IEEE double
 * (correctly rounded), s_j = 1 where either maximum is 0; afterwards max|x_j / s_j| and
 * max|W_nj * s_j| agree.
 *   xcal  in   bf16 bit patterns [C][K], a calibration batch of activations
 *   W     in   fp32 [N][K]
 *   s     out  fp32 [K]; usable by macaq_fold_weights as is
 * Offline, asynchronous on `stream` (a memset and two kernels; reads W once).  NaN or infinite
 * inputs give undefined s.  MACAQ_ESHAPE for K % 32 != 0, C or N out of range.
 */
int macaq_calibrate_scale(const uint16_t* xcal, int64_t C, const float* W, int64_t N, int64_t K,
                          float* s, void* stream);

/*
 * macaq_fold_weights -- offline weight preparation (Abstract: the inverse of the activation
 * transforms is folded into the layer's weights, which are then rounded to nearest).
 *   W        in   fp32 [N][K]
 *   s        in   fp32 [K], every s_k finite and > 0 (else MACAQ_EINVAL, nothing written)
 *   Wq       out  MXFP4 codes [N][K/2] of W' = W diag(s) H_bd / sqrt(32)
 *   Ws       out  E8M0 scales of W', MMA tile layout, macaq_scale_bytes(N, K) bytes
 *   act_mult out  fp32 [K], fl32(c / s_k): the online activation multiplier
 * This offline call copies s to the host to validate it and therefore synchronises
 * `stream`; the hot-path calls below never synchronise.
 */
int macaq_fold_weights(const float* W, int64_t N, int64_t K, const float* s, uint8_t* Wq,
                       uint8_t* Ws, float* act_mult, void* stream);

/*
 * macaq_act_transform_quant -- the online activation transform (Abstract: the layer's
 * activations are scaled per channel and rotated by a block Hadamard at inference time)
 * followed by MXFP4 quantisation (the A4 of W4A4).
 *   x        in   bf16 bit patterns [M][K]
 *   act_mult in   fp32 [K] (from macaq_fold_weights)
 *   Aq       out  MXFP4 codes [M][K/2]
 *   As       out  E8M0 scales, MMA tile layout, macaq_scale_bytes(M, K) bytes
 */
int macaq_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                              uint8_t* Aq, uint8_t* As, void* stream);

/*
 * macaq_w4a4_linear -- the layer's forward pass, y = x W^T computed as
 * MXFP4(x diag(act_mult) H) . MXFP4(W')^T (Abstract; the 2.3 % end-to-end cost the pages give
 * against MXFP4 without transforms is that of this online transform): the activation transform and
 * MXFP4 quantisation kernel writes the activations' codes and scales into the workspace,
 * then the block-scaled MXFP4 x MXFP4 GEMM (launched as a programmatic dependent of it)
 * contracts them on the tensor cores with fp32 accumulation and rounds y to bf16 (RNE).
 * Codes, scales and y are identical to those of macaq_act_transform_quant followed by
 * macaq_mxfp4_gemm with a workspace.
 *   x         in   bf16 [M][K];  act_mult in fp32 [K]
 *   Wq, Ws    in   folded weights from macaq_fold_weights (N rows)
 *   y         out  bf16 [M][N]
 *   workspace in   scratch of at least macaq_linear_workspace_bytes(M, N, K) bytes
 *                  (MACAQ_EWORKSPACE otherwise); its contents on entry and on return are
 *                  unspecified and calls sharing one workspace must be stream-ordered.
 */
int macaq_w4a4_linear(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                      const uint8_t* Wq, const uint8_t* Ws, int64_t N, uint16_t* y,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Baselines and building blocks (not part of the method; used to measure the overhead of
 * the online transform against "pure MXFP4", Abstract).
 *
 * macaq_act_quant_plain: MXFP4 quantisation of x with no scale and no transform.
 * macaq_mxfp4_linear: the plain MXFP4 linear layer, y = dec(MXFP4(x)) dec(Wq)^T in bf16,
 *   run exactly like macaq_w4a4_linear (same kernels, same workspace size and rules)
 *   without the per-channel scale and the Hadamard transform: the "pure MXFP4" against
 *   which the transform's overhead is measured.
 * macaq_mxfp4_gemm: y = dec(A) dec(W)^T for already-quantised operands, fp32 accumulate;
 *   y is bf16 [M][N] (y_is_fp32 = 0) or fp32 [M][N] (y_is_fp32 = 1).  With a workspace of
 *   macaq_gemm_workspace_bytes(M, N, K) the GEMM balances its last wave with a stream-K
 *   split of the K steps (partial sums added in a fixed order, so results are
 *   deterministic); with workspace = NULL it runs a data-parallel schedule.  Both
 *   schedules accumulate in fp32 and agree within fp32 summation order.  The workspace's
 *   contents on entry and on return are unspecified; calls sharing one workspace must be
 *   stream-ordered.
 */
int macaq_act_quant_plain(const uint16_t* x, int64_t M, int64_t K, uint8_t* Aq, uint8_t* As,
                          void* stream);
int macaq_mxfp4_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wq, const uint8_t* Ws,
                       int64_t N, uint16_t* y, void* workspace, size_t workspace_bytes, void* stream);
int macaq_mxfp4_gemm(const uint8_t* Aq, const uint8_t* As, int64_t M, const uint8_t* Wq,
                     const uint8_t* Ws, int64_t N, int64_t K, void* y, int y_is_fp32,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * macaq_w4a4_linear_multi -- G linear layers on the same activations x, e.g. the q, k and v
 * projections of an attention block or the gate and up projections of an MLP.  Each is its own
 * layer with its own per-channel scale and folded weights (the method is layer-local, Abstract),
 * so x is transformed and quantised once per layer, in ONE launch; then ONE GEMM runs over the
 * layers' weights stacked by rows, each weight tile against its own layer's activations: up to
 * 128 tokens swap-AB (128-row weight tiles), above on CTA pairs (256-row weight tiles) when every
 * N[g] is a multiple of 256; otherwise one GEMM per layer.
 *   x         in   bf16 [M][K]
 *   act_mult  in   fp32 [G][K], layer g's multipliers from macaq_fold_weights at g*K; NULL: plain
 *                  MXFP4 of x, quantised once and shared (the "pure MXFP4" baseline)
 *   Wq, Ws    in   the layers' folded weights stacked in order g = 0..G-1: codes [sum N][K/2],
 *                  scales the G buffers of macaq_scale_bytes(N[g], K) bytes one after another
 *   N         in   HOST int64 [G], 1 <= G <= 128, every N[g] a positive multiple of 128
 *   y         out  bf16 [M][sum N]: layer g's outputs in columns N[0] + .. + N[g-1] onwards
 *   workspace in   at least macaq_linear_multi_workspace_bytes(M, G, K) bytes.  With Mp = M
 *                  rounded up to a multiple of 128, layer g's activation codes [M][K/2] are left
 *                  at byte g*Mp*K/2 and their scales (MMA tile layout) at byte A + g *
 *                  macaq_scale_bytes(Mp, K), A = G*Mp*K/2 rounded up to 256 (act_mult NULL: the
 *                  one shared set at g = 0); the GEMM's stream-K scratch follows.  Other bytes
 *                  are unspecified on return; calls sharing it must be stream-ordered
 * Layer g's activation codes and scales equal those of macaq_act_transform_quant(x, act_mult +
 * g*K) bit for bit, and its y columns equal macaq_w4a4_linear's within the GEMM tolerance (the
 * stacked launch may split the K steps differently).  MACAQ_ESHAPE for G or an N[g] out of range.
 */
size_t macaq_linear_multi_workspace_bytes(int64_t M, int G, int64_t K);
int macaq_w4a4_linear_multi(const uint16_t* x, int64_t M, int64_t K, int G, const float* act_mult,
                            const uint8_t* Wq, const uint8_t* Ws, const int64_t* N, uint16_t* y,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * macaq_w4a4_grouped_linear -- a grouped (mixture-of-experts) W4A4 linear: E experts, each its
 * own layer with its own per-channel scale and block-Hadamard transform folded into its weights
 * (the method is layer-local, Abstract; the pages name MoE models among its targets), all of
 * them computed in two launches -- a grouped transform + quantisation, then a grouped GEMM.
 *   x         in   bf16 [T][K], the tokens grouped by expert: expert e's counts[e] rows follow
 *                  expert e-1's (T = sum of counts)
 *   counts    in   HOST int64 [E], tokens per expert (>= 0, zeros allowed), 1 <= E <= 128
 *   act_mult  in   fp32 [E][K], expert e's multipliers from macaq_fold_weights; NULL: plain
 *                  MXFP4 of x (the "pure MXFP4" baseline, no scale and no transform)
 *   Wq, Ws    in   the experts' folded weights stacked: codes [E][N][K/2], scales the E buffers
 *                  of macaq_scale_bytes(N, K) bytes one after another; N % 128 == 0
 *   y         out  bf16 [T][N], row t the output of token t's expert
 *   workspace in   at least macaq_grouped_workspace_bytes(counts, E, N, K) bytes (the activation
 *                  codes and scales, each expert padded to whole 128-row blocks); contents on
 *                  entry and on return unspecified; calls sharing it must be stream-ordered
 * Experts with up to 128 tokens each run swap-AB (weights as the 128-row MMA operand); larger
 * ones 128-token x 256-feature tiles.  y and the codes match the per-expert linear's (codes bit
 * for bit).  Returns MACAQ_OK without launching when T == 0.
 */
size_t macaq_grouped_workspace_bytes(const int64_t* counts, int E, int64_t N, int64_t K);
int macaq_w4a4_grouped_linear(const uint16_t* x, const int64_t* counts, int E, int64_t K,
                              const float* act_mult, const uint8_t* Wq, const uint8_t* Ws,
                              int64_t N, uint16_t* y, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * macaq_w4a4_grouped_linear_device -- macaq_w4a4_grouped_linear with the per-expert token counts in
 * DEVICE memory, as a router on the GPU produces them: nothing is copied to the host and the call
 * never synchronises.  A first kernel builds the expert table on the device, then the grouped
 * quantiser and GEMM run from it; grids and the workspace are sized on the host from T, E and the
 * capacity.
 *   x         in   bf16 [T][K], the tokens grouped by expert (T, the routed rows, known on the host)
 *   counts    in   DEVICE int32 (counts_bytes = 4) or int64 (8) [E], 1 <= E <= 128
 *   capacity  in   the most rows any expert may have (an expert capacity, known on the host: e.g. the
 *                  token count for top-k routing to distinct experts); <= 0 or > T means T.  It
 *                  picks the kernels: up to 128, the weights take the MMA's 128-row side (swap-AB,
 *                  N of the narrowest tile holding the capacity); above, 128-token x 256-feature tiles
 *   act_mult, Wq, Ws, N, y   as for macaq_w4a4_grouped_linear
 *   workspace in   at least macaq_grouped_device_workspace_bytes(T, E, N, K) bytes (the table and
 *                  activation codes for the most padded rows T tokens can need: T + 127 min(E, T))
 * Counts are expected to be >= 0, at most the capacity, and to sum to T.  A negative count is taken
 * as 0, a count that would run past row T is cut there, and an expert's rows beyond the capacity are
 * not computed (x keeps its layout); each of these sets MACAQ_ECOUNTS in macaq_device_status.  Rows
 * of y that are not computed are not written.  Results match macaq_w4a4_grouped_linear within the
 * GEMM tolerance (its kernel choice follows the largest expert, this one the capacity), activation
 * codes bit for bit.
 */
size_t macaq_grouped_device_workspace_bytes(int64_t T, int E, int64_t N, int64_t K);
int macaq_w4a4_grouped_linear_device(const uint16_t* x, int64_t T, const void* counts, int counts_bytes, int E,
                                     int64_t capacity, int64_t K, const float* act_mult, const uint8_t* Wq,
                                     const uint8_t* Ws, int64_t N, uint16_t* y, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * macaq_w4a4_linear_noalloc -- macaq_w4a4_linear for callers that cannot allocate device
 * memory.  The paper has no counterpart: it is a deployment variant of the call above.
 *
 * cudaMalloc synchronises the device and can fail or fragment memory at run time, so a
 * latency-critical serving loop that plans all of its memory up front must not call it, a
 * plugin whose host application owns every device allocation has no allocator to call,
 * and a plain C caller handed only device pointers for its inputs and outputs cannot
 * obtain a buffer.  This call therefore allocates nothing: the activation codes and scales
 * go to a static device array of MACAQ_NOALLOC_SCRATCH_BYTES inside the library, present
 * on every GPU that loads the library until the process exits.
 *   Arguments, layouts and results are those of macaq_w4a4_linear (without workspace).
 *   MACAQ_ETOOLARGE (nothing launched) when the activations' codes and scales (the first
 *   part of macaq_linear_workspace_bytes(M, N, K)) exceed MACAQ_NOALLOC_SCRATCH_BYTES; the
 *   GEMM uses its stream-K schedule when the whole workspace fits, else its data-parallel
 *   one.
 *   All calls share the one array and it keeps the previous call's contents; each call
 *   writes everything it later reads, so nothing needs clearing, but calls whose work
 *   overlaps on the GPU (unordered streams, concurrent host threads) race on it and
 *   corrupt each other's results -- order them on one stream.
 *   The first call on a device looks up the array's device address once
 *   (cudaGetSymbolAddress, with that device current); make that first call before any
 *   CUDA stream capture begins.
 */
#define MACAQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int macaq_w4a4_linear_noalloc(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                              const uint8_t* Wq, const uint8_t* Ws, int64_t N, uint16_t* y,
                              void* stream);

/*
 * Flip-Refinement (Abstract: a greedy coordinate descent, weighted by the Hessian, that shifts
 * single FP4 codes to a neighbouring grid value, starting from round-to-nearest).  An
 * offline step between macaq_fold_weights and inference; the pages give no more, and this library
 * reads it as follows (details in csrc/flip.cu):
 *   objective of weight row n:  L_n = (q_n - v_n) Hs (q_n - v_n)^T, q_n the decoded codes, v_n the
 *   fp32 folded row before quantisation, Hs = Xt^T Xt with Xt a calibration batch after the online
 *   transform; the E8M0 block scales stay as the fold set them; a move takes one code one step
 *   along the ordered E2M1 values -6 .. 6 (a code reaching zero keeps its sign bit); each step
 *   applies the row's single most-improving move (ties: smaller k, then downward); a row stops when
 *   no move lowers L or after max_moves moves.  All of it in fp64 in one fixed order, so the
 *   result is deterministic.
 *
 * macaq_calib_hessian -- Hs (fp64 [K][K], symmetric bit for bit) of a calibration batch.
 *   xcal      in   bf16 bit patterns [C][K] (the layer's calibration activations)
 *   act_mult  in   fp32 [K], the layer's multipliers (macaq_fold_weights)
 *   Hs        out  fp64 [K][K] = Xt^T Xt, Xt[c][k] the fp32 online transform of xcal (scale and
 *                  FWHT-32, as macaq_act_transform_quant computes it before quantising); each
 *                  entry an fma chain over the calibration rows in order
 *   workspace in   macaq_hessian_workspace_bytes(C, K) bytes (Xt, fp32)
 * macaq_flip_refine -- refine folded weight codes in place.
 *   W, s      in   the layer's fp32 weights [N][K] and per-channel scale [K] (as given to
 *                  macaq_fold_weights)
 *   Hs        in   from macaq_calib_hessian
 *   Wq        in/out  round-to-nearest codes [N][K/2] from macaq_fold_weights; refined on return
 *   Ws        in   their scales (unchanged)
 *   max_moves in   moves per row at most (>= 0)
 *   moves     out  int32 [N], moves applied per row (device; NULL: not reported)
 *   workspace in   macaq_flip_refine_workspace_bytes(N, K) bytes
 *   K <= 12288 (one row's state lives in shared memory), else MACAQ_ESHAPE.
 */
size_t macaq_hessian_workspace_bytes(int64_t C, int64_t K);
int macaq_calib_hessian(const uint16_t* xcal, int64_t C, int64_t K, const float* act_mult, double* Hs,
                        void* workspace, size_t workspace_bytes, void* stream);
size_t macaq_flip_refine_workspace_bytes(int64_t N, int64_t K);
int macaq_flip_refine(const float* W, int64_t N, int64_t K, const float* s, const double* Hs, uint8_t* Wq,
                      const uint8_t* Ws, int64_t max_moves, int32_t* moves, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Sticky device-side status of the current device: MACAQ_OK; MACAQ_ETIMEOUT once a bounded
 * wait inside a kernel gave up; MACAQ_ECOUNTS once device routing counts had to be corrected (the
 * last event recorded wins).  Synchronises the device.  `clear` != 0 resets it. */
int macaq_device_status(int clear);

#ifdef __cplusplus
}
#endif

#endif /* MACAQ_H_ */
