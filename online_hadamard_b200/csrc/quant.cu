// quant.cu -- MXFP4 quantisation kernels along K, with the online MACaQ transform.
//
//   act_transform: u = fl32(x * act_mult), block-Hadamard b = 32 (FWHT in registers),
//                  E8M0 scale, E2M1 RTN codes                       (activations, online)
//   weight_fold:   u = fl32(W * fl32(s * c)), same transform and quantisation (weights,
//                  offline; also writes act_mult = fl32(c / s))
//   plain:         MXFP4 of x with no scale and no transform       (baseline)
//
// "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
// Activations", Abstract: per-channel scale + block-Hadamard online on the activations,
// inverse transforms absorbed into the weights, MXFP4 W4A4, round-to-nearest weights.
//
// Work split (large inputs): one thread owns one 32-element block column and walks a group of rows, so
// its 32 multipliers stay in registers and the whole 32-point butterfly runs in its
// registers with no cross-lane traffic.  A warp covers 32 consecutive blocks (2 KB of
// bf16) of one row: its four 16-byte loads per row touch every sector of that span, and
// its 16-byte code stores are contiguous.  Two rows are loaded before either is used to
// keep enough bytes in flight (on inputs of 16 M elements and more the transform instead
// processes one row while loading the next); the launch bound holds the kernel to four CTAs of 128 per SM,
// the grid the rows are divided for, and lets the compiler use all 128 registers a thread
// has there (the plain quantiser measured 5-12 % faster for it on large inputs).  Every fp32
// operation is an explicit round-to-nearest
// intrinsic (scalar or the sm_100 packed f32x2 form), so the scale cannot be contracted
// into the first butterfly and the result is bit-identical to the canonical sequential
// order.  The kernel is HBM-bound: 2 (or 4) bytes in, 0.53 bytes out per element.
//
// Small activation inputs (decode, short prefill) are bound by latency instead: few threads,
// each with a long serial chain of loads and transform arithmetic.  There the transform runs
// with two threads per block (mx_quant_half_kernel below): half the registers and half the
// serial work per thread, twice the threads in flight.  Its extra shuffles make it slower
// once the input fills the GPU, so the launch picks the kernel by input size.
#include <cstdint>
#include <cmath>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

enum class QuantMode { kActTransform = 0, kWeightFold = 1, kPlain = 2 };

constexpr int kQuantThreads = 128;

// Eight E2M1 codes of q0..q7 packed two per byte, element 2j in the low nibble:
// cvt.rn.satfinite.e2m1x2 puts its first source in the high nibble.  The conversion keeps the
// IEEE sign, so a negative value that rounds to zero becomes code 0x8 (-0).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float2 q0, float2 q1, float2 q2, float2 q3) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q0.x), "f"(q0.y), "f"(q1.x), "f"(q1.y), "f"(q2.x), "f"(q2.y), "f"(q3.x), "f"(q3.y));
    return out;
}

// a - b on both lanes of a float pair, one round-to-nearest rounding each (sm_100 packed op).
__device__ __forceinline__ float2 fsub2_rn(float2 a, float2 b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
    return *reinterpret_cast<const float2*>(&d);
}

// max(a, b, c) of three floats (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 32 raw inputs of one block as 16 pairs (bf16 widened exactly, or fp32).
template <QuantMode MODE>
struct RawBlock {
    uint4 w[MODE == QuantMode::kWeightFold ? 8 : 4];
};

template <QuantMode MODE>
__device__ __forceinline__ void load_block(const void* __restrict__ in, int64_t off, RawBlock<MODE>& b) {
    if constexpr (MODE == QuantMode::kWeightFold) {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(in) + off);
#pragma unroll
        for (int j = 0; j < 8; ++j) b.w[j] = __ldcs(p + j);
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in) + off);
#pragma unroll
        for (int j = 0; j < 4; ++j) b.w[j] = __ldcs(p + j);
    }
}

template <QuantMode MODE>
__device__ __forceinline__ void widen(const RawBlock<MODE>& b, float2 (&u)[16]) {
    if constexpr (MODE == QuantMode::kWeightFold) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            u[2 * j] = make_float2(__uint_as_float(b.w[j].x), __uint_as_float(b.w[j].y));
            u[2 * j + 1] = make_float2(__uint_as_float(b.w[j].z), __uint_as_float(b.w[j].w));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w[4] = {b.w[j].x, b.w[j].y, b.w[j].z, b.w[j].w};
#pragma unroll
            for (int t = 0; t < 4; ++t)  // bf16 -> fp32 is exact: the bits move up 16 places
                u[4 * j + t] = make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xFFFF0000u));
        }
    }
}

// Scale by the per-channel multiplier and apply the unnormalised 32-point Walsh-Hadamard
// butterfly in the canonical stage order h = 1, 2, 4, 8, 16.  u[p] holds elements 2p, 2p+1.
__device__ __forceinline__ void scale_fwht32(float2 (&u)[16], const float2 (&m)[16]) {
#pragma unroll
    for (int p = 0; p < 16; ++p) u[p] = __fmul2_rn(u[p], m[p]);
#pragma unroll
    for (int p = 0; p < 16; ++p) {  // h = 1: the two halves of a pair
        const float a = u[p].x, b = u[p].y;
        u[p] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < 16; hp <<= 1) {  // h = 2 hp: whole pairs, packed
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            if ((p & hp) == 0) {
                const float2 a = u[p], b = u[p + hp];
                u[p] = __fadd2_rn(a, b);
                u[p + hp] = fsub2_rn(a, b);
            }
        }
    }
}

// E8M0 scale byte and the 16 code bytes of one transformed block.  Dividing by the scale
// 2^(e - 127) is an exact multiplication by 2^(127 - e) (both normal floats).
__device__ __forceinline__ uint32_t quantize32(const float2 (&v)[16], uint4& codes) {
    const float* f = reinterpret_cast<const float*>(v);  // the 32 values in order
    float amax = fmax3(fabsf(f[0]), fabsf(f[1]), fabsf(f[2]));
#pragma unroll
    for (int i = 3; i + 1 < 32; i += 2) amax = fmax3(amax, fabsf(f[i]), fabsf(f[i + 1]));
    amax = fmaxf(amax, fabsf(f[31]));
    const uint32_t E = (__float_as_uint(amax) >> 23) & 0xFFu;
    const uint32_t e = E >= 3u ? E - 2u : 0u;
    const float inv = __uint_as_float((254u - e) << 23);  // 2^(127 - e), a normal float
    const float2 inv2 = make_float2(inv, inv);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2* q = v + 4 * j;
        w[j] = cvt_e2m1x8(__fmul2_rn(q[0], inv2), __fmul2_rn(q[1], inv2), __fmul2_rn(q[2], inv2),
                          __fmul2_rn(q[3], inv2));
    }
    codes = make_uint4(w[0], w[1], w[2], w[3]);
    return e;
}

template <QuantMode MODE>
__device__ __forceinline__ void process_block(const RawBlock<MODE>& raw, const float2 (&m)[16], uint8_t* codes_row,
                                              uint8_t* scale_byte) {
    float2 u[16];
    widen<MODE>(raw, u);
    if constexpr (MODE != QuantMode::kPlain) scale_fwht32(u, m);
    uint4 c;
    const uint32_t e = quantize32(u, c);
    *reinterpret_cast<uint4*>(codes_row) = c;
    *scale_byte = static_cast<uint8_t>(e);
}

// Quantise one 32-block column (kb) of n consecutive rows: input row in0 + i becomes output
// row out0 + i.  AHEAD = false: rows go two at a time, both loaded before either is used.
// AHEAD = true: one row is processed while the next row's load is in flight (the transform on
// large inputs: 5-7 % faster there, measured; slower for the plain quantiser and small inputs).
template <QuantMode MODE, bool AHEAD = false>
__device__ __forceinline__ void quant_rows(const void* __restrict__ in, int64_t K, int64_t in0, int64_t out0,
                                           int64_t n, int64_t kb, int64_t kbp, const float2 (&m)[16],
                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    const int64_t k0 = kb * 32;
    if constexpr (AHEAD) {
        RawBlock<MODE> cur;
        load_block<MODE>(in, in0 * K + k0, cur);
        for (int64_t i = 0; i < n; ++i) {
            RawBlock<MODE> nxt = cur;
            if (i + 1 < n) load_block<MODE>(in, (in0 + i + 1) * K + k0, nxt);
            const int64_t o = out0 + i;
            process_block<MODE>(cur, m, codes + o * (K / 2) + kb * 16, scales + scale_offset(o, kb, kbp));
            cur = nxt;
        }
        return;
    }
    int64_t i = 0;
    for (; i + 1 < n; i += 2) {
        RawBlock<MODE> b0, b1;
        load_block<MODE>(in, (in0 + i) * K + k0, b0);
        load_block<MODE>(in, (in0 + i + 1) * K + k0, b1);
        const int64_t o = out0 + i;
        process_block<MODE>(b0, m, codes + o * (K / 2) + kb * 16, scales + scale_offset(o, kb, kbp));
        process_block<MODE>(b1, m, codes + (o + 1) * (K / 2) + kb * 16, scales + scale_offset(o + 1, kb, kbp));
    }
    if (i < n) {
        RawBlock<MODE> b0;
        load_block<MODE>(in, (in0 + i) * K + k0, b0);
        process_block<MODE>(b0, m, codes + (out0 + i) * (K / 2) + kb * 16, scales + scale_offset(out0 + i, kb, kbp));
    }
}

// One thread = (run of `rpg` rows) x (one 32-block column), columns fastest; threads of
// padded block columns (kb >= K/32) write the zero scale bytes of their rows.
template <QuantMode MODE, bool AHEAD = false>
__global__ void __launch_bounds__(kQuantThreads, 4) mx_quant_kernel(
    const void* __restrict__ in, int64_t R, int64_t K, int64_t rpg, const float* __restrict__ mult,
    const float* __restrict__ s, double c, float* __restrict__ act_mult_out, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
    griddep_launch_dependents();
    griddep_wait();  // x (and this workspace) may be written / still read by the preceding kernel
    const int64_t kb_real = K / 32;
    const int64_t kbp = padded_blocks(K);
    const int64_t item = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
    const int64_t kb = item % kbp;
    const int64_t r0 = (item / kbp) * rpg;
    if (r0 >= R) return;
    const int64_t n = r0 + rpg < R ? rpg : R - r0;
    if (kb >= kb_real) {
        for (int64_t r = r0; r < r0 + n; ++r) scales[scale_offset(r, kb, kbp)] = 0;
        return;
    }
    const int64_t k0 = kb * 32;
    float2 m[16];
    if constexpr (MODE == QuantMode::kActTransform) {
        const float4* mp = reinterpret_cast<const float4*>(mult + k0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = __ldcg(mp + j);  // through L2: launched before the kernel ahead ends
            m[2 * j] = make_float2(t.x, t.y);
            m[2 * j + 1] = make_float2(t.z, t.w);
        }
    } else if constexpr (MODE == QuantMode::kWeightFold) {
        const bool first = r0 == 0;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const double s0 = static_cast<double>(s[k0 + 2 * p]);
            const double s1 = static_cast<double>(s[k0 + 2 * p + 1]);
            m[p] = make_float2(__double2float_rn(__dmul_rn(s0, c)), __double2float_rn(__dmul_rn(s1, c)));
            if (first) {
                act_mult_out[k0 + 2 * p] = __double2float_rn(__ddiv_rn(c, s0));
                act_mult_out[k0 + 2 * p + 1] = __double2float_rn(__ddiv_rn(c, s1));
            }
        }
    }
    quant_rows<MODE, AHEAD>(in, K, r0, r0, n, kb, kbp, m, codes, scales);
}

// The activations of a grouped linear: thread = (run of `rpg` tokens of one expert) x (one
// 32-block column).  Expert e's token t (row x_row[e] + t of x) becomes row a_row[e] + t of the
// padded codes, quantised with the expert's own multipliers (act_mult + e K, transform mode).
// The padding rows up to the next 128-row boundary are left as they are: they reach only rows
// of the GEMM's output tile that are never stored.
template <QuantMode MODE, bool AHEAD = false, class SRC = HostGroups>
__global__ void __launch_bounds__(kQuantThreads, 4) mx_quant_grouped_kernel(
    const uint16_t* __restrict__ x, int64_t K, const float* __restrict__ act_mult, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, const __grid_constant__ SRC src) {
    static_assert(MODE != QuantMode::kWeightFold, "activations only");
    griddep_launch_dependents();
    griddep_wait();  // x (and this workspace) may be written / still read by the preceding kernel
    // A device-built table is copied to shared memory first: each thread's expert lookup is a binary
    // search, which would otherwise be a chain of dependent global loads.
    constexpr bool kDevTable = std::is_same<SRC, DeviceGroups>::value;
    constexpr int kTableWords = (sizeof(GroupTable) + sizeof(RowRuns)) / 4;
    __shared__ __align__(16) int s_table[kDevTable ? kTableWords : 1];
    if constexpr (kDevTable) {
        const int* g = reinterpret_cast<const int*>(&group_table(src));
        const int* r = reinterpret_cast<const int*>(&row_runs(src));
        for (int i = threadIdx.x; i < kTableWords; i += blockDim.x)
            s_table[i] = i < static_cast<int>(sizeof(GroupTable) / 4) ? g[i] : r[i - sizeof(GroupTable) / 4];
        __syncthreads();
    }
    const GroupTable& gt = kDevTable ? *reinterpret_cast<const GroupTable*>(s_table) : group_table(src);
    const RowRuns& rr = kDevTable ? *reinterpret_cast<const RowRuns*>(s_table + sizeof(GroupTable) / 4)
                                  : row_runs(src);
    const int64_t kbp = padded_blocks(K);
    const int64_t item = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
    const int64_t kb = item % kbp;
    const int run = static_cast<int>(item / kbp);
    if (run >= rr.run_start[gt.groups]) return;
    const int e = group_of(rr.run_start, gt.groups, run);
    const int64_t t0 = static_cast<int64_t>(run - rr.run_start[e]) * rr.rpg;
    const int64_t n = t0 + rr.rpg < gt.rows[e] ? rr.rpg : gt.rows[e] - t0;
    const int64_t out0 = gt.a_row[e] + t0;
    if (kb >= K / 32) {
        for (int64_t r = out0; r < out0 + n; ++r) scales[scale_offset(r, kb, kbp)] = 0;
        return;
    }
    float2 m[16];
    if constexpr (MODE == QuantMode::kActTransform) {
        const float4* mp = reinterpret_cast<const float4*>(act_mult + static_cast<int64_t>(e) * K + kb * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 t = __ldcg(mp + j);  // through L2: launched before the kernel ahead ends
            m[2 * j] = make_float2(t.x, t.y);
            m[2 * j + 1] = make_float2(t.z, t.w);
        }
    }
    quant_rows<MODE, AHEAD>(x, K, gt.x_row[e] + t0, out0, n, kb, kbp, m, codes, scales);
}

// Activation quantisers are launched as programmatic dependents of whatever precedes them on the
// stream (in a model, the previous layer's GEMM), so the launch is processed while that kernel's
// last CTAs finish; each kernel's first act is griddepcontrol.wait, which returns once the
// preceding grid has completed and its writes are visible, before x is read or the workspace
// written.  After a copy or with nothing before it the attribute has no effect.  (Measured on
// back-to-back decode linears: 0.3-0.7 us less per call.)  A consequence for the GEMM launched
// after such a quantiser: it can start before the kernel ahead of the quantiser has finished, so
// the GEMM touches no memory a preceding kernel may write (weights included) before its own
// dependency wait, apart from the device-built expert table, whose quantiser is therefore launched
// in plain stream order (launch_act_quant_grouped_device).
template <class Kern, class... Args>
static int launch_dependent(Kern kernel, dim3 grid, dim3 block, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) return MACAQ_ECUDA;
    return launch_status();
}

// Rows per thread: enough threads to fill the GPU, rows walked by each otherwise.
// The threads one wave of the transform kernel holds: 4 CTAs of 128 per SM (128 registers).
static int64_t quant_thread_target() { return static_cast<int64_t>(sm_count()) * 16 * 32; }

static int64_t quant_rows_per_thread(int64_t R, int64_t K) {
    const int64_t cols = padded_blocks(K);
    const int64_t target = quant_thread_target();
    int64_t rpg = (R * cols + target - 1) / target;
    if (rpg < 1) rpg = 1;
    return rpg;
}

static unsigned quant_blocks(int64_t R, int64_t K, int64_t rpg) {
    const int64_t items = padded_blocks(K) * ((R + rpg - 1) / rpg);
    return static_cast<unsigned>((items + kQuantThreads - 1) / kQuantThreads);
}


// ---------------------------------------------------------------- half-block transform
//
// Two adjacent lanes per 32-element block: each loads, scales and transforms 16 elements,
// stages h = 1, 2, 4, 8 in its own registers.  The last stage (h = 16) pairs element i of the
// low half with element i of the high half, so the two lanes swap their 16 values once and
// the low lane keeps the sums, the high lane the differences -- the same fp32 operations in
// the same order as the whole-block butterfly, so the codes are bit-identical.  amax is the
// larger of the two halves' maxima; each lane converts and stores its 8 code bytes, the low
// lane the scale byte.
__device__ __forceinline__ void half_scale_fwht(float2 (&u)[8], const float2 (&m)[8], int hf, unsigned pair_mask) {
#pragma unroll
    for (int p = 0; p < 8; ++p) u[p] = __fmul2_rn(u[p], m[p]);
#pragma unroll
    for (int p = 0; p < 8; ++p) {  // h = 1: the two halves of a pair
        const float a = u[p].x, b = u[p].y;
        u[p] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < 8; hp <<= 1) {  // h = 2, 4, 8: whole pairs, packed
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            if ((p & hp) == 0) {
                const float2 a = u[p], b = u[p + hp];
                u[p] = __fadd2_rn(a, b);
                u[p + hp] = fsub2_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) {  // h = 16 across the lane pair: a = low lane's value, b = high's
        float2 o;
        o.x = __shfl_xor_sync(pair_mask, u[p].x, 1);
        o.y = __shfl_xor_sync(pair_mask, u[p].y, 1);
        u[p] = hf == 0 ? __fadd2_rn(u[p], o) : fsub2_rn(o, u[p]);
    }
}

__device__ __forceinline__ void half_block(const uint4 (&raw)[2], const float2 (&m)[8], int hf, unsigned pair_mask,
                                           uint8_t* codes8, uint8_t* scale_byte) {
    float2 u[8];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int t = 0; t < 4; ++t)  // bf16 -> fp32 is exact: the bits move up 16 places
            u[4 * j + t] = make_float2(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xFFFF0000u));
    }
    half_scale_fwht(u, m, hf, pair_mask);
    const float* f = reinterpret_cast<const float*>(u);
    float amax = fmax3(fabsf(f[0]), fabsf(f[1]), fabsf(f[2]));
#pragma unroll
    for (int i = 3; i + 1 < 16; i += 2) amax = fmax3(amax, fabsf(f[i]), fabsf(f[i + 1]));
    amax = fmaxf(amax, fabsf(f[15]));
    amax = fmaxf(amax, __shfl_xor_sync(pair_mask, amax, 1));
    const uint32_t E = (__float_as_uint(amax) >> 23) & 0xFFu;
    const uint32_t e = E >= 3u ? E - 2u : 0u;
    const float inv = __uint_as_float((254u - e) << 23);  // 2^(127 - e), a normal float
    const float2 inv2 = make_float2(inv, inv);
    const uint32_t c0 = cvt_e2m1x8(__fmul2_rn(u[0], inv2), __fmul2_rn(u[1], inv2), __fmul2_rn(u[2], inv2),
                                   __fmul2_rn(u[3], inv2));
    const uint32_t c1 = cvt_e2m1x8(__fmul2_rn(u[4], inv2), __fmul2_rn(u[5], inv2), __fmul2_rn(u[6], inv2),
                                   __fmul2_rn(u[7], inv2));
    *reinterpret_cast<uint2*>(codes8) = make_uint2(c0, c1);
    if (hf == 0) *scale_byte = static_cast<uint8_t>(e);
}

constexpr int kHalfThreads = 128;
constexpr int kHalfMinBlocks = 6;                        // 80 registers: six CTAs per SM
constexpr int64_t kHalfKernelMaxElems = int64_t(1) << 22;  // above this the whole-block kernel wins
constexpr int64_t kAheadMinElems = int64_t(1) << 24;       // from here the transform loads one row ahead

// Thread = (run of `rpg` rows) x (block column kb) x (half hf), halves fastest, then columns;
// the low half of a padded block column (kb >= K/32) writes the zero scale bytes of its rows.
// blockIdx.y = g: the g-th of several linears on the same x, quantised with its own multipliers
// (mult + g K) into rows g * seg_rows onwards of the codes and scales (one linear: g = 0).  With
// seg_rows a multiple of 128 that segment's scale atoms are those of rows 0.. shifted by
// seg_rows * padded_blocks(K) bytes, so both offsets are applied to the base pointers once.
__global__ void __launch_bounds__(kHalfThreads, kHalfMinBlocks) mx_quant_half_kernel(
    const uint16_t* __restrict__ x, int64_t R, int64_t K, int64_t rpg, const float* __restrict__ mult,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int64_t seg_rows) {
    griddep_launch_dependents();
    griddep_wait();  // x (and this workspace) may be written / still read by the preceding kernel
    const int64_t kb_real = K / 32;
    const int64_t kbp = padded_blocks(K);
    const int64_t item = static_cast<int64_t>(blockIdx.x) * kHalfThreads + threadIdx.x;
    const int hf = static_cast<int>(item & 1);
    const int64_t kb = (item >> 1) % kbp;
    const int64_t r0 = ((item >> 1) / kbp) * rpg;
    if (r0 >= R) return;  // both lanes of a pair leave together: same block column, same rows
    const int64_t n = r0 + rpg < R ? rpg : R - r0;
    const int64_t o0 = static_cast<int64_t>(blockIdx.y) * seg_rows;  // this linear's first output row
    codes += o0 * (K / 2);
    scales += o0 * kbp;
    if (kb >= kb_real) {
        if (hf == 0)
            for (int64_t r = r0; r < r0 + n; ++r) scales[scale_offset(r, kb, kbp)] = 0;
        return;
    }
    const unsigned pair_mask = 3u << (threadIdx.x & 30u);
    const int64_t k0 = kb * 32 + hf * 16;
    float2 m[8];
    const float4* mp = reinterpret_cast<const float4*>(mult + static_cast<int64_t>(blockIdx.y) * K + k0);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 t = __ldcg(mp + j);  // through L2: launched before the kernel ahead ends
        m[2 * j] = make_float2(t.x, t.y);
        m[2 * j + 1] = make_float2(t.z, t.w);
    }
    auto load = [&](int64_t r, uint4 (&b)[2]) {
        const uint4* p = reinterpret_cast<const uint4*>(x + r * K + k0);
        b[0] = __ldcs(p);
        b[1] = __ldcs(p + 1);
    };
    auto out = [&](int64_t r) { return codes + r * (K / 2) + kb * 16 + hf * 8; };
    auto sc = [&](int64_t r) { return scales + scale_offset(r, kb, kbp); };
    int64_t i = 0;
    for (; i + 1 < n; i += 2) {  // two rows at a time, both loaded before either is used
        uint4 b0[2], b1[2];
        load(r0 + i, b0);
        load(r0 + i + 1, b1);
        half_block(b0, m, hf, pair_mask, out(r0 + i), sc(r0 + i));
        half_block(b1, m, hf, pair_mask, out(r0 + i + 1), sc(r0 + i + 1));
    }
    if (i < n) {
        uint4 b0[2];
        load(r0 + i, b0);
        half_block(b0, m, hf, pair_mask, out(r0 + i), sc(r0 + i));
    }
}

// Rows per thread of the half-block kernel: enough threads for one resident wave (six CTAs of
// 128 per SM), rows walked by each otherwise.
static int64_t half_rows_per_thread(int64_t R, int64_t K) {
    const int64_t items = 2 * padded_blocks(K);
    const int64_t target = static_cast<int64_t>(sm_count()) * kHalfMinBlocks * kHalfThreads;
    const int64_t rpg = (R * items + target - 1) / target;
    return rpg < 1 ? 1 : rpg;
}

// Launch helpers used by the C entry points and by the linear.
int launch_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                               uint8_t* Aq, uint8_t* As, cudaStream_t stream) {
    if (M * K <= kHalfKernelMaxElems) {
        const int64_t rpg = half_rows_per_thread(M, K);
        const int64_t items = 2 * padded_blocks(K) * ((M + rpg - 1) / rpg);
        const dim3 grid(static_cast<unsigned>((items + kHalfThreads - 1) / kHalfThreads));
        return launch_dependent(mx_quant_half_kernel, grid, dim3(kHalfThreads), stream, x, M, K, rpg, act_mult, Aq, As,
                                int64_t(0));
    }
    const int64_t rpg = quant_rows_per_thread(M, K);
    const auto kernel = M * K >= kAheadMinElems ? mx_quant_kernel<QuantMode::kActTransform, true>
                                                : mx_quant_kernel<QuantMode::kActTransform, false>;
    return launch_dependent(kernel, dim3(quant_blocks(M, K, rpg)), dim3(kQuantThreads), stream, x, M, K, rpg, act_mult,
                            static_cast<const float*>(nullptr), 0.0, static_cast<float*>(nullptr), Aq, As);
}

int launch_act_quant_grouped(const uint16_t* x, int64_t K, const float* act_mult, uint8_t* Aq, uint8_t* As,
                             const GroupTable& gt, cudaStream_t stream) {
    int64_t tokens = 0;
    for (int e = 0; e < gt.groups; ++e) tokens += gt.rows[e];
    if (tokens == 0) return MACAQ_OK;
    // The shortest runs that keep the grid within one resident wave: a second wave would share
    // the SMs with the GEMM's CTAs, which the programmatic launch makes resident as soon as
    // first-wave CTAs leave.  The run count falls as runs lengthen, and runs as long as the
    // largest expert give each expert one run, the fewest possible.
    const int64_t kbp = padded_blocks(K);
    int max_rows = 0;
    for (int e = 0; e < gt.groups; ++e) max_rows = gt.rows[e] > max_rows ? gt.rows[e] : max_rows;
    auto runs = [&](int rpg) {
        int64_t n = 0;
        for (int e = 0; e < gt.groups; ++e) n += (gt.rows[e] + rpg - 1) / rpg;
        return n;
    };
    int lo = static_cast<int>(quant_rows_per_thread(tokens, K)), hi = max_rows;
    if (lo > hi) lo = hi;
    while (lo < hi) {  // first rpg in [lo, hi] whose grid fits; hi if none does
        const int mid = lo + (hi - lo) / 2;
        if (kbp * runs(mid) <= quant_thread_target()) hi = mid;
        else lo = mid + 1;
    }
    HostGroups hg;
    hg.gt = gt;
    hg.rr.rpg = lo;
    hg.rr.run_start[0] = 0;
    for (int e = 0; e < gt.groups; ++e) hg.rr.run_start[e + 1] = hg.rr.run_start[e] + (gt.rows[e] + lo - 1) / lo;
    const int64_t items = kbp * hg.rr.run_start[gt.groups];
    const unsigned blocks = static_cast<unsigned>((items + kQuantThreads - 1) / kQuantThreads);
    if (act_mult) {
        const auto kernel = tokens * K >= kAheadMinElems ? mx_quant_grouped_kernel<QuantMode::kActTransform, true>
                                                         : mx_quant_grouped_kernel<QuantMode::kActTransform, false>;
        return launch_dependent(kernel, dim3(blocks), dim3(kQuantThreads), stream, x, K, act_mult, Aq, As, hg);
    }
    return launch_dependent(mx_quant_grouped_kernel<QuantMode::kPlain>, dim3(blocks), dim3(kQuantThreads), stream, x,
                            K, static_cast<const float*>(nullptr), Aq, As, hg);
}

// G linears on the same x (act_mult [G][K]): linear g's codes and scales are rows g * seg_rows to
// g * seg_rows + M - 1 (seg_rows a multiple of 128, so each linear's scale atoms start a 128-row
// block).  Small inputs: one half-block launch with a grid row per linear, its runs sized so all G
// fit one resident wave; larger ones: the grouped quantiser with every group reading rows 0..M-1.
int launch_act_transform_quant_multi(const uint16_t* x, int64_t M, int64_t K, int G, const float* act_mult,
                                     int64_t seg_rows, uint8_t* Aq, uint8_t* As, cudaStream_t stream) {
    if (M * K <= kHalfKernelMaxElems) {
        const int64_t rpg = half_rows_per_thread(G * M, K);
        const int64_t items = 2 * padded_blocks(K) * ((M + rpg - 1) / rpg);
        const dim3 grid(static_cast<unsigned>((items + kHalfThreads - 1) / kHalfThreads), static_cast<unsigned>(G));
        return launch_dependent(mx_quant_half_kernel, grid, dim3(kHalfThreads), stream, x, M, K, rpg, act_mult, Aq, As,
                                seg_rows);
    }
    GroupTable gt{};
    gt.groups = G;
    for (int g = 0; g < G; ++g) {
        gt.rows[g] = static_cast<int>(M);
        gt.x_row[g] = 0;
        gt.a_row[g] = static_cast<int>(g * seg_rows);
    }
    gt.a_row[G] = static_cast<int>(G * seg_rows);
    return launch_act_quant_grouped(x, K, act_mult, Aq, As, gt, stream);
}

// Rows per run of the grouped quantiser when only the total T of routed rows and the expert count
// are known on the host (device counts): the grid covers the most runs any split of T rows over E
// experts can need, T / rpg + E, and threads past the real runs return at once.  The runs are made
// long enough for that bound to fit one resident wave (as the host-count launch does for its actual
// runs): a second wave would run nearly as long as the first.
int64_t device_groups_rpg(int64_t T, int E, int64_t K) {
    int64_t rpg = quant_rows_per_thread(T, K);
    const int64_t wave_runs = quant_thread_target() / padded_blocks(K) - E;
    if (wave_runs >= 1) {
        const int64_t need = (T + wave_runs - 1) / wave_runs;
        if (need > rpg) rpg = need;
    }
    return rpg;
}
int64_t device_groups_max_runs(int64_t T, int E, int64_t rpg) { return T / rpg + E; }

// Launched in plain stream order, not as a programmatic dependent: the grouped GEMM that follows
// reads the expert table (written by the table kernel just before this one) in all its warps before
// its own dependency wait, which is safe only if this kernel -- and so the GEMM, launched after it
// started -- began after the table kernel had completed.
int launch_act_quant_grouped_device(const uint16_t* x, int64_t T, int E, int64_t K, const float* act_mult, uint8_t* Aq,
                                    uint8_t* As, const DeviceGroups& dg, cudaStream_t stream) {
    const int64_t rpg = device_groups_rpg(T, E, K);
    const int64_t items = padded_blocks(K) * device_groups_max_runs(T, E, rpg);
    const unsigned blocks = static_cast<unsigned>((items + kQuantThreads - 1) / kQuantThreads);
    if (act_mult) {
        const auto kernel = T * K >= kAheadMinElems
                                ? mx_quant_grouped_kernel<QuantMode::kActTransform, true, DeviceGroups>
                                : mx_quant_grouped_kernel<QuantMode::kActTransform, false, DeviceGroups>;
        kernel<<<blocks, kQuantThreads, 0, stream>>>(x, K, act_mult, Aq, As, dg);
    } else {
        mx_quant_grouped_kernel<QuantMode::kPlain, false, DeviceGroups><<<blocks, kQuantThreads, 0, stream>>>(
            x, K, nullptr, Aq, As, dg);
    }
    return launch_status();
}

int launch_act_quant_plain(const uint16_t* x, int64_t M, int64_t K, uint8_t* Aq, uint8_t* As,
                           cudaStream_t stream) {
    const int64_t rpg = quant_rows_per_thread(M, K);
    return launch_dependent(mx_quant_kernel<QuantMode::kPlain>, dim3(quant_blocks(M, K, rpg)), dim3(kQuantThreads),
                            stream, static_cast<const void*>(x), M, K, rpg, static_cast<const float*>(nullptr),
                            static_cast<const float*>(nullptr), 0.0, static_cast<float*>(nullptr), Aq, As);
}

}  // namespace macaq

using namespace macaq;

extern "C" int macaq_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                                         uint8_t* Aq, uint8_t* As, void* stream) {
    if (!x || !act_mult || !Aq || !As) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (!aligned16(x) || !aligned16(act_mult) || !aligned16(Aq) || !aligned16(As)) return MACAQ_EALIGN;
    return launch_act_transform_quant(x, M, K, act_mult, Aq, As, static_cast<cudaStream_t>(stream));
}

extern "C" int macaq_act_quant_plain(const uint16_t* x, int64_t M, int64_t K, uint8_t* Aq, uint8_t* As,
                                     void* stream) {
    if (!x || !Aq || !As) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (!aligned16(x) || !aligned16(Aq) || !aligned16(As)) return MACAQ_EALIGN;
    return launch_act_quant_plain(x, M, K, Aq, As, static_cast<cudaStream_t>(stream));
}

extern "C" int macaq_fold_weights(const float* W, int64_t N, int64_t K, const float* s, uint8_t* Wq,
                                  uint8_t* Ws, float* act_mult, void* stream) {
    if (!W || !s || !Wq || !Ws || !act_mult) return MACAQ_EINVAL;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(W) || !aligned16(s) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(act_mult))
        return MACAQ_EALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Offline call: bring s to the host once and reject non-finite or non-positive scales
    // before anything is written.
    std::vector<float> hs(static_cast<size_t>(K));
    if (cudaMemcpyAsync(hs.data(), s, sizeof(float) * K, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MACAQ_ECUDA;
    for (float v : hs)
        if (!(v > 0.0f) || !std::isfinite(v)) return MACAQ_EINVAL;
    const double c = 1.0 / std::sqrt(32.0);  // correctly rounded (IEEE sqrt and divide)
    const int64_t rpg = quant_rows_per_thread(N, K);
    mx_quant_kernel<QuantMode::kWeightFold><<<quant_blocks(N, K, rpg), kQuantThreads, 0, st>>>(
        W, N, K, rpg, nullptr, s, c, act_mult, Wq, Ws);
    return launch_status();
}
