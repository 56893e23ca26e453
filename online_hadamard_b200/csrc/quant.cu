// quant.cu -- MXFP4 quantisation kernels along K, with the online MACaQ transform.
//
//   act_transform: u = fl32(x * act_mult), block-Hadamard b = 32 (FWHT in registers and
//                  warp shuffles), E8M0 scale, E2M1 RTN codes       (activations, online)
//   weight_fold:   u = fl32(W * fl32(s * c)), same transform and quantisation (weights,
//                  offline; also writes act_mult = fl32(c / s))
//   plain:         MXFP4 of x with no scale and no transform       (baseline)
//
// "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
// Activations", Abstract: per-channel scale + block-Hadamard online on the activations,
// inverse transforms absorbed into the weights, MXFP4 W4A4, round-to-nearest weights.
//
// Work split: one warp task = one row x 256 consecutive elements (8 blocks of 32).  Lane
// quad q (lanes 4q..4q+3) owns block 8*task+q; each lane owns 8 consecutive elements,
// loaded as one 16-byte vector (bf16) or two (fp32).  Butterfly stages h = 1, 2, 4 stay
// in a lane's registers; h = 8, 16 cross lanes with __shfl_xor (masks 1, 2).  Every fp32
// operation is an explicit round-to-nearest intrinsic, so the compiler cannot contract
// the scale into the first butterfly, and the result is bit-identical to the canonical
// sequential order.  The kernel is HBM-bound: 2 (or 4) bytes in, 0.53 bytes out per
// element.
#include <cstdint>
#include <cmath>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

enum class QuantMode { kActTransform = 0, kWeightFold = 1, kPlain = 2 };

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;

// Eight E2M1 codes (magnitudes only) of |q0..q7| packed two per byte, element 2j in the
// low nibble: cvt.rn.satfinite.e2m1x2 puts its first source in the high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&q)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

template <QuantMode MODE>
struct QuantLoad {
    float x[8];
    float m[8];
};

template <QuantMode MODE>
__device__ __forceinline__ void load_item(const void* __restrict__ in, const float* __restrict__ mult,
                                          const float* __restrict__ s, double c, int64_t row_off,
                                          int64_t k0, QuantLoad<MODE>& it) {
    if constexpr (MODE == QuantMode::kWeightFold) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(in) + row_off + k0);
        const float4 a = __ldcs(p);
        const float4 b = __ldcs(p + 1);
        it.x[0] = a.x; it.x[1] = a.y; it.x[2] = a.z; it.x[3] = a.w;
        it.x[4] = b.x; it.x[5] = b.y; it.x[6] = b.z; it.x[7] = b.w;
        const float4* sp = reinterpret_cast<const float4*>(s + k0);
        const float4 s0 = __ldg(sp);
        const float4 s1 = __ldg(sp + 1);
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) it.m[j] = __double2float_rn(__dmul_rn(static_cast<double>(sv[j]), c));
    } else {
        const uint4 v = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in) + row_off + k0));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            it.x[2 * j] = __uint_as_float(w[j] << 16);            // bf16 -> fp32 is exact
            it.x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
        if constexpr (MODE == QuantMode::kActTransform) {
            const float4* mp = reinterpret_cast<const float4*>(mult + k0);
            const float4 m0 = __ldg(mp);
            const float4 m1 = __ldg(mp + 1);
            it.m[0] = m0.x; it.m[1] = m0.y; it.m[2] = m0.z; it.m[3] = m0.w;
            it.m[4] = m1.x; it.m[5] = m1.y; it.m[6] = m1.z; it.m[7] = m1.w;
        }
    }
}

// Scale + FWHT-32 of the block held by a lane quad; `sub` = lane % 4 = element bits 3-4.
template <QuantMode MODE>
__device__ __forceinline__ void transform(QuantLoad<MODE>& it, int sub) {
    if constexpr (MODE == QuantMode::kPlain) return;
    float (&u)[8] = it.x;
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = __fmul_rn(u[j], it.m[j]);
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((j & h) == 0) {
                const float a = u[j], b = u[j + h];
                u[j] = __fadd_rn(a, b);
                u[j + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int s = 1; s <= 2; s <<= 1) {  // h = 8 (lane bit 0), h = 16 (lane bit 1)
        const bool upper = (sub & s) != 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float p = __shfl_xor_sync(0xFFFFFFFFu, u[j], s);
            // lower partner holds u_i and keeps u_i + u_{i+h}; upper holds u_{i+h}, keeps u_i - u_{i+h}
            u[j] = upper ? __fsub_rn(p, u[j]) : __fadd_rn(u[j], p);
        }
    }
}

// E8M0 scale and packed codes of the block; returns the scale byte, writes 4 code bytes.
__device__ __forceinline__ uint32_t quantize_block(const float (&v)[8], uint32_t& packed) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    const uint32_t E = (__float_as_uint(amax) >> 23) & 0xFFu;
    const uint32_t e = E >= 3u ? E - 2u : 0u;
    const float inv_scale = __uint_as_float((254u - e) << 23);  // 2^(127 - e), a normal float
    float q[8];
    uint32_t signs = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        q[j] = __fmul_rn(fabsf(v[j]), inv_scale);  // exact unless far below the E2M1 grid
        signs |= (__float_as_uint(v[j]) >> 31) << (4 * j + 3);
    }
    packed = cvt_e2m1x8(q) | signs;
    return e;
}

template <QuantMode MODE>
__global__ void __launch_bounds__(kQuantThreads) mx_quant_kernel(
    const void* __restrict__ in, int64_t R, int64_t K, const float* __restrict__ mult,
    const float* __restrict__ s, double c, float* __restrict__ act_mult_out,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int quad = lane >> 2;
    const int sub = lane & 3;
    const int64_t kb_real = K / 32;
    const int64_t kbp = padded_blocks(K);
    const int64_t groups = kbp / 8;  // warp tasks per row
    const int64_t tasks = R * groups;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
    const int64_t w0 = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + (threadIdx.x >> 5);

    for (int64_t base = w0; base < tasks; base += warps * kQuantUnroll) {
        QuantLoad<MODE> it[kQuantUnroll];
        bool real[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const int64_t t = base + u * warps;
            const int64_t r = t / groups;
            const int64_t kb = (t - r * groups) * 8 + quad;
            real[u] = t < tasks && kb < kb_real;
            if (real[u]) load_item<MODE>(in, mult, s, c, r * K, kb * 32 + sub * 8, it[u]);
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const int64_t t = base + u * warps;
            if (t >= tasks) break;  // warp-uniform
            const int64_t r = t / groups;
            const int64_t kb = (t - r * groups) * 8 + quad;
            if (!real[u]) {
#pragma unroll
                for (int j = 0; j < 8; ++j) it[u].x[j] = 0.0f;
            }
            transform<MODE>(it[u], sub);
            uint32_t packed;
            const uint32_t e = quantize_block(it[u].x, packed);
            if (real[u]) {
                *reinterpret_cast<uint32_t*>(codes + r * (K / 2) + kb * 16 + sub * 4) = packed;
                if (sub == 0) scales[scale_offset(r, kb, kbp)] = static_cast<uint8_t>(e);
                if constexpr (MODE == QuantMode::kWeightFold) {
                    if (r == 0) {
                        const int64_t k0 = kb * 32 + sub * 8;
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            act_mult_out[k0 + j] =
                                __double2float_rn(__ddiv_rn(c, static_cast<double>(s[k0 + j])));
                    }
                }
            } else if (sub == 0) {
                scales[scale_offset(r, kb, kbp)] = 0;  // padded block of a real row
            }
        }
    }
}

int quant_grid(int64_t R, int64_t K) {
    const int64_t tasks = R * (padded_blocks(K) / 8);
    const int64_t per_block = (kQuantThreads / 32) * kQuantUnroll;
    int64_t blocks = (tasks + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// Launch helpers used by the C entry points and by the fused linear.
int launch_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                               uint8_t* Aq, uint8_t* As, cudaStream_t stream) {
    mx_quant_kernel<QuantMode::kActTransform><<<quant_grid(M, K), kQuantThreads, 0, stream>>>(
        x, M, K, act_mult, nullptr, 0.0, nullptr, Aq, As);
    return launch_status();
}

int launch_act_quant_plain(const uint16_t* x, int64_t M, int64_t K, uint8_t* Aq, uint8_t* As,
                           cudaStream_t stream) {
    mx_quant_kernel<QuantMode::kPlain><<<quant_grid(M, K), kQuantThreads, 0, stream>>>(
        x, M, K, nullptr, nullptr, 0.0, nullptr, Aq, As);
    return launch_status();
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
    mx_quant_kernel<QuantMode::kWeightFold><<<quant_grid(N, K), kQuantThreads, 0, st>>>(
        W, N, K, nullptr, s, c, act_mult, Wq, Ws);
    return launch_status();
}
