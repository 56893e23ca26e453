// calib.cu -- calibration of the per-channel scale s, the step before the weight fold.
//
// "MACaQ: Fast, Model Agnostic Calibrated Quantization ..." (Abstract) calibrates a per-channel
// scale for each layer but gives no rule; the reading used throughout is the SmoothQuant
// alpha = 1/2 balance
//     s_j = fl32( sqrt( max_r |xcal_rj| / max_n |W_nj| ) ),  quotient and root in IEEE double,
// with s_j = 1 where either maximum is zero.  After it, max|x_j / s_j| and max|W_nj * s_j|
// agree, which is what lets one MXFP4 scale per block serve both outliers and weights.
//
// Two kernels on the caller's stream after zeroing s: the column maxima of |W| (HBM-bound over
// the fp32 weights: 4 bytes per parameter read once) land in s as fp32 bit patterns through
// atomicMax -- exact, since non-negative floats order like their unsigned bit patterns -- and
// the finishing kernel takes each column's activation maximum over the small calibration batch
// and replaces the weight maximum by s_j.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"

namespace macaq {

constexpr int kCalibRows = 256;     // weight rows per CTA
constexpr int kCalibThreads = 256;  // 8 warps; lane = column of a 32-column slab

__global__ void __launch_bounds__(kCalibThreads) column_amax_kernel(const float* __restrict__ W, int64_t N,
                                                                    int64_t K, uint32_t* __restrict__ amax_bits) {
    __shared__ float part[kCalibThreads / 32][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + lane;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kCalibRows;
    const int64_t r1 = r0 + kCalibRows < N ? r0 + kCalibRows : N;
    float m = 0.0f;
    if (j < K) {
        int64_t r = r0 + warp;
        for (; r + 24 < r1; r += 32) {  // four rows per warp in flight; a warp reads 128 B per row
            const float a = __ldcs(W + r * K + j), b = __ldcs(W + (r + 8) * K + j);
            const float c = __ldcs(W + (r + 16) * K + j), d = __ldcs(W + (r + 24) * K + j);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d))));
        }
        for (; r < r1; r += 8) m = fmaxf(m, fabsf(__ldcs(W + r * K + j)));
    }
    part[warp][lane] = m;
    __syncthreads();
    if (warp == 0 && j < K) {
#pragma unroll
        for (int w = 1; w < kCalibThreads / 32; ++w) m = fmaxf(m, part[w][lane]);
        atomicMax(amax_bits + j, __float_as_uint(m));
    }
}

__global__ void __launch_bounds__(kCalibThreads) calib_finish_kernel(const uint16_t* __restrict__ xcal, int64_t C,
                                                                     int64_t K, float* s) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * kCalibThreads + threadIdx.x;
    if (j >= K) return;
    float ax = 0.0f;
    for (int64_t r = 0; r < C; ++r)  // bf16 -> fp32 is exact: the bits move up 16 places
        ax = fmaxf(ax, fabsf(__uint_as_float(static_cast<uint32_t>(xcal[r * K + j]) << 16)));
    const float aw = s[j];  // the weight column's maximum, left here by column_amax_kernel
    s[j] = (ax == 0.0f || aw == 0.0f)
               ? 1.0f
               : __double2float_rn(__dsqrt_rn(__ddiv_rn(static_cast<double>(ax), static_cast<double>(aw))));
}

}  // namespace macaq

extern "C" int macaq_calibrate_scale(const uint16_t* xcal, int64_t C, const float* W, int64_t N, int64_t K,
                                     float* s, void* stream) {
    using namespace macaq;
    if (!xcal || !W || !s) return MACAQ_EINVAL;
    if (int st = check_shape(C, K)) return st;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(xcal) || !aligned16(W) || !aligned16(s)) return MACAQ_EALIGN;
    if ((N + kCalibRows - 1) / kCalibRows > 65535) return MACAQ_ESHAPE;  // grid.y limit
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(s, 0, static_cast<size_t>(K) * sizeof(float), st) != cudaSuccess) return MACAQ_ECUDA;
    const dim3 grid(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>((N + kCalibRows - 1) / kCalibRows));
    column_amax_kernel<<<grid, kCalibThreads, 0, st>>>(W, N, K, reinterpret_cast<uint32_t*>(s));
    calib_finish_kernel<<<static_cast<unsigned>((K + kCalibThreads - 1) / kCalibThreads), kCalibThreads, 0, st>>>(
        xcal, C, K, s);
    return launch_status();
}
