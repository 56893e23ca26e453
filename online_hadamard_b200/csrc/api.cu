// api.cu -- status strings, buffer-size helpers and the device status flag of libmacaq.
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

}  // namespace macaq

using namespace macaq;

extern "C" const char* macaq_status_str(int status) {
    switch (status) {
        case MACAQ_OK: return "MACAQ_OK";
        case MACAQ_EINVAL: return "MACAQ_EINVAL: null pointer or invalid value";
        case MACAQ_ESHAPE: return "MACAQ_ESHAPE: M, N, K out of range or K not a multiple of 32";
        case MACAQ_EALIGN: return "MACAQ_EALIGN: pointer not 16-byte aligned";
        case MACAQ_ECUDA: return "MACAQ_ECUDA: CUDA runtime or launch failure";
        case MACAQ_ETIMEOUT: return "MACAQ_ETIMEOUT: a bounded device-side wait gave up";
        case MACAQ_EWORKSPACE: return "MACAQ_EWORKSPACE: workspace too small";
        case MACAQ_ETOOLARGE:
            return "MACAQ_ETOOLARGE: problem needs more scratch than the no-allocation entry point holds";
        case MACAQ_ECOUNTS:
            return "MACAQ_ECOUNTS: device routing counts were negative or ran past the rows of x (corrected)";
        default: return "MACAQ: unknown status";
    }
}

extern "C" size_t macaq_scale_bytes(int64_t rows, int64_t K) {
    if (check_shape(rows, K) != MACAQ_OK) return 0;
    return static_cast<size_t>(scale_bytes(rows, K));
}

extern "C" int64_t macaq_scale_offset(int64_t r, int64_t kb, int64_t K) {
    if (r < 0 || r > kMaxDim || K < kBlock || K > kMaxDim || K % kBlock != 0) return -1;
    if (kb < 0 || kb >= padded_blocks(K)) return -1;
    return scale_offset(r, kb, padded_blocks(K));
}

namespace macaq {

// One thread per scale byte of the tiled buffer (rows padded to 128, blocks to KBp): row-major
// [rows][K/32] E8M0 bytes to the MMA tile layout (padded blocks and padded rows written as 0),
// or back (real rows and blocks only).
__global__ void scales_layout_kernel(const uint8_t* __restrict__ src, int64_t rows, int64_t K, uint8_t* __restrict__ dst,
                                     int to_tiled) {
    const int64_t kb_real = K / 32, kbp = padded_blocks(K);
    const int64_t prow = (rows + 127) / 128 * 128;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= prow * kbp) return;
    const int64_t r = i / kbp, kb = i % kbp;
    const int64_t off = scale_offset(r, kb, kbp);
    const bool real = r < rows && kb < kb_real;
    if (to_tiled)
        dst[off] = real ? src[r * kb_real + kb] : 0;
    else if (real)
        dst[r * kb_real + kb] = src[off];
}

static int launch_scales_layout(const uint8_t* src, int64_t rows, int64_t K, uint8_t* dst, int to_tiled, void* stream) {
    if (!src || !dst) return MACAQ_EINVAL;
    if (int st = check_shape(rows, K)) return st;
    const int64_t n = (rows + 127) / 128 * 128 * padded_blocks(K);
    scales_layout_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        src, rows, K, dst, to_tiled);
    return launch_status();
}

}  // namespace macaq

extern "C" int macaq_scales_to_tiled(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* tiled, void* stream) {
    return launch_scales_layout(rowmajor, rows, K, tiled, 1, stream);
}

extern "C" int macaq_scales_to_rowmajor(const uint8_t* tiled, int64_t rows, int64_t K, uint8_t* rowmajor,
                                        void* stream) {
    return launch_scales_layout(tiled, rows, K, rowmajor, 0, stream);
}

extern "C" int macaq_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MACAQ_ECUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MACAQ_ECUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MACAQ_ECUDA;
    }
    return v;  // MACAQ_OK, or the code of the last event recorded (MACAQ_ETIMEOUT, MACAQ_ECOUNTS)
}
