// noalloc.cu -- macaq_w4a4_linear_noalloc: the W4A4 linear layer for callers that cannot
// allocate device memory.
//
// macaq_w4a4_linear needs scratch for the quantised activations (MXFP4 codes and E8M0
// scales) and takes it from the caller.  Some callers cannot provide it.  cudaMalloc
// synchronises the device and can fail or fragment memory at run time, so a
// latency-critical serving loop that plans all of its memory up front must not call it;
// a plugin whose host application owns every device allocation has no allocator to call;
// and a plain C caller that is only handed device pointers for its inputs and outputs
// has no way to obtain a buffer.  For them this variant keeps the scratch in a fixed-size
// array in the library's own device memory.
//
// Costs and rules of that array:
//   * it is kNoAllocScratchBytes (32 MiB) on every GPU that loads the library, held until
//     the process exits;
//   * problems whose activation codes and scales exceed it are rejected with
//     MACAQ_ETOOLARGE before anything is launched; what is left of the array after them
//     serves as the GEMM's stream-K scratch when it is large enough, otherwise the GEMM
//     runs its data-parallel schedule (same results up to fp32 summation order);
//   * every call shares it and it keeps the previous call's contents.  Nothing in it has
//     to start at zero: each call writes every code byte and every scale byte of its real
//     rows before reading them, a stream-K flag counts only when it holds the tag of the
//     current launch (and each launch clears the flags it consumed), and the bytes it does
//     not write (padded rows of the last 128-row scale atom, stale partial sums) are never
//     used for a stored output;
//   * the stream-K flag words sit after each call's own activation bytes, so their offset
//     changes with the shape, and a later call of another shape may find an earlier call's
//     flag words among its activation codes or its own flags at bytes an earlier call used
//     for codes.  None of that needs clearing: the library never reuses a launch tag (a
//     per-process random start, one step per launch), except when a CUDA graph replays a
//     captured launch of the same call, whose flags sit at the same place and were cleared
//     by the launch that consumed them;
//   * two calls whose kernels overlap on the GPU (different streams without ordering, or
//     several host threads) race on the array and corrupt each other's results: order
//     them on one stream or serialise them;
//   * its device address is looked up once per device with cudaGetSymbolAddress on the
//     first call made with that device current; make that first call before any CUDA
//     stream capture begins.
#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace macaq {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// The scratch itself: static device memory, never allocated or freed at run time.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];


// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in: a kernel given it would fault or, where the GPU can
// reach host memory, silently use the wrong memory.  So the real address is looked up
// once per device, with that device current, and cached.
static int noalloc_scratch(uint8_t** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static uint8_t* addr[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ECUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MACAQ_ECUDA;
        addr[dev] = static_cast<uint8_t*>(p);
    }
    *out = addr[dev];
    return MACAQ_OK;
}

}  // namespace macaq

using namespace macaq;

extern "C" int macaq_w4a4_linear_noalloc(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                                         const uint8_t* Wq, const uint8_t* Ws, int64_t N, uint16_t* y,
                                         void* stream) {
    if (!x || !act_mult || !Wq || !Ws || !y) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(x) || !aligned16(act_mult) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y))
        return MACAQ_EALIGN;
    const size_t act_bytes = linear_activation_bytes(M, K);
    if (act_bytes > kNoAllocScratchBytes) return MACAQ_ETOOLARGE;
    uint8_t* scratch = nullptr;
    if (int st = noalloc_scratch(&scratch)) return st;
    const LinearWorkspace l = linear_workspace_layout(scratch, M, K);
    const bool streamk = act_bytes + l.gemm_bytes <= kNoAllocScratchBytes;
    return run_linear(x, M, K, act_mult, Wq, Ws, N, y, l, streamk, static_cast<cudaStream_t>(stream));
}
