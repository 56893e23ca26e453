// common.cuh -- shapes, the E8M0 scale tile layout and host-side validation shared by the
// library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <mutex>

#include "macaq.h"

namespace macaq {

constexpr int64_t kBlock = 32;          // MX block = Hadamard block (elements along K)
constexpr int64_t kMaxDim = 0x7FFFFFFF;  // M, N, K < 2^31

// Scale blocks per row, padded so every 256-element K tile owns two full 512-byte atoms.
__host__ __device__ __forceinline__ int64_t padded_blocks(int64_t K) {
    return ((K + 255) / 256) * 8;
}

// Byte offset of the E8M0 scale of (row r, 32-block kb) in the MMA tile layout: 512-byte
// atoms of 128 rows x 4 blocks, atom (r/128, kb/4) at ((r/128) * KBp/4 + kb/4) * 512,
// inside it row r at (r%32)*16 + ((r/32)%4)*4 and block kb at kb%4.
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t kb, int64_t kbp) {
    return ((r >> 7) * (kbp >> 2) + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

__host__ __device__ __forceinline__ int64_t scale_bytes(int64_t rows, int64_t K) {
    return ((rows + 127) / 128) * 128 * padded_blocks(K);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int check_shape(int64_t rows, int64_t K) {
    if (rows < 1 || rows > kMaxDim || K < kBlock || K > kMaxDim || K % kBlock != 0) return MACAQ_ESHAPE;
    return MACAQ_OK;
}

// Experts of a grouped (mixture-of-experts) linear, passed to its kernels by value.  x and y hold
// the tokens grouped by expert; the quantised activations give every expert a segment of whole
// 128-row blocks, so its scale atoms stay aligned; the weights are stacked [E][N][K].
constexpr int kMaxGroups = 128;

struct GroupTable {
    int groups;
    int rows[kMaxGroups];             // tokens of expert e
    int x_row[kMaxGroups];            // its first row in x and y
    int a_row[kMaxGroups + 1];        // its first row in the padded activation codes; a_row[E] = total
    int tile_start[kMaxGroups + 1];   // its first GEMM tile; tile_start[E] = all tiles
};

struct NoGroups {};

// Several linears on the same activations (the q, k and v projections of a layer, or gate and up),
// each with its own per-channel scale and folded weights, run as one GEMM over their weights stacked
// by rows: weight tile t (128 rows) belongs to linear group_of(tile_start, groups, t), whose
// activation codes (x transformed with that linear's multipliers) start at row a_row of the codes.
struct SharedActGroups {
    int groups;
    int tile_start[kMaxGroups + 1];  // first 128-row weight tile of linear e; [groups] = all tiles
    int a_row[kMaxGroups];           // first row of linear e's activation codes
};

// The grouped quantiser's threads: expert e's tokens split into runs of `rpg` rows, its runs
// numbered from run_start[e]; run_start[E] = all runs (padding rows get no thread).
struct RowRuns {
    int rpg;
    int run_start[kMaxGroups + 1];
};

// Where the grouped kernels find the expert table: passed by value (built on the host from host
// counts) or in device memory (built by a kernel from device counts, so a router on the GPU needs
// no device-to-host copy).
struct HostGroups {
    GroupTable gt;
    RowRuns rr;
};
struct DeviceGroups {
    const GroupTable* gt;
    const RowRuns* rr;
};
__host__ __device__ __forceinline__ const GroupTable& group_table(const GroupTable& g) { return g; }
__host__ __device__ __forceinline__ const GroupTable& group_table(const HostGroups& g) { return g.gt; }
__host__ __device__ __forceinline__ const GroupTable& group_table(const DeviceGroups& g) { return *g.gt; }
__host__ __device__ __forceinline__ const RowRuns& row_runs(const HostGroups& g) { return g.rr; }
__host__ __device__ __forceinline__ const RowRuns& row_runs(const DeviceGroups& g) { return *g.rr; }

// The expert whose range [starts[e], starts[e + 1]) holds v (0 <= v < starts[E]); empty ranges
// are skipped.
__host__ __device__ __forceinline__ int group_of(const int* starts, int groups, int v) {
    int lo = 0, hi = groups - 1;
    while (lo < hi) {  // first e with starts[e + 1] > v
        const int mid = (lo + hi) >> 1;
        if (starts[mid + 1] > v)
            hi = mid;
        else
            lo = mid + 1;
    }
    return lo;
}

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ECUDA;
}

// Number of SMs of the current device (cached per device ordinal).
int sm_count();

// The driver's cuTensorMapEncodeTiled, looked up once through the runtime (no -lcuda needed);
// null if the driver does not provide it.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace macaq
