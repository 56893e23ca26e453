// gemm.cu -- block-scaled MXFP4 x MXFP4 GEMM on the sm_100a tensor cores, and the fused
// MACaQ W4A4 linear layer built on it.
//
// y[m][n] = sum_b 2^(eA[m][b]-127) 2^(eW[n][b]-127) sum_{i<32} e2m1(A[m][32b+i]) e2m1(W[n][32b+i])
// with fp32 accumulation (tcgen05.mma kind::mxf4, E8M0 scales, one per 32 elements), y in
// bf16 (round to nearest even) or fp32.  "MACaQ: Fast, Model Agnostic Calibrated
// Quantization for Low-Precision Weights and Activations", Abstract: MXFP4 W4A4 -- both
// operands of every linear layer are MXFP4; the W4A4 matmul is the dense contraction the
// method runs at inference time.
//
// Kernel design (one CTA per SM, persistent over output tiles):
//   tile       128 rows of the "P" operand (MMA M) x BN rows of the "Q" operand (MMA N),
//              K consumed 256 elements (128 bytes of codes per row) per pipeline stage.
//              P = A, Q = W for large M;  P = W, Q = A ("swap-AB") for small M, so the
//              weight rows fill the 128-row MMA and a few tokens form a narrow N.
//   warp 0     producer: TMA (128-byte swizzle) loads of both code tiles and linear bulk
//              copies of the matching 512-byte scale atoms into a STAGES-deep ring.
//   warp 1     allocates tensor memory; one lane issues, per stage, four tcgen05.mma
//              (K = 64 each), then commits the stage back to the producer and, per tile,
//              the accumulator to the epilogue.
//   warps 2-3  idle.
//   warps 4-7  scale warps, one per TMEM sub-partition: per stage they move the scale atoms
//              from shared memory into the stage's own TMEM scale buffer with tcgen05.st (the
//              MMA thread issues no tcgen05.cp) and signal the MMA thread.
//   warps 8-15 epilogue: two warps per TMEM sub-partition (warp w reads lanes of
//              sub-partition w % 4, one half of the tile's columns each) copy the fp32
//              accumulator into registers, hand the TMEM back to the MMA warp at once, then
//              convert and store y, so the next tile's mainloop overlaps the stores.
//   Each pipeline stage has its own TMEM scale buffer, free again once the stage's MMAs
//   have completed.  Accumulators are double-buffered when BN <= 128.  The first two
//   warpgroups hand registers to the epilogue's (setmaxnreg).  All waits are bounded (see
//   sm100.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <chrono>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

int launch_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                               uint8_t* Aq, uint8_t* As, cudaStream_t stream);
int launch_act_quant_plain(const uint16_t* x, int64_t M, int64_t K, uint8_t* Aq, uint8_t* As,
                           cudaStream_t stream);
int launch_act_quant_grouped(const uint16_t* x, int64_t K, const float* act_mult, uint8_t* Aq, uint8_t* As,
                             const GroupTable& gt, cudaStream_t stream);
int launch_act_quant_grouped_device(const uint16_t* x, int64_t T, int E, int64_t K, const float* act_mult, uint8_t* Aq,
                                    uint8_t* As, const DeviceGroups& dg, cudaStream_t stream);
int64_t device_groups_rpg(int64_t T, int E, int64_t K);
int launch_act_transform_quant_multi(const uint16_t* x, int64_t M, int64_t K, int G, const float* act_mult,
                                     int64_t seg_rows, uint8_t* Aq, uint8_t* As, cudaStream_t stream);

constexpr int kBM = 128;           // MMA M
constexpr int kStageK = 256;       // K elements per stage
constexpr int kStageKBytes = 128;  // code bytes per row per stage
constexpr int kGemmThreads = 512;  // producer, MMA, 2 idle, 4 scale and 8 epilogue warps
constexpr int kEpiThreads = 256;
constexpr int kLaunchRegs = 65536 / kGemmThreads;  // registers per thread at launch
constexpr int kLowRegs = 80;                        // producer, MMA and scale warpgroups
constexpr int kEpiRegs = 176;                       // epilogue warpgroups
static_assert(2 * 128 * kLowRegs + 2 * 128 * kEpiRegs <= kGemmThreads * kLaunchRegs,
              "the register split must fit in the registers the block is launched with");
constexpr int kStagingBytes = 8 * 2048;  // output staging of the TMA-store epilogue
// Critical-path cost of a stream-K fix-up, in K steps of the tile: a 128 x 256 fp32 partial
// round trip through L2 (measured ~24 steps of a 128 x 256 tile) or a narrow swap-AB one.
template <int BN>
constexpr int streamk_cost_steps() { return BN >= 256 ? 24 : 6; }

template <int BN>
struct TileCfg {
    static constexpr int kQBlocks = (BN + 127) / 128;  // 128-row scale atoms on the Q side
    static constexpr int kPBytes = kBM * kStageKBytes;
    static constexpr int kQBytes = BN * kStageKBytes;
    static constexpr int kSFPBytes = 1024;             // 2 atoms: 128 rows x 8 blocks
    static constexpr int kSFQBytes = 1024 * kQBlocks;
    static constexpr int kStageBytes = kPBytes + kQBytes + kSFPBytes + kSFQBytes;
    static constexpr int kNumAcc = BN <= 128 ? 2 : 1;
    static constexpr int kAccStride = ((BN + 31) / 32) * 32;
    static constexpr int kSFQColsPerGroup = 4 * kQBlocks;
    static constexpr int kSFBufCols = 8 + 2 * kSFQColsPerGroup;    // P: 2 groups x 4, then Q
    static constexpr int kSFBase = kNumAcc * kAccStride;           // one scale buffer per stage follows
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(kStageBytes % 1024 == 0, "stage alignment for the 128-byte swizzle");
};

// Tensor memory of a configuration: accumulators, then one scale buffer per stage.
template <int BN, int STAGES>
struct TileTmem {
    static constexpr int kColsUsed = TileCfg<BN>::kSFBase + STAGES * TileCfg<BN>::kSFBufCols;
    static constexpr int kCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                               : kColsUsed <= 256 ? 256 : 512;
    static_assert(kColsUsed <= 512, "tensor memory budget");
};

struct GemmParams {
    const uint8_t* sf_p;  // scales of P, MMA tile layout
    const uint8_t* sf_q;  // scales of Q
    int64_t p_rows, q_rows, K, kbp;
    void* y;
    int64_t ldy;          // elements per row of y
    int y_fp32;
    int num_p_tiles, num_q_tiles, num_k_tiles, q_row_blocks;
    int raster_group;     // pair kernel: activation panels per group of the tile order (pair_tile)
    int dp_tiles;         // tiles scheduled data-parallel (blockIdx.x + i * gridDim.x)
    const int* dp_tiles_dev;  // if set: the data-parallel tile count in device memory (device-built expert table)
    int64_t sk_units;     // K steps of the remaining tiles, split evenly over the first sk_count units
    int sk_count;         // scheduling units that take part in the split (<= the units launched)
    int64_t group_n;      // grouped linear: output features per expert (weights stacked [E][N][K])
    float* partials;      // stream-K fp32 partial accumulators, one 128 x BN slot per CTA
    uint64_t* flags;      // stream-K hand-off: one word per (partial slot, epilogue thread)
    uint64_t tag;         // this launch's value of a written flag word (unique per launch)
    uint64_t owner_tag;   // the value an owner waits for: tag (a fault-injection build can shift it)
    int tma_store;        // bf16 output written by TMA from shared memory (non-swap, N % 8 == 0)
};

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<uint32_t*>(&v);
}

// Store CH accumulator columns [qc, qc+CH) of P-row `prow`, in y's index space: only rows below
// p_end and columns below q_end exist (swap-AB: P indexes y's columns and Q its rows).
template <int CH, bool SWAP>
__device__ __forceinline__ void store_chunk(const GemmParams& prm, int64_t prow, int64_t qc, const uint32_t* r,
                                            int64_t p_end, int64_t q_end) {
    if (prow >= p_end) return;
    if constexpr (!SWAP) {
        const int64_t base = prow * prm.ldy + qc;
        const bool full = qc + CH <= q_end;
        if (prm.y_fp32) {
            float* y = static_cast<float*>(prm.y) + base;
            if (full && (prm.ldy % 4) == 0) {
#pragma unroll
                for (int j = 0; j < CH; j += 4)
                    *reinterpret_cast<uint4*>(y + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < CH; ++j)
                    if (qc + j < q_end) y[j] = __uint_as_float(r[j]);
            }
        } else {
            __nv_bfloat16* y = static_cast<__nv_bfloat16*>(prm.y) + base;
            if (full && (prm.ldy % 8) == 0) {
#pragma unroll
                for (int j = 0; j < CH; j += 8)
                    *reinterpret_cast<uint4*>(y + j) =
                        make_uint4(pack_bf16x2(r[j], r[j + 1]), pack_bf16x2(r[j + 2], r[j + 3]),
                                   pack_bf16x2(r[j + 4], r[j + 5]), pack_bf16x2(r[j + 6], r[j + 7]));
            } else {
#pragma unroll
                for (int j = 0; j < CH; ++j)
                    if (qc + j < q_end) y[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
            }
        }
    } else {
        // accumulator row = output column (feature), accumulator column = output row (token)
        if (prm.y_fp32) {
            float* y = static_cast<float*>(prm.y);
#pragma unroll
            for (int j = 0; j < CH; ++j)
                if (qc + j < q_end) y[(qc + j) * prm.ldy + prow] = __uint_as_float(r[j]);
        } else {
            __nv_bfloat16* y = static_cast<__nv_bfloat16*>(prm.y);
#pragma unroll
            for (int j = 0; j < CH; ++j)
                if (qc + j < q_end) y[(qc + j) * prm.ldy + prow] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
    }
}

// ------------------------------------------------------------------------ schedule
//
// Work of one CTA, identical for its producer, MMA and epilogue roles:
//   1. data-parallel tiles: tile = blockIdx.x + i * gridDim.x for tile < dp_tiles;
//   2. stream-K: the K steps ("units") of the remaining tiles, numbered tile-major, split
//      into gridDim.x contiguous, equal ranges; CTA c takes [U c / G, U (c+1) / G).
// A stream-K segment covering a whole tile is stored directly.  A tile split between CTAs
// is finished by its "owner", the CTA holding the tile's first K step: that segment is the
// last one of the owner's range, while the other contributors (the next CTAs) hold the
// rest of the tile as the FIRST segment of their ranges.  Each contributor writes its fp32
// partial accumulator to its own slot and counts its epilogue threads into the slot's flag;
// the owner waits (bounded) for each full count and adds the slots in CTA order, so the
// sum is deterministic, then stores y.  No CTA-wide barrier is involved, so a wait that
// gives up cannot strand other threads.
enum WorkKind : int { kFull = 0, kOwner = 1, kPartial = 2 };

struct Work {
    int tile, k0, k1, kind, c_last;
};

struct WorkIter {
    int dp_next, id, count, dp_tiles;
    int64_t pos, hi;

    // `id` of `count` scheduling units: the CTA for the one-CTA kernel, the CTA pair for the
    // pair kernel (both CTAs of a pair walk the same items).
    __device__ __forceinline__ WorkIter(const GemmParams& p, int id_, int count_) : id(id_), count(count_) {
        dp_tiles = p.dp_tiles_dev ? *p.dp_tiles_dev : p.dp_tiles;
        dp_next = id;
        pos = id < p.sk_count ? p.sk_units * id / p.sk_count : 0;
        hi = id < p.sk_count ? p.sk_units * (id + 1) / p.sk_count : 0;
    }

    __device__ __forceinline__ bool next(const GemmParams& p, Work& w) {
        const int KT = p.num_k_tiles;
        if (dp_next < dp_tiles) {
            w.tile = dp_next;
            w.k0 = 0;
            w.k1 = KT;
            w.kind = kFull;
            w.c_last = 0;
            dp_next += count;
            return true;
        }
        if (pos >= hi) return false;
        const int64_t ts = pos / KT;
        const int64_t t0 = ts * KT;
        const int64_t end = hi < t0 + KT ? hi : t0 + KT;
        w.tile = dp_tiles + static_cast<int>(ts);
        w.k0 = static_cast<int>(pos - t0);
        w.k1 = static_cast<int>(end - t0);
        if (w.k0 == 0 && w.k1 == KT) {
            w.kind = kFull;
        } else if (w.k0 == 0) {
            w.kind = kOwner;
            // last unit whose range holds a K step of this tile: max c with U c / count <= t0 + KT - 1
            const int64_t U = p.sk_units;
            w.c_last = static_cast<int>(((t0 + KT) * p.sk_count + U - 1) / U - 1);
        } else {
            w.kind = kPartial;
        }
        pos = end;
        return true;
    }
};

// Bound of an owner's wait for a contributor's stream-K flag.  A fault-injection build of the
// library (MACAQ_TEST_HOOKS, tests only) shortens it, so a test can make the wait run out: the
// owner then records MACAQ_ETIMEOUT in the device status and finishes its item.
#ifdef MACAQ_FLAG_WAIT_LIMIT
constexpr long long kFlagWaitLimitCycles = MACAQ_FLAG_WAIT_LIMIT;
#else
constexpr long long kFlagWaitLimitCycles = kWaitLimitCycles;
#endif

#ifdef MACAQ_TEST_HOOKS
// Added to the tag owners wait for (0: none): with 1 no contributor ever writes the awaited value.
static std::atomic<int64_t> g_test_owner_tag_offset{0};
static uint64_t owner_tag_of(uint64_t tag) { return tag + static_cast<uint64_t>(g_test_owner_tag_offset.load()); }
#else
static uint64_t owner_tag_of(uint64_t tag) { return tag; }
#endif

__device__ __forceinline__ uint64_t ld_acquire64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Per-thread state of an epilogue thread for one work item.
struct EpiCtx {
    int etid, lane, warp;
    int unit, units;              // scheduling unit of this CTA (CTA or pair) and their number
    int slot_self;                // this CTA's partial-sum slot
    int slot_stride, slot_off;    // contributor unit c -> its slot c * slot_stride + slot_off
    int64_t prow;                 // output row (P side) of this thread
    int64_t row0;                 // first output row of this warp's 32 rows
    int64_t q0;                   // first output column (Q side) of this warp's half of the tile
    int64_t p_end, q_end;         // exclusive limits of prow and of Q indices (see store_chunk)
    uint8_t* staging;             // this warp's 2 KB output staging buffer (TMA-store path)
};

// Owner of a split tile: waits (bounded) for each contributor's flag, adds its partial sums to
// `sum` (this thread's BN/2 columns, contributors in order) and clears the flag, so a later
// launch repeating this launch's tag (a CUDA graph replay) cannot take it for its own signal.
template <int BN>
__device__ __forceinline__ void sum_partials(const GemmParams& prm, const Work& w, int unit, int slot_stride,
                                             int slot_off, int etid, float* sum, int& abort) {
    constexpr int kHalf = BN / 2;
    const int64_t U = prm.sk_units, G = prm.sk_count;
    for (int c = unit + 1; c <= w.c_last; ++c) {
        if (U * c / G == U * (c + 1) / G) continue;  // empty range: no partial
        const int slot_id = c * slot_stride + slot_off;
        uint64_t* flag = prm.flags + static_cast<int64_t>(slot_id) * kEpiThreads + etid;
        if (!abort) {
            const long long t0 = clock64();
            while (ld_acquire64(flag) != prm.owner_tag) {
                if (clock64() - t0 > kFlagWaitLimitCycles) {
                    atomicExch(&g_device_status, MACAQ_ETIMEOUT);
                    abort = 1;
                    break;
                }
            }
        }
        const float4* slot = reinterpret_cast<const float4*>(prm.partials + static_cast<int64_t>(slot_id) * (kBM * BN));
#pragma unroll
        for (int j = 0; j < kHalf / 4; ++j) {
            const float4 q = __ldcg(slot + j * kEpiThreads + etid);
            sum[4 * j] += q.x;
            sum[4 * j + 1] += q.y;
            sum[4 * j + 2] += q.z;
            sum[4 * j + 3] += q.w;
        }
        __stcg(reinterpret_cast<unsigned long long*>(flag), 0ull);
    }
}

// After the accumulator of `w` is in registers (v = this thread's BN/2 fp32 columns): write a
// stream-K partial, or add the contributors' partials (owner), then store y.
template <int BN, bool SWAP>
__device__ __forceinline__ void finish_item(const GemmParams& prm, const CUtensorMap* tmap_y, const Work& w,
                                            const EpiCtx& e, uint32_t* v, int& abort) {
    constexpr int kHalf = BN / 2;
    constexpr int kChunk = kHalf >= 32 ? 32 : kHalf;
    if (w.kind == kPartial) {
        // fp32 partial to this CTA's slot, [chunk of 4 columns][epilogue thread]; then this
        // thread's flag word takes the launch's tag (release: after its part of the partial).
        // The owner's thread with the same index reads exactly this part and then clears the
        // word, so no flag is shared or counted, and every launch starts from cleared words
        // (a CUDA graph replays a captured launch with the same tag).
        float4* slot = reinterpret_cast<float4*>(prm.partials + static_cast<int64_t>(e.slot_self) * (kBM * BN));
#pragma unroll
        for (int j = 0; j < kHalf / 4; ++j)
            __stcg(slot + j * kEpiThreads + e.etid,
                   make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
        st_release(prm.flags + static_cast<int64_t>(e.slot_self) * kEpiThreads + e.etid, prm.tag);
        return;
    }
    if (w.kind == kOwner) {
        const int64_t U = prm.sk_units, G = prm.sk_count;
        for (int c = e.unit + 1; c <= w.c_last; ++c) {
            if (U * c / G == U * (c + 1) / G) continue;  // empty range: no partial
            const int slot_id = c * e.slot_stride + e.slot_off;
            uint64_t* flag = prm.flags + static_cast<int64_t>(slot_id) * kEpiThreads + e.etid;
            if (!abort) {
                const long long t0 = clock64();
                while (ld_acquire64(flag) != prm.owner_tag) {
                    if (clock64() - t0 > kFlagWaitLimitCycles) {
                        atomicExch(&g_device_status, MACAQ_ETIMEOUT);
                        abort = 1;
                        break;
                    }
                }
            }
            const float4* slot = reinterpret_cast<const float4*>(prm.partials + static_cast<int64_t>(slot_id) * (kBM * BN));
#pragma unroll
            for (int j = 0; j < kHalf / 4; ++j) {
                const float4 q = __ldcg(slot + j * kEpiThreads + e.etid);
                v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + q.x);
                v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + q.y);
                v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + q.z);
                v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + q.w);
            }
            // consumed: clear the word, so a later launch that repeats this tag (a graph replay)
            // cannot take it for its own contributor's signal
            __stcg(reinterpret_cast<unsigned long long*>(flag), 0ull);
        }
    }
    if constexpr (!SWAP && kHalf % 32 == 0) {
        if (prm.tma_store) {
            // bf16 tile through this warp's 2 KB staging buffer (32 rows x 64 B, 64-byte
            // swizzle: conflict-free 16-byte writes), then per 32 columns either a TMA store
            // (which clips at the matrix edge) when all 32 rows are below p_end, or -- where
            // the rows past p_end belong to someone else (the next expert of a grouped linear)
            // -- 16-byte stores of whole 64-byte row pieces, 8 rows per warp instruction,
            // each row checked against p_end.
            const bool whole = e.row0 + 32 <= e.p_end;
#pragma unroll
            for (int c = 0; c < kHalf; c += 32) {
                if (e.lane == 0) bulk_wait_group_read<0>();  // previous store has read the buffer
                __syncwarp();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t* r = v + c + 8 * q4;
                    *reinterpret_cast<uint4*>(e.staging + e.lane * 64 + 16 * (q4 ^ ((e.lane >> 1) & 3))) =
                        make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                                   pack_bf16x2(r[6], r[7]));
                }
                if (whole) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (e.lane == 0) {
                        tma_store_2d(tmap_y, e.staging, static_cast<int32_t>(e.q0 + c), static_cast<int32_t>(e.row0));
                        bulk_commit_group();
                    }
                } else {
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = i * 8 + (e.lane >> 2), q4 = e.lane & 3;
                        const int64_t row = e.row0 + rr, col = e.q0 + c + 8 * q4;
                        if (row >= e.p_end) continue;
                        const uint4 val = *reinterpret_cast<const uint4*>(e.staging + rr * 64 + 16 * (q4 ^ ((rr >> 1) & 3)));
                        uint16_t* dst = static_cast<uint16_t*>(prm.y) + row * prm.ldy + col;
                        if (col + 8 <= e.q_end) {
                            *reinterpret_cast<uint4*>(dst) = val;
                        } else {
                            const uint16_t* h = reinterpret_cast<const uint16_t*>(&val);
                            for (int j = 0; j < 8; ++j)
                                if (col + j < e.q_end) dst[j] = h[j];
                        }
                    }
                }
            }
            return;
        }
    }
#pragma unroll
    for (int c = 0; c < kHalf; c += kChunk) store_chunk<kChunk, SWAP>(prm, e.prow, e.q0 + c, v + c, e.p_end, e.q_end);
}

// Where one output tile of the one-CTA kernel lives: its first P and Q operand rows (TMA
// coordinates; the scale atoms of row r are in 128-row block r / 128), and the y coordinates of
// its accumulator row 0 / column 0 with their exclusive limits (store_chunk's index space).
struct TileRef {
    int64_t p_row, q_row;
    int64_t y_p, y_q, p_end, q_end;
};

template <int BN, bool SWAP, bool GROUPED, class GT>
__device__ __forceinline__ TileRef tile_ref(const GemmParams& prm, const GT& groups, int tile) {
    static_assert(SWAP || !std::is_same<GT, SharedActGroups>::value, "stacked linears run swap-AB");
    TileRef t;
    if constexpr (!GROUPED) {
        const int pt = tile % prm.num_p_tiles, qt = tile / prm.num_p_tiles;
        t.p_row = static_cast<int64_t>(pt) * kBM;
        t.q_row = static_cast<int64_t>(qt) * BN;
        t.y_p = t.p_row;
        t.y_q = t.q_row;
        t.p_end = prm.p_rows;
        t.q_end = prm.q_rows;
        if constexpr (std::is_same<GT, SharedActGroups>::value) {
            // stacked linears on one x (swap-AB: P = the stacked weights): the activation tile is
            // the one transformed for the linear this weight tile belongs to
            t.q_row += groups.a_row[group_of(groups.tile_start, groups.groups, pt)];
        }
    } else {
        const GroupTable& gt = group_table(groups);
        const int e = group_of(gt.tile_start, gt.groups, tile);
        const int local = tile - gt.tile_start[e];
        const int64_t rows = gt.rows[e], N = prm.group_n;
        if constexpr (!SWAP) {  // P: the expert's tokens (its padded segment), Q: its weights
            const int ptiles = static_cast<int>((rows + kBM - 1) / kBM);
            const int pt = local % ptiles, qt = local / ptiles;
            t.p_row = gt.a_row[e] + static_cast<int64_t>(pt) * kBM;
            t.q_row = e * N + static_cast<int64_t>(qt) * BN;
            t.y_p = gt.x_row[e] + static_cast<int64_t>(pt) * kBM;  // y rows
            t.p_end = gt.x_row[e] + rows;
            t.y_q = static_cast<int64_t>(qt) * BN;  // y columns
            t.q_end = N;
        } else {  // P: the expert's weights, Q: its tokens (one tile: BN >= every expert's tokens)
            t.p_row = e * N + static_cast<int64_t>(local) * kBM;
            t.q_row = gt.a_row[e];
            t.y_p = static_cast<int64_t>(local) * kBM;  // y columns
            t.p_end = N;
            t.y_q = gt.x_row[e];  // y rows
            t.q_end = gt.x_row[e] + rows;
        }
    }
    return t;
}

// The expert table tile_ref reads: the kernel parameter (host-built table, or no groups), or the
// shared-memory copy of a device-built table, so a tile's expert lookup (a binary search) reads
// shared memory instead of a chain of dependent global loads.
template <class GT>
__device__ __forceinline__ const auto& tile_table(const GT& gt, const int* s_table) {
    if constexpr (std::is_same<GT, DeviceGroups>::value)
        return *reinterpret_cast<const GroupTable*>(s_table);
    else
        return gt;
}

// GROUPED: a grouped (mixture-of-experts) linear; `gt` maps work tiles to experts.
template <int BN, int STAGES, bool SWAP, bool GROUPED = false,
          class GT = typename std::conditional<GROUPED, GroupTable, NoGroups>::type>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mxf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm, const __grid_constant__ GT gt) {
    using Cfg = TileCfg<BN>;
    constexpr int kTmemCols = TileTmem<BN, STAGES>::kCols;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* staging = smem + STAGES * Cfg::kStageBytes;  // per epilogue warp: 32 x 32 bf16 (non-swap)
    uint64_t* full = reinterpret_cast<uint64_t*>(staging + (SWAP ? 0 : kStagingBytes));
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;
    uint64_t* acc_full = sf_full + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // A device-built expert table is copied to shared memory once (visible after the barrier below;
    // it was written by a kernel that completed before the quantiser this GEMM follows had started).
    constexpr bool kDevTable = std::is_same<GT, DeviceGroups>::value;
    __shared__ __align__(16) int s_table[kDevTable ? sizeof(GroupTable) / 4 : 1];
    if constexpr (kDevTable) {
        const int* src = reinterpret_cast<const int*>(gt.gt);
        for (int i = threadIdx.x; i < static_cast<int>(sizeof(GroupTable) / 4); i += blockDim.x) s_table[i] = src[i];
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 4);  // the four scale warps
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kEpiThreads);
        }
        fence_mbar_init();
        prefetch_tmap(&tmap_p);
        prefetch_tmap(&tmap_q);
        if (prm.tma_store) prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    int abort = 0;

    if (warp < 8) setmaxnreg_dec<kLowRegs>();
    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            griddep_wait();  // operands may come from the kernel launched just before
            int stage = 0;
            uint32_t phase = 0;
            WorkIter it(prm, blockIdx.x, gridDim.x);
            Work w;
            while (!abort && it.next(prm, w)) {
                const TileRef t = tile_ref<BN, SWAP, GROUPED>(prm, tile_table(gt, s_table), w.tile);
                const uint8_t* sfp = prm.sf_p + (t.p_row / 128) * (prm.kbp / 4) * 512;
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, &abort)) break;
                    uint8_t* sb = smem + stage * Cfg::kStageBytes;
                    mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
                    tma_load_2d(sb, &tmap_p, kt * kStageKBytes, static_cast<int32_t>(t.p_row), &full[stage]);
                    tma_load_2d(sb + Cfg::kPBytes, &tmap_q, kt * kStageKBytes, static_cast<int32_t>(t.q_row),
                                &full[stage]);
                    bulk_load(sb + Cfg::kPBytes + Cfg::kQBytes, sfp + kt * 1024, 1024, &full[stage]);
#pragma unroll
                    for (int i = 0; i < Cfg::kQBlocks; ++i) {
                        int64_t qb = t.q_row / 128 + i;
                        if (qb >= prm.q_row_blocks) qb = prm.q_row_blocks - 1;  // rows past the end: masked
                        bulk_load(sb + Cfg::kPBytes + Cfg::kQBytes + Cfg::kSFPBytes + 1024 * i,
                                  prm.sf_q + static_cast<int64_t>(qb) * (prm.kbp / 4) * 512 + kt * 1024, 1024,
                                  &full[stage]);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // -------------------------------------------------------------- MMA issuer
            // instruction descriptor: E2M1 x E2M1 (kind::mxf4), UE8M0 scales, K-major A/B
            const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) | (1u << 23) |
                                   (static_cast<uint32_t>(kBM >> 4) << 24);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            WorkIter it(prm, blockIdx.x, gridDim.x);
            Work w;
            while (!abort && it.next(prm, w)) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, &abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * Cfg::kAccStride;
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&full[stage], phase, &abort)) break;
                    if (!mbar_wait(&sf_full[stage], phase, &abort)) break;
                    tc_fence_after();  // the scale warps' tcgen05.st precede these MMAs
                    const uint32_t sp = smem_u32(smem + stage * Cfg::kStageBytes);
                    const uint32_t sq = sp + Cfg::kPBytes;
                    const uint32_t tsfp = tmem_base + Cfg::kSFBase + stage * Cfg::kSFBufCols;
                    const uint32_t tsfq = tsfp + 8;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t g = j >> 1;
                        const uint32_t id = (j & 1) * 2;  // byte of the scale word: blocks 2j%4, 2j%4+1
                        const uint32_t sfa = (tsfp + 4 * g) | (id << 30);
                        const uint32_t sfb = (tsfq + Cfg::kSFQColsPerGroup * g) | (id << 30);
                        tc_mma_mxf4(d_tmem, desc_sw128(sp + 32 * j), desc_sw128(sq + 32 * j),
                                    idesc | (id << 29) | (id << 4), sfa, sfb, (kt != w.k0 || j != 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);  // frees the stage and its scale buffer once these MMAs have read them
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tc_commit(&acc_full[acc]);
                if (++acc == Cfg::kNumAcc) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ scale warps
        // Warp (4 + sub) writes TMEM lanes 32 sub .. 32 sub + 31 of the stage's scale buffer,
        // each lane 16 bytes of every atom (the bytes a 32x128b.warpx4 copy puts there):
        // columns 0-7 the two P atoms, then per 4-block group g the Q atoms of each 128-row
        // block, in the order of the MMA's scale addresses.  A stage is refilled only after
        // the MMAs of its previous use completed, so its TMEM buffer is free once it is full.
        constexpr int kVals = 2 + 2 * Cfg::kQBlocks;
        const int sub = warp & 3;
        int stage = 0;
        uint32_t phase = 0;
        WorkIter it(prm, blockIdx.x, gridDim.x);
        Work w;
        while (!abort && it.next(prm, w)) {
            for (int kt = w.k0; kt < w.k1; ++kt) {
                if (!mbar_wait(&full[stage], phase, &abort)) break;
                const uint8_t* ssfp = smem + stage * Cfg::kStageBytes + Cfg::kPBytes + Cfg::kQBytes + lane * 16;
                const uint8_t* ssfq = ssfp + Cfg::kSFPBytes;
                uint4 v[kVals];
                v[0] = *reinterpret_cast<const uint4*>(ssfp);
                v[1] = *reinterpret_cast<const uint4*>(ssfp + 512);
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int i = 0; i < Cfg::kQBlocks; ++i)
                        v[2 + g * Cfg::kQBlocks + i] = *reinterpret_cast<const uint4*>(ssfq + 1024 * i + 512 * g);
                const uint32_t taddr =
                    tmem_base + Cfg::kSFBase + stage * Cfg::kSFBufCols + (static_cast<uint32_t>(sub * 32) << 16);
                tmem_st16(taddr, reinterpret_cast<const uint32_t*>(&v[0]));
                if constexpr (kVals == 6) tmem_st8(taddr + 16, reinterpret_cast<const uint32_t*>(&v[4]));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ epilogue
        setmaxnreg_inc<kEpiRegs>();
        constexpr int kHalf = BN / 2;            // columns per epilogue warp
        constexpr int kChunk = kHalf >= 32 ? 32 : kHalf;
        const int sub = warp & 3;                // TMEM sub-partition this warp may read
        const int half = (warp - 8) >> 2;        // which half of the tile's columns
        const int etid = threadIdx.x - 256;      // 0..255 among the epilogue threads
        int acc = 0;
        uint32_t acc_phase = 0;
        WorkIter it(prm, blockIdx.x, gridDim.x);
        Work w;
        while (!abort && it.next(prm, w)) {
            const TileRef t = tile_ref<BN, SWAP, GROUPED>(prm, tile_table(gt, s_table), w.tile);
            // Narrow tiles (decode): the owner of a split tile adds its contributors' partial
            // sums while its own MMAs still run.  The contributors did their part of the tile
            // first in their ranges; the owner reaches the tile's first K steps last in its own.
            constexpr bool kEarlyPartials = kHalf <= 32;
            float pre[kEarlyPartials ? kHalf : 1];
            const bool early = kEarlyPartials && w.kind == kOwner;
            if constexpr (kEarlyPartials) {
                if (early) {
#pragma unroll
                    for (int j = 0; j < kHalf; ++j) pre[j] = 0.0f;
                    sum_partials<BN>(prm, w, blockIdx.x, 1, 0, etid, pre, abort);
                }
            }
            if (!mbar_wait(&acc_full[acc], acc_phase, &abort)) break;
            tc_fence_after();
            const int64_t prow = t.y_p + sub * 32 + lane;
            const uint32_t tbase = tmem_base + acc * Cfg::kAccStride + half * kHalf +
                                   (static_cast<uint32_t>(sub * 32) << 16);
            uint32_t v[kHalf];
#pragma unroll
            for (int c = 0; c < kHalf; c += kChunk) tmem_ld_cols<kChunk>(tbase + c, v + c);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);  // accumulator is in registers: TMEM is free again
            if (++acc == Cfg::kNumAcc) {
                acc = 0;
                acc_phase ^= 1u;
            }
            Work wf = w;
            if constexpr (kEarlyPartials) {
                if (early) {
#pragma unroll
                    for (int j = 0; j < kHalf; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + pre[j]);
                    wf.kind = kFull;  // the partials are in: store like a whole tile
                }
            }
            EpiCtx e;
            e.etid = etid;
            e.lane = lane;
            e.warp = warp;
            e.unit = blockIdx.x;
            e.units = gridDim.x;
            e.slot_self = blockIdx.x;
            e.slot_stride = 1;
            e.slot_off = 0;
            e.prow = prow;
            e.row0 = t.y_p + sub * 32;
            e.q0 = t.y_q + half * kHalf;
            e.p_end = t.p_end;
            e.q_end = t.q_end;
            e.staging = staging + (warp - 8) * 2048;
            finish_item<BN, SWAP>(prm, &tmap_y, wf, e, v, abort);
        }
        if (lane == 0) bulk_wait_group<0>();  // output stores complete before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------ CTA-pair kernel
//
// Prefill tiles of 256 x 256 on a cluster of two CTAs (the two SMs of a TPC) sharing one
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64):
//   - each CTA TMA-loads its own 128 rows of the activation tile and its own 128 rows of the
//     weight tile per K step, so a weight panel crosses L2 -> SM once per pair instead of once
//     per CTA (32 KB of codes per CTA per K step instead of 48 KB), completing on the even
//     CTA's "full" barrier;
//   - each CTA also loads the K step's scale atoms (its 128 activation rows, all 256 weight
//     rows: 3 KB) into the same stage, completing on its own "sf_smem" barrier.  Four "scale
//     warps" per CTA, one per TMEM sub-partition, move them from shared memory into that
//     stage's TMEM scale buffer with tcgen05.st, in the layout a 32x128b.warpx4 copy gives
//     (each lane's four columns hold 16 bytes of an atom, repeated in every sub-partition),
//     and arrive on the even CTA's "sf_full" barrier.  Issuing the copies as tcgen05.cp from
//     the MMA thread instead puts six copies per K step into the MMA issue stream (measured:
//     64.4 us against 53 us for the Llama-3-8B up projection, 2048 x 4096 x 14336);
//   - the even CTA's single MMA thread waits for both barriers, issues the pair MMAs and
//     multicasts each stage's release to both CTAs' "empty" barriers (which also free the
//     stage's TMEM scale buffer) and each tile's completion to both "acc_full" barriers;
//   - each CTA's eight epilogue warps drain its 128 accumulator rows and release them on the
//     even CTA's "acc_empty" barrier (512 arrivals: both CTAs).
// 512 threads: warp 0 producer, warp 1 TMEM allocation and MMA issue, warps 2-3 idle, warps
// 4-7 scale warps, warps 8-15 epilogue.  The first two warpgroups give registers to the
// epilogue's (setmaxnreg), which holds 128 accumulator columns per thread.
// Scheduling (data-parallel waves then stream-K) works on pairs; partial-sum slots stay per CTA.
constexpr int kPairStages = 5;
constexpr int kPairThreads = kGemmThreads;  // same warp roles and register split
struct PairCfg {
    static constexpr int kABytes = 128 * kStageKBytes;     // this CTA's 128 activation rows
    static constexpr int kBBytes = 128 * kStageKBytes;     // this CTA's 128 weight rows
    static constexpr int kSFABytes = 1024;                 // 128 rows x 8 blocks
    static constexpr int kSFBBytes = 2048;                 // all 256 weight rows x 8 blocks
    static constexpr int kCodeBytes = kABytes + kBBytes;
    static constexpr int kStageBytes = kCodeBytes + kSFABytes + kSFBBytes;
    static constexpr int kSFBufCols = 8 + 16;              // SFA 2 groups x 4, SFB 2 groups x 8
    static constexpr int kSFBase = 256;                    // after the 256-column accumulator
    static constexpr int kTmemCols = 512;
    static_assert(kStageBytes % 1024 == 0, "stage alignment for the 128-byte swizzle");
    static_assert(kSFBase + kPairStages * kSFBufCols <= kTmemCols, "tensor memory budget");
};

// Order of the pair kernel's 256 x 256 tiles: groups of `raster_group` activation panels (256
// rows each), the last group possibly smaller; within a group the weight panel varies slowest
// and the activation panel fastest.  A wave of consecutive tiles then touches about
// raster_group activation panels and (pairs / raster_group) weight panels, and a group's
// activation panels are reused from L2 across the waves that sweep the weight panels, instead
// of every wave streaming the whole weight matrix again (activation-major order: each wave
// touches every weight panel).  Tile numbers past dp_tiles (stream-K) follow the same order.
__device__ __forceinline__ void pair_tile(const GemmParams& prm, int tile, int& pt, int& qt) {
    const int per_group = prm.raster_group * prm.num_q_tiles;
    const int g = tile / per_group;
    const int local = tile - g * per_group;
    const int first = g * prm.raster_group;
    const int rows = prm.num_p_tiles - first < prm.raster_group ? prm.num_p_tiles - first : prm.raster_group;
    pt = first + local % rows;
    qt = local / rows;
}

// GT = SharedActGroups: stacked linears on one x (weights = B, stacked by rows; tile_start counts
// 256-row weight tiles); each weight tile's activation panel is taken from its linear's segment.
template <int STAGES, class GT = NoGroups>
__global__ void __launch_bounds__(kPairThreads, 1)
    mxf4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                          const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm,
                          const __grid_constant__ GT gt) {
    using Cfg = PairCfg;
    constexpr int BN = 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* staging = smem + STAGES * Cfg::kStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(staging + kStagingBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_smem = empty + STAGES;
    uint64_t* sf_full = sf_smem + STAGES;
    uint64_t* acc_full = sf_full + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_smem[s], 1);
            mbar_init(&sf_full[s], 8);  // four scale warps in each CTA
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * kEpiThreads);
        fence_mbar_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_sfa);
        prefetch_tmap(&tmap_sfb);
        if (prm.tma_store) prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers and tensor memory exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    int abort = 0;

    if (warp < 8) setmaxnreg_dec<kLowRegs>();
    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------- producer (both CTAs)
            griddep_wait();
            int stage = 0;
            uint32_t phase = 0;
            WorkIter it(prm, pair, pairs);
            Work w;
            while (!abort && it.next(prm, w)) {
                int pt, qt;
                pair_tile(prm, w.tile, pt, qt);
                int a_base = 0;  // first activation row of this tile's linear (a multiple of 128)
                if constexpr (std::is_same<GT, SharedActGroups>::value)
                    a_base = gt.a_row[group_of(gt.tile_start, gt.groups, qt)];
                const int a_row = a_base + pt * 256 + static_cast<int>(rank) * 128;
                const int b_row = qt * 256 + static_cast<int>(rank) * 128;
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, &abort)) break;
                    uint8_t* sb = smem + stage * Cfg::kStageBytes;
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::kCodeBytes);
                    tma_load_2d_pair(sb, &tmap_a, kt * kStageKBytes, a_row, &full[stage]);
                    tma_load_2d_pair(sb + Cfg::kABytes, &tmap_b, kt * kStageKBytes, b_row, &full[stage]);
                    // scale atoms: 1 KB (two 512-byte atoms) per 128 rows per K step, as uint32 boxes
                    uint8_t* sf = sb + Cfg::kCodeBytes;
                    mbar_arrive_expect_tx(&sf_smem[stage], Cfg::kSFABytes + Cfg::kSFBBytes);
                    tma_load_2d(sf, &tmap_sfa, kt * 256, a_base / 128 + 2 * pt + static_cast<int>(rank),
                                &sf_smem[stage]);
                    tma_load_2d(sf + 1024, &tmap_sfb, kt * 256, 2 * qt, &sf_smem[stage]);
                    tma_load_2d(sf + 2048, &tmap_sfb, kt * 256, 2 * qt + 1, &sf_smem[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (even CTA only)
            const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) | (1u << 23) |
                                   (static_cast<uint32_t>(256 >> 4) << 24);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase = 0;
            WorkIter it(prm, pair, pairs);
            Work w;
            while (!abort && it.next(prm, w)) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1u, &abort)) break;
                acc_phase ^= 1u;
                tc_fence_after();
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&full[stage], phase, &abort)) break;
                    if (!mbar_wait(&sf_full[stage], phase, &abort)) break;
                    tc_fence_after();  // the scale warps' tcgen05.st precede these MMAs
                    const uint32_t sp = smem_u32(smem + stage * Cfg::kStageBytes);
                    const uint32_t sq = sp + Cfg::kABytes;
                    const uint32_t tsfa = tmem_base + Cfg::kSFBase + stage * Cfg::kSFBufCols;
                    const uint32_t tsfb = tsfa + 8;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t g = j >> 1;
                        const uint32_t id = (j & 1) * 2;
                        const uint32_t sfa = (tsfa + 4 * g) | (id << 30);
                        const uint32_t sfb = (tsfb + 8 * g) | (id << 30);
                        tc_mma_mxf4_pair(tmem_base, desc_sw128(sp + 32 * j), desc_sw128(sq + 32 * j),
                                         idesc | (id << 29) | (id << 4), sfa, sfb, (kt != w.k0 || j != 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&empty[stage]);  // frees the stage and its scale buffer in both CTAs
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tc_commit_pair(acc_full);
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // -------------------------------------------------------- scale warps (both CTAs)
        // Warp (4 + sub) writes TMEM lanes 32 sub .. 32 sub + 31 of each stage's scale buffer:
        // columns 0-7 the activation atoms (rows of this CTA), 8-23 the weight atoms (all 256
        // rows of the tile), ordered as the MMA's scale addresses expect.  The stage's smem
        // was refilled only after its previous MMAs completed, so its TMEM buffer is free too.
        const int sub = warp & 3;
        int stage = 0;
        uint32_t phase = 0;
        WorkIter it(prm, pair, pairs);
        Work w;
        while (!abort && it.next(prm, w)) {
            for (int kt = w.k0; kt < w.k1; ++kt) {
                if (!mbar_wait(&sf_smem[stage], phase, &abort)) break;
                const uint8_t* sf = smem + stage * Cfg::kStageBytes + Cfg::kCodeBytes + lane * 16;
                uint4 v[6];
                v[0] = *reinterpret_cast<const uint4*>(sf);          // SFA atom 0
                v[1] = *reinterpret_cast<const uint4*>(sf + 512);    // SFA atom 1
                v[2] = *reinterpret_cast<const uint4*>(sf + 1024);   // SFB rows 0-127, atom 0
                v[3] = *reinterpret_cast<const uint4*>(sf + 2048);   // SFB rows 128-255, atom 0
                v[4] = *reinterpret_cast<const uint4*>(sf + 1536);   // SFB rows 0-127, atom 1
                v[5] = *reinterpret_cast<const uint4*>(sf + 2560);   // SFB rows 128-255, atom 1
                const uint32_t taddr =
                    tmem_base + Cfg::kSFBase + stage * Cfg::kSFBufCols + (static_cast<uint32_t>(sub * 32) << 16);
                tmem_st16(taddr, reinterpret_cast<const uint32_t*>(&v[0]));
                tmem_st8(taddr + 16, reinterpret_cast<const uint32_t*>(&v[4]));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(&sf_full[stage]);
                    else
                        mbar_arrive_cluster(&sf_full[stage], 0);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp >= 8) {
        // ----------------------------------------------------------- epilogue (both CTAs)
        setmaxnreg_inc<kEpiRegs>();
        constexpr int kHalf = BN / 2;
        const int sub = warp & 3;
        const int half = (warp - 8) >> 2;
        const int etid = threadIdx.x - 256;
        uint32_t acc_phase = 0;
        WorkIter it(prm, pair, pairs);
        Work w;
        while (!abort && it.next(prm, w)) {
            int pt, qt;
            pair_tile(prm, w.tile, pt, qt);
            if (!mbar_wait(acc_full, acc_phase, &abort)) break;
            acc_phase ^= 1u;
            tc_fence_after();
            const int64_t row0 = static_cast<int64_t>(pt) * 256 + rank * 128 + sub * 32;
            const uint32_t tbase = tmem_base + half * kHalf + (static_cast<uint32_t>(sub * 32) << 16);
            uint32_t v[kHalf];
#pragma unroll
            for (int c = 0; c < kHalf; c += 32) tmem_ld_cols<32>(tbase + c, v + c);
            tmem_ld_wait();
            tc_fence_before();
            if (leader)
                mbar_arrive(acc_empty);
            else
                mbar_arrive_cluster(acc_empty, 0);
            EpiCtx e;
            e.etid = etid;
            e.lane = lane;
            e.warp = warp;
            e.unit = pair;
            e.units = pairs;
            e.slot_self = blockIdx.x;
            e.slot_stride = 2;
            e.slot_off = static_cast<int>(rank);
            e.prow = row0 + lane;
            e.row0 = row0;
            e.p_end = prm.p_rows;
            e.q_end = prm.q_rows;
            e.q0 = static_cast<int64_t>(qt) * BN + half * kHalf;
            e.staging = staging + (warp - 8) * 2048;
            finish_item<BN, false>(prm, &tmap_y, w, e, v, abort);
        }
        if (lane == 0) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's shared memory and tensor memory are no longer in use
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
}

// --------------------------------------------------------------------------- host side

// Tensor map of an MXFP4 code matrix [rows][K/2] bytes: boxes of box_rows x 128 bytes,
// 128-byte swizzle, zero fill past the edges (ragged M, N and K tails).
static bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kStageKBytes), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map of an E8M0 scale buffer in the MMA tile layout, viewed as uint32 [row blocks]
// [KBp * 32]: one box = 256 words = the two 512-byte atoms of one 128-row block for one
// 256-element K step.
static bool make_sf_map(CUtensorMap* map, const uint8_t* scales, int64_t rows, int64_t K) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    const int64_t kbp = padded_blocks(K);
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kbp * 32), static_cast<cuuint64_t>((rows + 127) / 128)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kbp * 128)};
    cuuint32_t box[2] = {256, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(scales), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool SWAP>
static int smem_bytes() {
    return STAGES * TileCfg<BN>::kStageBytes + (SWAP ? 0 : kStagingBytes) + (3 * STAGES + 4) * 8 + 16 + 1024;
}

// Tensor map of the bf16 output [rows][cols]: 32 x 32 boxes, 64-byte swizzle.
static bool make_out_map(CUtensorMap* map, void* y, int64_t rows, int64_t cols, int64_t ldy) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldy * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// setmaxnreg.inc takes registers from those the block was launched with: a kernel built with
// fewer than the split assumes would wait forever there, so it is never launched.
static bool register_split_fits(const cudaFuncAttributes& fa) {
    return fa.numRegs * kGemmThreads >= 2 * 128 * kLowRegs + 2 * 128 * kEpiRegs;
}

// Per-device cache of a launch-configuration query (the answers depend only on the device).
template <class F>
static int cached_per_device(int (&cache)[64], F&& query) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return query();
    if (cache[dev] == 0) {
        const int v = query();
        cache[dev] = v > 0 ? v : -1;
    }
    return cache[dev] > 0 ? cache[dev] : 0;
}

// CTAs of the persistent grid: SMs x resident CTAs per SM (shared memory and TMEM permitting).
template <int BN, int STAGES, bool SWAP>
static int grid_ctas_query();

template <int BN, int STAGES, bool SWAP>
static int grid_ctas() {
    static int cache[64] = {0};
    return cached_per_device(cache, [] { return grid_ctas_query<BN, STAGES, SWAP>(); });
}

template <int BN, int STAGES, bool SWAP>
static int grid_ctas_query() {
    auto kernel = mxf4_gemm_kernel<BN, STAGES, SWAP>;
    const int smem = smem_bytes<BN, STAGES, SWAP>();
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || !register_split_fits(fa)) {
        cudaGetLastError();
        return -1;
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1;
    // all of the unified L1/shared storage as shared memory, so small configurations fit twice per SM
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return -1;
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kGemmThreads, smem) != cudaSuccess || occ < 1)
        occ = 1;
    if (occ * TileTmem<BN, STAGES>::kCols > 512) occ = 512 / TileTmem<BN, STAGES>::kCols;
    return sm_count() * occ;  // occ is 1: the runtime keeps tensor-memory kernels at one CTA per SM
}

// Stream-K scratch of one launch: a flag per CTA (rounded to 256 B) and an fp32 partial
// accumulator slot (128 x BN) per CTA.
// Schedule of the persistent grid over `tiles` output tiles of KT K steps on `units`
// scheduling units (CTAs, or CTA pairs), chosen by its estimated critical path in K steps:
//   data-parallel  ceil(tiles / units) rounds of whole tiles;
//   stream-K       all but the last full wave data-parallel, the K steps of the rest split
//                  evenly over the units, plus the fix-up's cost `streamk_cost` (needs the
//                  stream-K scratch).  A tile is split at most in two when it is short (<= 32
//                  K steps), else in pieces of at least 16 K steps and at most four: the owner
//                  waits for and reads its contributors' partials one after another, and each
//                  one measured 1-2.5 us (a 1024-row weight matrix at decode, split eighteen
//                  ways over 148 CTAs, took 19.5 us for 2.8 MB of weights; in two, 8.3 us),
//                  while long tiles need all SMs streaming (the 25600-deep decode down
//                  projection in two pieces: 23.0 us on 80 CTAs against 20.2 us on 148).
// (Splitting only the leftover tiles, each over a few units, measured slower on B200: the
// owner reads its contributors' partials one after another.)
struct Schedule {
    int dp_tiles = 0;
    int64_t sk_units = 0;
    int sk_count = 0;
    int64_t grid = 0;  // units launched
};

static Schedule plan_schedule(int64_t tiles, int64_t units, int KT, bool scratch, int streamk_cost) {
    const int64_t full = tiles / units, rem = tiles % units;
    const int64_t est_dp = (full + (rem ? 1 : 0)) * KT;
    const int64_t dp = (full > 0 ? full - 1 : 0) * units;
    const int64_t sk_units = (tiles - dp) * static_cast<int64_t>(KT);
    const int64_t half = (KT + 1) / 2, quarter = (KT + 3) / 4;
    const int64_t min_steps = half < (quarter > 16 ? quarter : 16) ? half : (quarter > 16 ? quarter : 16);
    int64_t split = (sk_units + min_steps - 1) / min_steps;
    if (split > units) split = units;
    const int64_t est_sk = (dp / units) * KT + (sk_units + split - 1) / split + streamk_cost;
    Schedule s;
    if (scratch && rem != 0 && KT > 1 && est_sk <= est_dp) {
        s.dp_tiles = static_cast<int>(dp);
        s.sk_units = sk_units;
        s.sk_count = static_cast<int>(split);  // units 0 .. split-1 share the K steps
        s.grid = dp > 0 ? units : split;        // all units when whole tiles precede the split
    } else {
        s.dp_tiles = static_cast<int>(tiles);
        s.grid = units < tiles ? units : tiles;
    }
    return s;
}

// Stream-K scratch: a flag word per (CTA slot, epilogue thread), then one 128 x BN fp32
// partial-sum slot per CTA.  A flag counts as set only when it holds the tag of the current
// launch, and the owner clears every flag it consumed, so the scratch needs no initialisation
// (any contents on entry are fine) and a CUDA graph may replay a captured launch, tag included.
static size_t streamk_flag_bytes(int ctas) {
    return (static_cast<size_t>(ctas) * kEpiThreads * 8 + 255) / 256 * 256;
}

template <int BN>
static size_t streamk_bytes(int ctas) {
    return streamk_flag_bytes(ctas) + static_cast<size_t>(ctas) * kBM * BN * 4;
}

// A value no flag word of any earlier launch in this process holds: a per-process random
// start, then one step per launch.
static uint64_t next_launch_tag() {
    static std::atomic<uint64_t> next{[] {
        const uint64_t t = static_cast<uint64_t>(std::chrono::high_resolution_clock::now().time_since_epoch().count());
        return (t * 0x9E3779B97F4A7C15ull) | 1ull;
    }()};
    return next.fetch_add(2, std::memory_order_relaxed);
}

struct GemmOperands {
    const uint8_t *pq, *ps, *qq, *qs;
    int64_t p_rows, q_rows, K;
    void* y;
    int64_t ldy;
    int y_fp32;
    int64_t q_map_rows = 0;  // rows of Q's codes and scales if more than q_rows (stacked linears)
    int64_t p_map_rows = 0;  // the same for P (pair kernel: the activations)
};

// Scratch of the stream-K schedule (nullptr: data-parallel schedule only).
struct GemmScratch {
    void* ptr;
    size_t bytes;
};

// Shared-memory attributes of one kernel instantiation, set once per device.
template <int BN, int STAGES, bool SWAP, bool GROUPED, class GT>
static bool kernel_attributes() {
    static int cache[64] = {0};
    return cached_per_device(cache, [] {
               auto kernel = mxf4_gemm_kernel<BN, STAGES, SWAP, GROUPED, GT>;
               const int smem = smem_bytes<BN, STAGES, SWAP>();
               cudaFuncAttributes fa;
               if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || !register_split_fits(fa)) {
                   cudaGetLastError();
                   return -1;
               }
               return (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess &&
                       cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) == cudaSuccess)
                          ? 1
                          : -1;
           }) == 1;
}

// Shape of a grouped launch: rows of y, the tile count (an upper bound when the expert table is in
// device memory, whose own count `tiles_dev` the kernel reads), output features per expert.
struct GroupedShape {
    int64_t y_rows, tiles, group_n;
    const int* tiles_dev;
};

// GT = GroupTable (host-built, by value) or DeviceGroups (device-built): `groups` maps the work tiles
// to experts (data-parallel schedule, no scratch); the operands are the padded activation codes and
// the stacked weights, y is [tokens][N].  GT = NoGroups: a plain GEMM.
template <int BN, int STAGES, bool SWAP, class GT = NoGroups>
static int launch_gemm(const GemmOperands& op, const GemmScratch& ws, cudaStream_t stream, bool pdl,
                       const GT& groups = GT{}, const GroupedShape* gs = nullptr) {
    using Cfg = TileCfg<BN>;
    constexpr bool GROUPED = std::is_same<GT, GroupTable>::value || std::is_same<GT, DeviceGroups>::value;
    if (!std::is_same<GT, NoGroups>::value && !kernel_attributes<BN, STAGES, SWAP, GROUPED, GT>()) return MACAQ_ECUDA;
    const int64_t q_map_rows = op.q_map_rows > op.q_rows ? op.q_map_rows : op.q_rows;
    CUtensorMap mp, mq;
    if (!make_codes_map(&mp, op.pq, op.p_rows, op.K, kBM) || !make_codes_map(&mq, op.qq, q_map_rows, op.K, BN))
        return MACAQ_ECUDA;
    GemmParams prm{};
    prm.sf_p = op.ps;
    prm.sf_q = op.qs;
    prm.p_rows = op.p_rows;
    prm.q_rows = op.q_rows;
    prm.K = op.K;
    prm.kbp = padded_blocks(op.K);
    prm.y = op.y;
    prm.ldy = op.ldy;
    prm.y_fp32 = op.y_fp32;
    prm.num_p_tiles = static_cast<int>((op.p_rows + kBM - 1) / kBM);
    prm.num_q_tiles = static_cast<int>((op.q_rows + BN - 1) / BN);
    prm.num_k_tiles = static_cast<int>((op.K + kStageK - 1) / kStageK);
    prm.q_row_blocks = static_cast<int>((q_map_rows + 127) / 128);

    const int ctas = grid_ctas<BN, STAGES, SWAP>();
    if (ctas < 1) return MACAQ_ECUDA;
    CUtensorMap my;
    // y is [p_rows][q_rows], or for a grouped linear [tokens][group_n]
    const int64_t y_rows = GROUPED ? gs->y_rows : op.p_rows;
    const int64_t y_cols = GROUPED ? gs->group_n : op.q_rows;
    prm.tma_store = (!SWAP && !op.y_fp32 && op.ldy % 8 == 0) ? 1 : 0;
    if (prm.tma_store && !make_out_map(&my, op.y, y_rows, y_cols, op.ldy)) return MACAQ_ECUDA;
    if (!prm.tma_store) my = mq;  // unused placeholder
    const int64_t tiles = GROUPED ? gs->tiles : static_cast<int64_t>(prm.num_p_tiles) * prm.num_q_tiles;
    if (tiles == 0) return MACAQ_OK;
    prm.group_n = GROUPED ? gs->group_n : 0;
    prm.dp_tiles_dev = GROUPED ? gs->tiles_dev : nullptr;
    const bool scratch = !GROUPED && ws.ptr != nullptr && ws.bytes >= streamk_bytes<BN>(ctas);
    const Schedule sch = plan_schedule(tiles, ctas, prm.num_k_tiles, scratch, streamk_cost_steps<BN>());
    const int64_t grid = sch.grid;
    prm.dp_tiles = sch.dp_tiles;
    prm.sk_units = sch.sk_units;
    prm.sk_count = sch.sk_count;
    prm.flags = nullptr;
    prm.partials = nullptr;
    if (sch.sk_units > 0) {
        prm.flags = static_cast<uint64_t*>(ws.ptr);
        prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws.ptr) + streamk_flag_bytes(ctas));
        prm.tag = next_launch_tag();
        prm.owner_tag = owner_tag_of(prm.tag);
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem_bytes<BN, STAGES, SWAP>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, mxf4_gemm_kernel<BN, STAGES, SWAP, GROUPED, GT>, mp, mq, my, prm, groups) !=
        cudaSuccess)
        return MACAQ_ECUDA;
    return launch_status();
}

// Kernel configuration for M rows of activations: swap-AB with the narrowest N that holds
// the tokens for M <= 128, 128 x 256 tiles above.  `f` is called with the configuration.
static int pair_smem_bytes() {
    return kPairStages * PairCfg::kStageBytes + kStagingBytes + (4 * kPairStages + 2) * 8 + 16 + 1024;
}

static int gemm_pairs_query();

// CTA pairs that can be resident at once (two SMs of a TPC each); 0 if cluster launch fails.
static int gemm_pairs() {
    static int cache[64] = {0};
    return cached_per_device(cache, [] { return gemm_pairs_query(); });
}

static int gemm_pairs_query() {
    auto kernel = mxf4_gemm_pair_kernel<kPairStages>;
    const int smem = pair_smem_bytes();
    // setmaxnreg.inc takes registers from those the block was launched with: a kernel built
    // with fewer than the split assumes would wait forever there, so it is never launched.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (!register_split_fits(fa)) return 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sm_count() & ~1));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return clusters;
}

// Activation panels per group of the pair kernel's tile order: a wave of `pairs` tiles touches
// about g activation and pairs / g weight panels (equal sizes), fewest near g = sqrt(pairs).
static int pair_raster_group(int p_tiles, int pairs) {
    int g = 1;
    while ((g + 1) * (g + 1) <= pairs) ++g;
    return g < p_tiles ? g : p_tiles;
}

// Shared-memory attributes of a pair-kernel instantiation other than the plain one (which
// gemm_pairs_query sets), once per device.
template <class GT>
static bool pair_kernel_attributes() {
    static int cache[64] = {0};
    return cached_per_device(cache, [] {
               auto kernel = mxf4_gemm_pair_kernel<kPairStages, GT>;
               cudaFuncAttributes fa;
               if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || !register_split_fits(fa)) {
                   cudaGetLastError();
                   return -1;
               }
               return (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pair_smem_bytes()) ==
                           cudaSuccess &&
                       cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) == cudaSuccess)
                          ? 1
                          : -1;
           }) == 1;
}

template <class GT = NoGroups>
static int launch_gemm_pair(const GemmOperands& op, const GemmScratch& ws, int pairs, cudaStream_t stream, bool pdl,
                            const GT& groups = GT{}) {
    if (!std::is_same<GT, NoGroups>::value && !pair_kernel_attributes<GT>()) return MACAQ_ECUDA;
    const int64_t p_map_rows = op.p_map_rows > op.p_rows ? op.p_map_rows : op.p_rows;
    CUtensorMap ma, mb, msa, msb, my;
    if (!make_codes_map(&ma, op.pq, p_map_rows, op.K, 128) || !make_codes_map(&mb, op.qq, op.q_rows, op.K, 128) ||
        !make_sf_map(&msa, op.ps, p_map_rows, op.K) || !make_sf_map(&msb, op.qs, op.q_rows, op.K))
        return MACAQ_ECUDA;
    GemmParams prm{};
    prm.sf_p = op.ps;
    prm.sf_q = op.qs;
    prm.p_rows = op.p_rows;
    prm.q_rows = op.q_rows;
    prm.K = op.K;
    prm.kbp = padded_blocks(op.K);
    prm.y = op.y;
    prm.ldy = op.ldy;
    prm.y_fp32 = op.y_fp32;
    prm.num_p_tiles = static_cast<int>((op.p_rows + 255) / 256);
    prm.num_q_tiles = static_cast<int>((op.q_rows + 255) / 256);
    prm.num_k_tiles = static_cast<int>((op.K + kStageK - 1) / kStageK);
    prm.q_row_blocks = static_cast<int>((op.q_rows + 127) / 128);
    prm.raster_group = pair_raster_group(prm.num_p_tiles, pairs);
    prm.tma_store = (!op.y_fp32 && op.ldy % 8 == 0) ? 1 : 0;
    if (prm.tma_store && !make_out_map(&my, op.y, op.p_rows, op.q_rows, op.ldy)) return MACAQ_ECUDA;
    if (!prm.tma_store) my = ma;  // unused placeholder

    const int64_t tiles = static_cast<int64_t>(prm.num_p_tiles) * prm.num_q_tiles;
    const int ctas = 2 * pairs;
    const bool scratch = ws.ptr != nullptr && ws.bytes >= streamk_bytes<256>(ctas);
    const Schedule sch = plan_schedule(tiles, pairs, prm.num_k_tiles, scratch, streamk_cost_steps<256>());
    const int64_t grid_pairs = sch.grid;
    prm.dp_tiles = sch.dp_tiles;
    prm.sk_units = sch.sk_units;
    prm.sk_count = sch.sk_count;
    prm.flags = nullptr;
    prm.partials = nullptr;
    if (sch.sk_units > 0) {
        prm.flags = static_cast<uint64_t*>(ws.ptr);
        prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws.ptr) + streamk_flag_bytes(ctas));
        prm.tag = next_launch_tag();
        prm.owner_tag = owner_tag_of(prm.tag);
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * grid_pairs));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = pair_smem_bytes();
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, mxf4_gemm_pair_kernel<kPairStages, GT>, ma, mb, msa, msb, my, prm, groups) !=
        cudaSuccess)
        return MACAQ_ECUDA;
    return launch_status();
}

// A kernel that allocates tensor memory runs one CTA per SM, so each configuration takes
// as many pipeline stages as fit in the SM's shared memory.
template <class F>
static auto with_config(int64_t M, F&& f) {
    if (M <= 16) return f(std::integral_constant<int, 16>{}, std::integral_constant<int, 10>{}, std::true_type{});
    if (M <= 32) return f(std::integral_constant<int, 32>{}, std::integral_constant<int, 9>{}, std::true_type{});
    if (M <= 64) return f(std::integral_constant<int, 64>{}, std::integral_constant<int, 8>{}, std::true_type{});
    if (M <= 128) return f(std::integral_constant<int, 128>{}, std::integral_constant<int, 6>{}, std::true_type{});
    return f(std::integral_constant<int, 256>{}, std::integral_constant<int, 4>{}, std::false_type{});
}

// Large M runs on CTA pairs when the device can co-schedule them (the 256 x 256 pair tile).
static bool use_pairs(int64_t M) { return M > 128 && gemm_pairs() > 0; }

// CTAs whose stream-K flags the GEMM for M rows may use.
int gemm_ctas(int64_t M) {
    if (use_pairs(M)) return 2 * gemm_pairs();
    return with_config(M, [](auto bn, auto st, auto sw) -> int {
        return grid_ctas<decltype(bn)::value, decltype(st)::value, decltype(sw)::value>();
    });
}

size_t gemm_workspace_bytes(int64_t M) {
    if (use_pairs(M)) return streamk_bytes<256>(2 * gemm_pairs());
    return with_config(M, [](auto bn, auto st, auto sw) -> size_t {
        const int ctas = grid_ctas<decltype(bn)::value, decltype(st)::value, decltype(sw)::value>();
        return ctas < 1 ? 0 : streamk_bytes<decltype(bn)::value>(ctas);
    });
}

// y[M][N] = dec(A) dec(W)^T, row m of y at y + m * ldy elements (ldy = 0: N).  Small M runs
// swap-AB (weights on the MMA M side).
int run_mxfp4_gemm(const uint8_t* Aq, const uint8_t* As, int64_t M, const uint8_t* Wq, const uint8_t* Ws,
                   int64_t N, int64_t K, void* y, int y_fp32, const GemmScratch& ws, cudaStream_t stream, bool pdl,
                   int64_t ldy = 0) {
    if (ldy == 0) ldy = N;
    if (use_pairs(M)) {
        const GemmOperands op{Aq, As, Wq, Ws, M, N, K, y, ldy, y_fp32};
        return launch_gemm_pair(op, ws, gemm_pairs(), stream, pdl);
    }
    return with_config(M, [&](auto bn, auto st, auto sw) -> int {
        constexpr bool kSwap = decltype(sw)::value;
        const GemmOperands op = kSwap ? GemmOperands{Wq, Ws, Aq, As, N, M, K, y, ldy, y_fp32}
                                      : GemmOperands{Aq, As, Wq, Ws, M, N, K, y, ldy, y_fp32};
        return launch_gemm<decltype(bn)::value, decltype(st)::value, kSwap>(op, ws, stream, pdl);
    });
}

// Layout of the linear's workspace: activation codes, their scales, then the GEMM's stream-K
// scratch.
struct LinearWorkspace {
    uint8_t *Aq, *As, *gemm;
    size_t gemm_bytes;
};

static size_t round256(size_t v) { return (v + 255) / 256 * 256; }

LinearWorkspace linear_workspace_layout(void* base, int64_t M, int64_t K) {
    LinearWorkspace l;
    l.Aq = static_cast<uint8_t*>(base);
    l.As = l.Aq + round256(static_cast<size_t>(M * (K / 2)));
    l.gemm = l.As + round256(static_cast<size_t>(scale_bytes(M, K)));
    l.gemm_bytes = gemm_workspace_bytes(M);
    return l;
}

size_t linear_activation_bytes(int64_t M, int64_t K) {
    return round256(static_cast<size_t>(M * (K / 2))) + round256(static_cast<size_t>(scale_bytes(M, K)));
}

// The layer's forward pass on a laid-out workspace: the quantiser, then the GEMM launched with
// programmatic dependent launch so its set-up overlaps the quantiser's tail.  act_mult ==
// nullptr: plain MXFP4 of x (the "pure MXFP4" baseline).  `gemm_scratch`: whether l.gemm
// holds the stream-K scratch.
int run_linear(const uint16_t* x, int64_t M, int64_t K, const float* act_mult, const uint8_t* Wq, const uint8_t* Ws,
               int64_t N, uint16_t* y, const LinearWorkspace& l, bool gemm_scratch, cudaStream_t st) {
    const int rc = act_mult ? launch_act_transform_quant(x, M, K, act_mult, l.Aq, l.As, st)
                            : launch_act_quant_plain(x, M, K, l.Aq, l.As, st);
    if (rc) return rc;
    const GemmScratch ws{gemm_scratch ? l.gemm : nullptr, gemm_scratch ? l.gemm_bytes : 0};
    return run_mxfp4_gemm(l.Aq, l.As, M, Wq, Ws, N, K, y, 0, ws, st, true);
}

// Several linears on one x (the q, k and v projections, or gate and up), each with its own
// multipliers and folded weights, stacked by rows: Wq / Ws hold linear g's N[g] rows after those of
// the linears before it, and y [M][sum N] holds its outputs in the matching column block.  The
// workspace holds G segments of activation codes and scales, one per linear, each of whole
// 128-row blocks (plain MXFP4 of x: one segment, shared), then the GEMM's stream-K scratch.
size_t grouped_activation_bytes(int64_t padded_rows, int64_t K);

struct MultiWorkspace {
    uint8_t *Aq, *As, *gemm;
    size_t gemm_bytes, bytes;
    int64_t seg_rows;  // rows per linear's segment (a multiple of 128)
};

static MultiWorkspace multi_workspace_layout(void* base, int64_t M, int G, int64_t K) {
    MultiWorkspace l;
    l.seg_rows = (M + 127) / 128 * 128;
    const int64_t P = G * l.seg_rows;
    const size_t act = grouped_activation_bytes(P, K);
    l.Aq = static_cast<uint8_t*>(base);
    l.As = l.Aq + round256(static_cast<size_t>(P * (K / 2)));
    l.gemm = l.Aq + act;
    l.gemm_bytes = gemm_workspace_bytes(M);
    l.bytes = act + l.gemm_bytes;
    return l;
}

// One quantiser launch for all G linears; then ONE GEMM over the stacked weights, each weight tile
// paired with its own linear's activations, so the small k / v weights share the grid (and its
// waves) with the rest instead of each running on a few SMs: up to 128 tokens swap-AB with
// 128-row weight tiles, above on CTA pairs with 256-row weight tiles when every N[g] is a multiple
// of 256 (a tile then never spans two linears).  Otherwise one GEMM per linear, each into its
// column block of y.
static int run_linear_multi(const uint16_t* x, int64_t M, int64_t K, int G, const float* act_mult, const uint8_t* Wq,
                            const uint8_t* Ws, const int64_t* N, int64_t n_total, uint16_t* y,
                            const MultiWorkspace& l, cudaStream_t st) {
    const int64_t seg = act_mult ? l.seg_rows : 0;  // row offset between the linears' segments
    const int rc = act_mult ? launch_act_transform_quant_multi(x, M, K, G, act_mult, l.seg_rows, l.Aq, l.As, st)
                            : launch_act_quant_plain(x, M, K, l.Aq, l.As, st);
    if (rc) return rc;
    const GemmScratch ws{l.gemm, l.gemm_bytes};
    const int64_t kbp = padded_blocks(K);
    if (M <= 128) {
        SharedActGroups sg{};
        sg.groups = G;
        sg.tile_start[0] = 0;
        for (int g = 0; g < G; ++g) {
            sg.tile_start[g + 1] = sg.tile_start[g] + static_cast<int>(N[g] / 128);
            sg.a_row[g] = static_cast<int>(g * seg);
        }
        return with_config(M, [&](auto bn, auto stages, auto sw) -> int {
            if constexpr (decltype(sw)::value) {
                GemmOperands op{Wq, Ws, l.Aq, l.As, n_total, M, K, y, n_total, 0};
                op.q_map_rows = (G - 1) * seg + M;
                return launch_gemm<decltype(bn)::value, decltype(stages)::value, true, SharedActGroups>(op, ws, st,
                                                                                                        true, sg);
            } else {
                return MACAQ_EINVAL;  // not reached: up to 128 tokens always take a swap-AB configuration
            }
        });
    }
    bool whole_pair_tiles = true;
    for (int g = 0; g < G; ++g) whole_pair_tiles = whole_pair_tiles && N[g] % 256 == 0;
    if (use_pairs(M) && whole_pair_tiles) {
        SharedActGroups sg{};
        sg.groups = G;
        sg.tile_start[0] = 0;
        for (int g = 0; g < G; ++g) {
            sg.tile_start[g + 1] = sg.tile_start[g] + static_cast<int>(N[g] / 256);
            sg.a_row[g] = static_cast<int>(g * seg);
        }
        GemmOperands op{l.Aq, l.As, Wq, Ws, M, n_total, K, y, n_total, 0};
        op.p_map_rows = (G - 1) * seg + M;
        return launch_gemm_pair(op, ws, gemm_pairs(), st, true, sg);
    }
    int64_t n0 = 0;
    for (int g = 0; g < G; ++g) {
        const int64_t a0 = g * seg;
        // only the first GEMM is a programmatic dependent (of the quantiser); the rest follow the
        // GEMM before them in plain stream order, as they share its stream-K scratch
        if (int r = run_mxfp4_gemm(l.Aq + a0 * (K / 2), l.As + (a0 / 128) * 128 * kbp, M, Wq + n0 * (K / 2),
                                   Ws + (n0 / 128) * 128 * kbp, N[g], K, y + n0, 0, ws, st, g == 0, n_total))
            return r;
        n0 += N[g];
    }
    return MACAQ_OK;
}

// The group table of a grouped linear from the host token counts: tokens per expert, their rows in
// x / y and in the padded activation codes (whole 128-row blocks per expert), and the GEMM tiles
// per expert (swap-AB when no expert has more than 128 tokens: N / 128 weight tiles each; else
// 128-token x 256-feature tiles).  Returns MACAQ_ESHAPE for counts out of range.
static int build_group_table(const int64_t* counts, int E, int64_t N, GroupTable* gt, int64_t* max_rows) {
    if (E < 1 || E > kMaxGroups) return MACAQ_ESHAPE;
    gt->groups = E;
    int64_t x = 0, a = 0, mx = 0;
    for (int e = 0; e < E; ++e) {
        if (counts[e] < 0) return MACAQ_ESHAPE;
        gt->rows[e] = static_cast<int>(counts[e]);
        gt->x_row[e] = static_cast<int>(x);
        gt->a_row[e] = static_cast<int>(a);
        x += counts[e];
        a += (counts[e] + 127) / 128 * 128;
        mx = counts[e] > mx ? counts[e] : mx;
        if (a > kMaxDim) return MACAQ_ESHAPE;
    }
    gt->a_row[E] = static_cast<int>(a);
    int64_t t = 0;
    for (int e = 0; e < E; ++e) {
        gt->tile_start[e] = static_cast<int>(t);
        if (counts[e] > 0)
            t += mx <= 128 ? N / 128 : (counts[e] + 127) / 128 * ((N + 255) / 256);
    }
    gt->tile_start[E] = static_cast<int>(t);
    *max_rows = mx;
    return MACAQ_OK;
}

// The expert table from DEVICE counts (int32 or int64 [E]): the same quantities build_group_table
// computes on the host, plus the quantiser's runs of `rpg` rows.  One CTA of 128 threads, one
// expert each (E <= 128): the counts load in parallel, four running sums (x rows, padded rows,
// tiles, runs) come from one block-wide exclusive scan, and every entry is stored in parallel.
// Counts are made safe before use -- a negative count becomes 0 and a count that would run past
// the T rows of x is cut at T -- and an expert's rows beyond `capacity` are not computed (x keeps
// its layout); each correction records MACAQ_ECOUNTS in the device status, so no kernel ever indexes
// outside x, y or the workspace.  `swap`: every expert fits one swap-AB tile (capacity <= 128).
constexpr int kGroupThreads = kMaxGroups;

__device__ __forceinline__ longlong4 add4(longlong4 a, longlong4 b) {
    return make_longlong4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__global__ void __launch_bounds__(kGroupThreads) build_groups_kernel(
    const void* __restrict__ counts, int counts_bytes, int E, int64_t T, int64_t capacity, int64_t N, int swap, int rpg,
    GroupTable* __restrict__ gt, RowRuns* __restrict__ rr) {
    __shared__ longlong4 warp_sum[kGroupThreads / 32];
    __shared__ int64_t clamp_x[kGroupThreads];
    __shared__ int bad;
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    if (e == 0) bad = 0;
    __syncthreads();
    int64_t c = 0;
    if (e < E)
        c = counts_bytes == 4 ? static_cast<int64_t>(static_cast<const int32_t*>(counts)[e])
                              : static_cast<const int64_t*>(counts)[e];
    if (c < 0) {
        c = 0;
        bad = 1;
    }
    // 1. where expert e's rows start in x: exclusive scan of the counts, then the cut at T
    int64_t incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int64_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sum[warp].x = incl;
    __syncthreads();
    int64_t before = incl - c;
    for (int w = 0; w < warp; ++w) before += warp_sum[w].x;
    const int64_t x0 = before < T ? before : T;
    if (c > T - x0) {
        c = T - x0;
        bad = 1;
    }
    int64_t rows = c;
    if (rows > capacity) {
        rows = capacity;
        bad = 1;
    }
    clamp_x[e] = x0;
    __syncthreads();
    // 2. padded rows, tiles and runs of the rows computed: one more scan
    longlong4 v = make_longlong4((rows + 127) / 128 * 128,
                                 rows > 0 ? (swap ? N / 128 : (rows + 127) / 128 * ((N + 255) / 256)) : 0,
                                 (rows + rpg - 1) / rpg, 0);
    longlong4 inc4 = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        longlong4 o;
        o.x = __shfl_up_sync(0xFFFFFFFFu, inc4.x, off);
        o.y = __shfl_up_sync(0xFFFFFFFFu, inc4.y, off);
        o.z = __shfl_up_sync(0xFFFFFFFFu, inc4.z, off);
        o.w = 0;
        if (lane >= off) inc4 = add4(inc4, o);
    }
    __syncthreads();
    if (lane == 31) warp_sum[warp] = inc4;
    __syncthreads();
    longlong4 pre = make_longlong4(inc4.x - v.x, inc4.y - v.y, inc4.z - v.z, 0);
    for (int w = 0; w < warp; ++w) pre = add4(pre, warp_sum[w]);
    if (e < E) {
        gt->rows[e] = static_cast<int>(rows);
        gt->x_row[e] = static_cast<int>(clamp_x[e]);
        gt->a_row[e] = static_cast<int>(pre.x);
        gt->tile_start[e] = static_cast<int>(pre.y);
        rr->run_start[e] = static_cast<int>(pre.z);
    }
    if (e == E - 1) {
        gt->groups = E;
        gt->a_row[E] = static_cast<int>(pre.x + v.x);
        gt->tile_start[E] = static_cast<int>(pre.y + v.y);
        rr->run_start[E] = static_cast<int>(pre.z + v.z);
        rr->rpg = rpg;
    }
    __syncthreads();
    if (e == 0 && bad) atomicExch(&g_device_status, MACAQ_ECOUNTS);
}

// Layout of the device-count grouped linear's workspace: the expert table, the quantiser's runs,
// then the activation codes and scales for the most padded rows T tokens can need over E experts
// (each non-empty expert pads to whole 128-row blocks: T + 127 min(E, T), rounded up to 128).
struct DeviceGroupedWorkspace {
    GroupTable* gt;
    RowRuns* rr;
    uint8_t *Aq, *As;
    int64_t P;  // padded rows the codes can hold
    size_t bytes;
};

static DeviceGroupedWorkspace device_grouped_layout(void* base, int64_t T, int E, int64_t K) {
    DeviceGroupedWorkspace l;
    const int64_t nz = E < T ? E : T;
    l.P = (T + 127 * nz + 127) / 128 * 128;
    const size_t off_rr = round256(sizeof(GroupTable));
    const size_t off_aq = off_rr + round256(sizeof(RowRuns));
    const size_t off_as = off_aq + round256(static_cast<size_t>(l.P * (K / 2)));
    l.bytes = off_as + round256(static_cast<size_t>(scale_bytes(l.P, K)));
    uint8_t* p = static_cast<uint8_t*>(base);
    l.gt = reinterpret_cast<GroupTable*>(p);
    l.rr = reinterpret_cast<RowRuns*>(p + off_rr);
    l.Aq = p + off_aq;
    l.As = p + off_as;
    return l;
}

size_t grouped_activation_bytes(int64_t padded_rows, int64_t K) {
    return round256(static_cast<size_t>(padded_rows * (K / 2))) +
           round256(static_cast<size_t>(scale_bytes(padded_rows, K)));
}

}  // namespace macaq

using namespace macaq;

extern "C" size_t macaq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (check_shape(M, K) != MACAQ_OK || check_shape(N, K) != MACAQ_OK) return 0;
    return gemm_workspace_bytes(M);
}

extern "C" size_t macaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (check_shape(M, K) != MACAQ_OK || check_shape(N, K) != MACAQ_OK) return 0;
    return linear_activation_bytes(M, K) + gemm_workspace_bytes(M);
}

extern "C" int macaq_mxfp4_gemm(const uint8_t* Aq, const uint8_t* As, int64_t M, const uint8_t* Wq,
                                const uint8_t* Ws, int64_t N, int64_t K, void* y, int y_is_fp32, void* workspace,
                                size_t workspace_bytes, void* stream) {
    if (!Aq || !As || !Wq || !Ws || !y) return MACAQ_EINVAL;
    if (y_is_fp32 != 0 && y_is_fp32 != 1) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(Aq) || !aligned16(As) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) ||
        (workspace && !aligned16(workspace)))
        return MACAQ_EALIGN;
    if (workspace && workspace_bytes < gemm_workspace_bytes(M)) return MACAQ_EWORKSPACE;
    const GemmScratch ws{workspace, workspace ? workspace_bytes : 0};
    return run_mxfp4_gemm(Aq, As, M, Wq, Ws, N, K, y, y_is_fp32, ws, static_cast<cudaStream_t>(stream), false);
}

extern "C" int macaq_w4a4_linear(const uint16_t* x, int64_t M, int64_t K, const float* act_mult, const uint8_t* Wq,
                                 const uint8_t* Ws, int64_t N, uint16_t* y, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    if (!x || !act_mult || !Wq || !Ws || !y || !workspace) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(x) || !aligned16(act_mult) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) ||
        !aligned16(workspace))
        return MACAQ_EALIGN;
    if (workspace_bytes < macaq_linear_workspace_bytes(M, N, K)) return MACAQ_EWORKSPACE;
    return run_linear(x, M, K, act_mult, Wq, Ws, N, y, linear_workspace_layout(workspace, M, K), true,
                      static_cast<cudaStream_t>(stream));
}

extern "C" int macaq_mxfp4_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wq, const uint8_t* Ws,
                                  int64_t N, uint16_t* y, void* workspace, size_t workspace_bytes, void* stream) {
    if (!x || !Wq || !Ws || !y || !workspace) return MACAQ_EINVAL;
    if (int st = check_shape(M, K)) return st;
    if (int st = check_shape(N, K)) return st;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) || !aligned16(workspace))
        return MACAQ_EALIGN;
    if (workspace_bytes < macaq_linear_workspace_bytes(M, N, K)) return MACAQ_EWORKSPACE;
    return run_linear(x, M, K, nullptr, Wq, Ws, N, y, linear_workspace_layout(workspace, M, K), true,
                      static_cast<cudaStream_t>(stream));
}

extern "C" size_t macaq_grouped_workspace_bytes(const int64_t* counts, int E, int64_t N, int64_t K) {
    if (!counts || check_shape(1, K) || N < 128 || N % 128 != 0 || N > kMaxDim) return 0;
    GroupTable gt;
    int64_t mx = 0;
    if (build_group_table(counts, E, N, &gt, &mx)) return 0;
    return grouped_activation_bytes(gt.a_row[E], K);
}

extern "C" int macaq_w4a4_grouped_linear(const uint16_t* x, const int64_t* counts, int E, int64_t K,
                                         const float* act_mult, const uint8_t* Wq, const uint8_t* Ws, int64_t N,
                                         uint16_t* y, void* workspace, size_t workspace_bytes, void* stream) {
    if (!counts || !Wq || !Ws) return MACAQ_EINVAL;
    if (int st = check_shape(1, K)) return st;
    if (N < 128 || N % 128 != 0 || N > kMaxDim || static_cast<int64_t>(E) * N > kMaxDim) return MACAQ_ESHAPE;
    GroupTable gt;
    int64_t mx = 0;
    if (int st = build_group_table(counts, E, N, &gt, &mx)) return st;
    if (mx == 0) return MACAQ_OK;  // no token routed to any expert
    if (!x || !y || !workspace) return MACAQ_EINVAL;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) || !aligned16(workspace) ||
        (act_mult && !aligned16(act_mult)))
        return MACAQ_EALIGN;
    const int64_t P = gt.a_row[E];
    if (workspace_bytes < grouped_activation_bytes(P, K)) return MACAQ_EWORKSPACE;
    uint8_t* Aq = static_cast<uint8_t*>(workspace);
    uint8_t* As = Aq + round256(static_cast<size_t>(P * (K / 2)));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (int rc = launch_act_quant_grouped(x, K, act_mult, Aq, As, gt, st)) return rc;
    const GemmScratch none{nullptr, 0};
    const GroupedShape gs{gt.x_row[E - 1] + gt.rows[E - 1], gt.tile_start[E], N, nullptr};
    if (mx <= 128) {  // decode-sized experts: weights on the MMA's 128-row side, tokens as N
        return with_config(mx, [&](auto bn, auto stages, auto sw) -> int {
            if constexpr (decltype(sw)::value) {
                const GemmOperands op{Wq, Ws, Aq, As, E * N, P, K, y, N, 0};
                return launch_gemm<decltype(bn)::value, decltype(stages)::value, true, GroupTable>(op, none, st, true,
                                                                                                   gt, &gs);
            } else {
                return MACAQ_EINVAL;  // not reached: up to 128 tokens always take a swap-AB configuration
            }
        });
    }
    const GemmOperands op{Aq, As, Wq, Ws, P, E * N, K, y, N, 0};
    return launch_gemm<256, 4, false, GroupTable>(op, none, st, true, gt, &gs);
}

// Shape checks of the stacked-linears call; the total of the N[g] in *n_total.
static int check_multi(int64_t M, int64_t K, int G, const int64_t* N, int64_t* n_total) {
    if (int st = check_shape(M, K)) return st;
    if (G < 1 || G > kMaxGroups) return MACAQ_ESHAPE;
    if (static_cast<int64_t>(G) * ((M + 127) / 128 * 128) > kMaxDim) return MACAQ_ESHAPE;
    int64_t t = 0;
    for (int g = 0; g < G; ++g) {
        if (N[g] < 128 || N[g] % 128 != 0 || N[g] > kMaxDim) return MACAQ_ESHAPE;
        t += N[g];
        if (t > kMaxDim) return MACAQ_ESHAPE;
    }
    *n_total = t;
    return MACAQ_OK;
}

extern "C" size_t macaq_linear_multi_workspace_bytes(int64_t M, int G, int64_t K) {
    if (check_shape(M, K) || G < 1 || G > kMaxGroups || static_cast<int64_t>(G) * ((M + 127) / 128 * 128) > kMaxDim)
        return 0;
    return multi_workspace_layout(nullptr, M, G, K).bytes;
}

extern "C" int macaq_w4a4_linear_multi(const uint16_t* x, int64_t M, int64_t K, int G, const float* act_mult,
                                       const uint8_t* Wq, const uint8_t* Ws, const int64_t* N, uint16_t* y,
                                       void* workspace, size_t workspace_bytes, void* stream) {
    if (!x || !Wq || !Ws || !N || !y || !workspace) return MACAQ_EINVAL;
    int64_t n_total = 0;
    if (int st = check_multi(M, K, G, N, &n_total)) return st;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) || !aligned16(workspace) ||
        (act_mult && !aligned16(act_mult)))
        return MACAQ_EALIGN;
    const MultiWorkspace l = multi_workspace_layout(workspace, M, G, K);
    if (workspace_bytes < l.bytes) return MACAQ_EWORKSPACE;
    return run_linear_multi(x, M, K, G, act_mult, Wq, Ws, N, n_total, y, l, static_cast<cudaStream_t>(stream));
}

#ifdef MACAQ_TEST_HOOKS
// Fault injection (test build only): offset of the tag stream-K owners wait for.
extern "C" void macaq_test_owner_tag_offset(int64_t offset) { macaq::g_test_owner_tag_offset.store(offset); }
#endif

extern "C" size_t macaq_grouped_device_workspace_bytes(int64_t T, int E, int64_t N, int64_t K) {
    if (check_shape(T, K) || E < 1 || E > kMaxGroups || N < 128 || N % 128 != 0 || N > kMaxDim) return 0;
    if (T + 127 * static_cast<int64_t>(E) + 128 > kMaxDim) return 0;
    return device_grouped_layout(nullptr, T, E, K).bytes;
}

extern "C" int macaq_w4a4_grouped_linear_device(const uint16_t* x, int64_t T, const void* counts, int counts_bytes,
                                                int E, int64_t capacity, int64_t K, const float* act_mult,
                                                const uint8_t* Wq, const uint8_t* Ws, int64_t N, uint16_t* y,
                                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!x || !counts || !Wq || !Ws || !y || !workspace) return MACAQ_EINVAL;
    if (counts_bytes != 4 && counts_bytes != 8) return MACAQ_EINVAL;
    if (int st = check_shape(T, K)) return st;
    if (E < 1 || E > kMaxGroups) return MACAQ_ESHAPE;
    if (N < 128 || N % 128 != 0 || N > kMaxDim || static_cast<int64_t>(E) * N > kMaxDim) return MACAQ_ESHAPE;
    if (T + 127 * static_cast<int64_t>(E) + 128 > kMaxDim) return MACAQ_ESHAPE;
    if (!aligned16(x) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y) || !aligned16(workspace) ||
        (act_mult && !aligned16(act_mult)) || (reinterpret_cast<uintptr_t>(counts) % counts_bytes) != 0)
        return MACAQ_EALIGN;
    const DeviceGroupedWorkspace l = device_grouped_layout(workspace, T, E, K);
    if (workspace_bytes < l.bytes) return MACAQ_EWORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t cap = capacity < 1 || capacity > T ? T : capacity;  // rows per expert at most
    const bool swap = cap <= 128;  // every expert then fits one swap-AB tile of the narrowest N holding cap
    const int64_t rpg = device_groups_rpg(T, E, K);
    build_groups_kernel<<<1, kGroupThreads, 0, st>>>(counts, counts_bytes, E, T, cap, N, swap ? 1 : 0,
                                                     static_cast<int>(rpg), l.gt, l.rr);
    if (int rc = launch_status()) return rc;
    const DeviceGroups dg{l.gt, l.rr};
    if (int rc = launch_act_quant_grouped_device(x, T, E, K, act_mult, l.Aq, l.As, dg, st)) return rc;
    const GemmScratch none{nullptr, 0};
    const int64_t nz = E < T ? E : T;
    if (swap) {
        const GroupedShape gs{T, nz * (N / 128), N, &l.gt->tile_start[E]};
        return with_config(cap, [&](auto bn, auto stages, auto sw) -> int {
            if constexpr (decltype(sw)::value) {
                const GemmOperands op{Wq, Ws, l.Aq, l.As, E * N, l.P, K, y, N, 0};
                return launch_gemm<decltype(bn)::value, decltype(stages)::value, true, DeviceGroups>(op, none, st, true,
                                                                                                     dg, &gs);
            } else {
                return MACAQ_EINVAL;  // not reached: up to 128 tokens always take a swap-AB configuration
            }
        });
    }
    const GroupedShape gs{T, (T / 128 + nz + 1) * ((N + 255) / 256), N, &l.gt->tile_start[E]};
    const GemmOperands op{l.Aq, l.As, Wq, Ws, l.P, E * N, K, y, N, 0};
    return launch_gemm<256, 4, false, DeviceGroups>(op, none, st, true, dg, &gs);
}
