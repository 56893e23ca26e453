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
//   warp 1     allocates tensor memory; one lane issues, per stage, tcgen05.cp of the
//              scale atoms into TMEM and four tcgen05.mma (K = 64 each), then commits the
//              stage back to the producer and, per tile, the accumulator to the epilogue.
//   warps 2-9  epilogue: two warps per TMEM sub-partition (warp w reads lanes of
//              sub-partition w % 4, one half of the tile's columns each) copy the fp32
//              accumulator into registers, hand the TMEM back to the MMA warp at once, then
//              convert and store y, so the next tile's mainloop overlaps the stores.
//   Scale factors are double-buffered in TMEM (alternating per k-tile), so the copy for
//   k-tile t+1 never writes columns the MMAs of k-tile t still read.  Accumulators are
//   double-buffered too when BN <= 128.  All waits are bounded (see sm100.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace macaq {

int launch_act_transform_quant(const uint16_t* x, int64_t M, int64_t K, const float* act_mult,
                               uint8_t* Aq, uint8_t* As, cudaStream_t stream, uint32_t* clear, int clear_words);

constexpr int kBM = 128;           // MMA M
constexpr int kStageK = 256;       // K elements per stage
constexpr int kStageKBytes = 128;  // code bytes per row per stage
constexpr int kGemmThreads = 320;  // producer, MMA, 8 epilogue warps
constexpr int kEpiThreads = 256;
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
    static constexpr int kSFBase = kNumAcc * kAccStride;           // two scale buffers follow
    static constexpr int kColsUsed = kSFBase + 2 * kSFBufCols;
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
    static_assert(kColsUsed <= 512, "tensor memory budget");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(kStageBytes % 1024 == 0, "stage alignment for the 128-byte swizzle");
};

struct GemmParams {
    const uint8_t* sf_p;  // scales of P, MMA tile layout
    const uint8_t* sf_q;  // scales of Q
    int64_t p_rows, q_rows, K, kbp;
    void* y;
    int64_t ldy;          // elements per row of y
    int y_fp32;
    int num_p_tiles, num_q_tiles, num_k_tiles, q_row_blocks;
    int dp_tiles;         // tiles scheduled data-parallel (blockIdx.x + i * gridDim.x)
    int64_t sk_units;     // K steps of the remaining tiles, split evenly over the CTAs
    float* partials;      // stream-K fp32 partial accumulators, one 128 x BN slot per CTA
    uint32_t* flags;      // stream-K partial-ready counters, one per CTA, zero at launch
    int tma_store;        // bf16 output written by TMA from shared memory (non-swap, N % 8 == 0)
};

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<uint32_t*>(&v);
}

// Store CH accumulator columns [qc, qc+CH) of P-row `prow`.
template <int CH, bool SWAP>
__device__ __forceinline__ void store_chunk(const GemmParams& prm, int64_t prow, int64_t qc,
                                            const uint32_t* r) {
    if (prow >= prm.p_rows) return;
    if constexpr (!SWAP) {
        const int64_t base = prow * prm.ldy + qc;
        const bool full = qc + CH <= prm.q_rows;
        if (prm.y_fp32) {
            float* y = static_cast<float*>(prm.y) + base;
            if (full && (prm.ldy % 4) == 0) {
#pragma unroll
                for (int j = 0; j < CH; j += 4)
                    *reinterpret_cast<uint4*>(y + j) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < CH; ++j)
                    if (qc + j < prm.q_rows) y[j] = __uint_as_float(r[j]);
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
                    if (qc + j < prm.q_rows) y[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
            }
        }
    } else {
        // accumulator row = output column (feature), accumulator column = output row (token)
        if (prm.y_fp32) {
            float* y = static_cast<float*>(prm.y);
#pragma unroll
            for (int j = 0; j < CH; ++j)
                if (qc + j < prm.q_rows) y[(qc + j) * prm.ldy + prow] = __uint_as_float(r[j]);
        } else {
            __nv_bfloat16* y = static_cast<__nv_bfloat16*>(prm.y);
#pragma unroll
            for (int j = 0; j < CH; ++j)
                if (qc + j < prm.q_rows) y[(qc + j) * prm.ldy + prow] = __float2bfloat16_rn(__uint_as_float(r[j]));
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
    int dp_next;
    int64_t pos, hi;

    __device__ __forceinline__ explicit WorkIter(const GemmParams& p) {
        dp_next = blockIdx.x;
        const int64_t G = gridDim.x;
        pos = p.sk_units * blockIdx.x / G;
        hi = p.sk_units * (blockIdx.x + 1) / G;
    }

    __device__ __forceinline__ bool next(const GemmParams& p, Work& w) {
        const int KT = p.num_k_tiles;
        if (dp_next < p.dp_tiles) {
            w.tile = dp_next;
            w.k0 = 0;
            w.k1 = KT;
            w.kind = kFull;
            w.c_last = 0;
            dp_next += gridDim.x;
            return true;
        }
        if (pos >= hi) return false;
        const int64_t ts = pos / KT;
        const int64_t t0 = ts * KT;
        const int64_t end = hi < t0 + KT ? hi : t0 + KT;
        w.tile = p.dp_tiles + static_cast<int>(ts);
        w.k0 = static_cast<int>(pos - t0);
        w.k1 = static_cast<int>(end - t0);
        if (w.k0 == 0 && w.k1 == KT) {
            w.kind = kFull;
        } else if (w.k0 == 0) {
            w.kind = kOwner;
            // last CTA whose range holds a unit of this tile: max c with U c / G <= t0 + KT - 1
            const int64_t U = p.sk_units, G = gridDim.x;
            w.c_last = static_cast<int>(((t0 + KT) * G + U - 1) / U - 1);
        } else {
            w.kind = kPartial;
        }
        pos = end;
        return true;
    }
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <int BN, int STAGES, bool SWAP>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mxf4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams prm) {
    using Cfg = TileCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* staging = smem + STAGES * Cfg::kStageBytes;  // per epilogue warp: 32 x 32 bf16 (non-swap)
    uint64_t* full = reinterpret_cast<uint64_t*>(staging + (SWAP ? 0 : kStagingBytes));
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
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
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    int abort = 0;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            griddep_wait();  // operands may come from the kernel launched just before
            int stage = 0;
            uint32_t phase = 0;
            WorkIter it(prm);
            Work w;
            while (!abort && it.next(prm, w)) {
                const int pt = w.tile % prm.num_p_tiles;
                const int qt = w.tile / prm.num_p_tiles;
                const uint8_t* sfp = prm.sf_p + static_cast<int64_t>(pt) * (prm.kbp / 4) * 512;
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, &abort)) break;
                    uint8_t* sb = smem + stage * Cfg::kStageBytes;
                    mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
                    tma_load_2d(sb, &tmap_p, kt * kStageKBytes, pt * kBM, &full[stage]);
                    tma_load_2d(sb + Cfg::kPBytes, &tmap_q, kt * kStageKBytes, qt * BN, &full[stage]);
                    bulk_load(sb + Cfg::kPBytes + Cfg::kQBytes, sfp + kt * 1024, 1024, &full[stage]);
#pragma unroll
                    for (int i = 0; i < Cfg::kQBlocks; ++i) {
                        int qb = (qt * BN) / 128 + i;
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
            uint32_t sfbuf = 0;
            WorkIter it(prm);
            Work w;
            while (!abort && it.next(prm, w)) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, &abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * Cfg::kAccStride;
                for (int kt = w.k0; kt < w.k1; ++kt) {
                    if (!mbar_wait(&full[stage], phase, &abort)) break;
                    tc_fence_after();
                    const uint32_t sp = smem_u32(smem + stage * Cfg::kStageBytes);
                    const uint32_t sq = sp + Cfg::kPBytes;
                    const uint32_t ssfp = sq + Cfg::kQBytes;
                    const uint32_t ssfq = ssfp + Cfg::kSFPBytes;
                    const uint32_t tsfp = tmem_base + Cfg::kSFBase + sfbuf * Cfg::kSFBufCols;
                    const uint32_t tsfq = tsfp + 8;
                    sfbuf ^= 1u;
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        tc_cp_sf(tsfp + 4 * g, desc_sf(ssfp + 512 * g));
#pragma unroll
                        for (int i = 0; i < Cfg::kQBlocks; ++i)
                            tc_cp_sf(tsfq + Cfg::kSFQColsPerGroup * g + 4 * i, desc_sf(ssfq + 1024 * i + 512 * g));
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t g = j >> 1;
                        const uint32_t id = (j & 1) * 2;  // byte of the scale word: blocks 2j%4, 2j%4+1
                        const uint32_t sfa = (tsfp + 4 * g) | (id << 30);
                        const uint32_t sfb = (tsfq + Cfg::kSFQColsPerGroup * g) | (id << 30);
                        tc_mma_mxf4(d_tmem, desc_sw128(sp + 32 * j), desc_sw128(sq + 32 * j),
                                    idesc | (id << 29) | (id << 4), sfa, sfb, (kt != w.k0 || j != 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);  // frees the stage once these MMAs have read it
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
    } else {
        // ------------------------------------------------------------------ epilogue
        constexpr int kHalf = BN / 2;            // columns per epilogue warp
        constexpr int kChunk = kHalf >= 32 ? 32 : kHalf;
        const int sub = warp & 3;                // TMEM sub-partition this warp may read
        const int half = (warp - 2) >> 2;        // which half of the tile's columns
        const int etid = threadIdx.x - 64;       // 0..255 among the epilogue threads
        int acc = 0;
        uint32_t acc_phase = 0;
        WorkIter it(prm);
        Work w;
        if (prm.sk_units > 0) griddep_wait();  // the flags were cleared by the kernel launched before
        while (!abort && it.next(prm, w)) {
            const int pt = w.tile % prm.num_p_tiles;
            const int qt = w.tile / prm.num_p_tiles;
            if (!mbar_wait(&acc_full[acc], acc_phase, &abort)) break;
            tc_fence_after();
            const int64_t prow = static_cast<int64_t>(pt) * kBM + sub * 32 + lane;
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
            if (w.kind == kPartial) {
                // fp32 partial to this CTA's slot, [chunk of 4 columns][epilogue thread]; the
                // slot's counter reaches kEpiThreads once every thread's part is visible
                float4* slot = reinterpret_cast<float4*>(prm.partials + static_cast<int64_t>(blockIdx.x) * (kBM * BN));
#pragma unroll
                for (int j = 0; j < kHalf / 4; ++j)
                    __stcg(slot + j * kEpiThreads + etid,
                           make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                       __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
                __threadfence();
                atomicAdd(prm.flags + blockIdx.x, 1u);
                continue;
            }
            if (w.kind == kOwner) {
                const int64_t U = prm.sk_units, G = gridDim.x;
                for (int c = blockIdx.x + 1; c <= w.c_last; ++c) {
                    if (U * c / G == U * (c + 1) / G) continue;  // empty range: no partial
                    if (!abort) {
                        const long long t0 = clock64();
                        while (ld_acquire(prm.flags + c) < static_cast<uint32_t>(kEpiThreads)) {
                            if (clock64() - t0 > kWaitLimitCycles) {
                                atomicExch(&g_device_status, MACAQ_ETIMEOUT);
                                abort = 1;
                                break;
                            }
                        }
                    }
                    const float4* slot = reinterpret_cast<const float4*>(prm.partials + static_cast<int64_t>(c) * (kBM * BN));
#pragma unroll
                    for (int j = 0; j < kHalf / 4; ++j) {
                        const float4 q = __ldcg(slot + j * kEpiThreads + etid);
                        v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + q.x);
                        v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + q.y);
                        v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + q.z);
                        v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + q.w);
                    }
                }
            }
            const int64_t q0 = static_cast<int64_t>(qt) * BN + half * kHalf;
            if constexpr (!SWAP && kHalf % 32 == 0) {
                if (prm.tma_store) {
                    // bf16 tile through this warp's 2 KB staging buffer (32 rows x 64 B, 64-byte
                    // swizzle: conflict-free 16-byte writes) and a TMA store per 32 columns;
                    // the store clips rows and columns past the matrix edge.
                    uint8_t* stg = staging + (warp - 2) * 2048;
#pragma unroll
                    for (int c = 0; c < kHalf; c += 32) {
                        if (lane == 0) bulk_wait_group_read<0>();  // previous store has read the buffer
                        __syncwarp();
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint32_t* r = v + c + 8 * q4;
                            *reinterpret_cast<uint4*>(stg + lane * 64 + 16 * (q4 ^ ((lane >> 1) & 3))) =
                                make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                                           pack_bf16x2(r[6], r[7]));
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmap_y, stg, static_cast<int32_t>(q0 + c), pt * kBM + sub * 32);
                            bulk_commit_group();
                        }
                    }
                    continue;
                }
            }
#pragma unroll
            for (int c = 0; c < kHalf; c += kChunk) store_chunk<kChunk, SWAP>(prm, prow, q0 + c, v + c);
        }
        if (lane == 0) bulk_wait_group<0>();  // output stores complete before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

// --------------------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

template <int BN, int STAGES, bool SWAP>
static int smem_bytes() {
    return STAGES * TileCfg<BN>::kStageBytes + (SWAP ? 0 : kStagingBytes) + (2 * STAGES + 4) * 8 + 16 + 1024;
}

// Tensor map of the bf16 output [rows][cols]: 32 x 32 boxes, 64-byte swizzle.
static bool make_out_map(CUtensorMap* map, void* y, int64_t rows, int64_t cols) {
    auto encode = tensor_map_encoder();
    if (!encode) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// CTAs of the persistent grid: SMs x resident CTAs per SM (shared memory and TMEM permitting).
template <int BN, int STAGES, bool SWAP>
static int grid_ctas() {
    auto kernel = mxf4_gemm_kernel<BN, STAGES, SWAP>;
    const int smem = smem_bytes<BN, STAGES, SWAP>();
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1;
    // all of the unified L1/shared storage as shared memory, so small configurations fit twice per SM
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return -1;
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kGemmThreads, smem) != cudaSuccess || occ < 1)
        occ = 1;
    if (occ * TileCfg<BN>::kTmemCols > 512) occ = 512 / TileCfg<BN>::kTmemCols;
    return sm_count() * occ;  // occ is 1: the runtime keeps tensor-memory kernels at one CTA per SM
}

// Stream-K scratch of one launch: a flag per CTA (rounded to 256 B) and an fp32 partial
// accumulator slot (128 x BN) per CTA.
template <int BN>
static size_t streamk_bytes(int ctas) {
    return static_cast<size_t>(((ctas * 4 + 255) / 256) * 256) + static_cast<size_t>(ctas) * kBM * BN * 4;
}

struct GemmOperands {
    const uint8_t *pq, *ps, *qq, *qs;
    int64_t p_rows, q_rows, K;
    void* y;
    int64_t ldy;
    int y_fp32;
};

// Scratch of the stream-K schedule and where its flags must be cleared before the GEMM.
struct GemmScratch {
    void* ptr;            // nullptr: data-parallel schedule only
    size_t bytes;
    bool clear_flags;     // clear the flags here (false: an earlier kernel on the stream did)
};

template <int BN, int STAGES, bool SWAP>
static int launch_gemm(const GemmOperands& op, const GemmScratch& ws, cudaStream_t stream, bool pdl) {
    using Cfg = TileCfg<BN>;
    CUtensorMap mp, mq;
    if (!make_codes_map(&mp, op.pq, op.p_rows, op.K, kBM) || !make_codes_map(&mq, op.qq, op.q_rows, op.K, BN))
        return MACAQ_ECUDA;
    GemmParams prm;
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
    prm.q_row_blocks = static_cast<int>((op.q_rows + 127) / 128);

    const int ctas = grid_ctas<BN, STAGES, SWAP>();
    if (ctas < 1) return MACAQ_ECUDA;
    CUtensorMap my;
    prm.tma_store = (!SWAP && !op.y_fp32 && op.ldy % 8 == 0) ? 1 : 0;
    if (prm.tma_store && !make_out_map(&my, op.y, op.p_rows, op.q_rows)) return MACAQ_ECUDA;
    if (!prm.tma_store) my = mq;  // unused placeholder
    const int64_t tiles = static_cast<int64_t>(prm.num_p_tiles) * prm.num_q_tiles;
    int64_t grid = ctas;
    // Stream-K only with scratch for it, and only where it pays: the data-parallel schedule
    // runs ceil(tiles / ctas) rounds, stream-K about tiles / ctas rounds plus a fix-up that
    // costs roughly streamk_cost_steps<BN>() K steps on the critical path (one partial-sum
    // round trip through L2).
    const int64_t rounds_dp = (tiles + ctas - 1) / ctas;
    const int64_t saved_steps = (rounds_dp * ctas - tiles) * prm.num_k_tiles / ctas;
    const bool streamk = ws.ptr != nullptr && ws.bytes >= streamk_bytes<BN>(ctas) && tiles % ctas != 0 &&
                         prm.num_k_tiles > 1 && saved_steps >= streamk_cost_steps<BN>();
    if (streamk) {
        const int64_t full_waves = tiles / ctas;
        prm.dp_tiles = static_cast<int>((full_waves > 0 ? full_waves - 1 : 0) * ctas);
        prm.sk_units = (tiles - prm.dp_tiles) * static_cast<int64_t>(prm.num_k_tiles);
        if (grid > prm.sk_units) grid = prm.sk_units;  // every CTA gets at least one K step
        prm.flags = static_cast<uint32_t*>(ws.ptr);
        prm.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws.ptr) + ((ctas * 4 + 255) / 256) * 256);
        if (ws.clear_flags && cudaMemsetAsync(prm.flags, 0, sizeof(uint32_t) * ctas, stream) != cudaSuccess)
            return MACAQ_ECUDA;
    } else {
        if (grid > tiles) grid = tiles;
        prm.dp_tiles = static_cast<int>(tiles);
        prm.sk_units = 0;
        prm.flags = nullptr;
        prm.partials = nullptr;
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
    if (cudaLaunchKernelEx(&cfg, mxf4_gemm_kernel<BN, STAGES, SWAP>, mp, mq, my, prm) != cudaSuccess)
        return MACAQ_ECUDA;
    return launch_status();
}

// Kernel configuration for M rows of activations: swap-AB with the narrowest N that holds
// the tokens for M <= 128, 128 x 256 tiles above.  `f` is called with the configuration.
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

int gemm_ctas(int64_t M) {
    return with_config(M, [](auto bn, auto st, auto sw) -> int {
        return grid_ctas<decltype(bn)::value, decltype(st)::value, decltype(sw)::value>();
    });
}

size_t gemm_workspace_bytes(int64_t M) {
    return with_config(M, [](auto bn, auto st, auto sw) -> size_t {
        const int ctas = grid_ctas<decltype(bn)::value, decltype(st)::value, decltype(sw)::value>();
        return ctas < 1 ? 0 : streamk_bytes<decltype(bn)::value>(ctas);
    });
}

// y[M][N] = dec(A) dec(W)^T.  Small M runs swap-AB (weights on the MMA M side).
int run_mxfp4_gemm(const uint8_t* Aq, const uint8_t* As, int64_t M, const uint8_t* Wq, const uint8_t* Ws,
                   int64_t N, int64_t K, void* y, int y_fp32, const GemmScratch& ws, cudaStream_t stream, bool pdl) {
    return with_config(M, [&](auto bn, auto st, auto sw) -> int {
        constexpr bool kSwap = decltype(sw)::value;
        const GemmOperands op = kSwap ? GemmOperands{Wq, Ws, Aq, As, N, M, K, y, N, y_fp32}
                                      : GemmOperands{Aq, As, Wq, Ws, M, N, K, y, N, y_fp32};
        return launch_gemm<decltype(bn)::value, decltype(st)::value, kSwap>(op, ws, stream, pdl);
    });
}

// Layout of the fused linear's workspace: activation codes, their scales, then the GEMM's
// stream-K scratch (flags first).
struct LinearWorkspace {
    uint8_t *Aq, *As, *gemm;
    size_t gemm_bytes;
};

LinearWorkspace linear_workspace_layout(void* base, int64_t M, int64_t K) {
    LinearWorkspace l;
    l.Aq = static_cast<uint8_t*>(base);
    l.As = l.Aq + ((M * (K / 2) + 255) / 256) * 256;
    l.gemm = l.As + ((scale_bytes(M, K) + 255) / 256) * 256;
    l.gemm_bytes = gemm_workspace_bytes(M);
    return l;
}

size_t linear_activation_bytes(int64_t M, int64_t K) {
    return static_cast<size_t>(((M * (K / 2) + 255) / 256) * 256 + ((scale_bytes(M, K) + 255) / 256) * 256);
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
    const GemmScratch ws{workspace, workspace ? workspace_bytes : 0, true};
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const LinearWorkspace l = linear_workspace_layout(workspace, M, K);
    // the quantiser also clears the stream-K flags, so the GEMM needs no extra launch
    if (int rc = launch_act_transform_quant(x, M, K, act_mult, l.Aq, l.As, st, reinterpret_cast<uint32_t*>(l.gemm),
                                            gemm_ctas(M)))
        return rc;
    const GemmScratch ws{l.gemm, l.gemm_bytes, false};
    return run_mxfp4_gemm(l.Aq, l.As, M, Wq, Ws, N, K, y, 0, ws, st, true);
}
