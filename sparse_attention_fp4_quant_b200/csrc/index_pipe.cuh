// index_pipe.cuh -- the TMA -> tcgen05 scoring pipeline shared by the index
// kernels (index_tc.cu: streaming Top-K per share; index_cluster.cu: one
// thread-block cluster per query with an exact radix select).
//
// Scoring as a block-scaled FP4 MMA.  A = 128 indexer-K rows (E2M1, K = 64
// channels) with their E4M3 block scales; B = the query as a block-diagonal
// 16 x 64 operand: column n = 4 h + b holds head h's codes in block b only, so
// accumulator column n of row t is exactly one block's
//   T[h][b] = (sum over 16 channels of q k) * sq[h][b] * sk[b]
// (at most 20 significant bits: exact in fp32 whatever the MMA's summation
// order).  The epilogue then sums the blocks and heads in the fixed order
// ((T0 + T1) + T2) + T3 and ((w0 r0 + w1 r1) + w2 r2) + w3 r3 on CUDA cores
// (score_of below), which reproduces the defined score bit for bit.
//
// Warp 0 streams 128-row tiles with TMA (32-byte swizzle) and brings the scale
// bytes into the TMEM-copy layout: 4-byte cp.async per row (producer), or, with
// the rows of each tile permuted so that layout is their stored order, one
// bulk copy per stage (producer_perm); warp 1 owns TMEM, copies the scales to
// TMEM and issues the MMAs; the epilogue warps read the accumulators.  Every mbarrier wait is bounded; a timeout sets the
// workspace status word and the CTA winds down.
#pragma once
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {
namespace pipe {

constexpr int kTile = 128;       // rows per MMA (M)
constexpr int kTPS = 4;          // tiles per pipeline stage
constexpr int kAcc = 2;          // accumulator stages (each with its own scale-factor slot)
constexpr uint32_t kPipeCols = 256;   // TMEM columns of the pipeline (a power of two)
constexpr uint32_t kColAcc = 0, kColSfa = kAcc * kTPS * 16, kColSfb = kColSfa + kAcc * kTPS * 4;
static_assert(kColSfb + 4 <= kPipeCols, "TMEM columns");
constexpr uint32_t kIdesc = tc::idesc_mxf4nvf4(128, 16);
constexpr int kPoolPerTile = kTile / kBlk;   // 16 pool blocks of 8 rows per tile

// Shared-memory part of the pipeline with ST ring stages.  Must start on a
// 1024-byte boundary.
template <int ST>
struct Pipe {
    static constexpr int kStages = ST;
    uint8_t A[ST][kTPS][kTile * 32];   // K-major, 32-byte swizzle (written by TMA)
    uint8_t SF[ST][kTPS][512];         // scale bytes in the 32 x (4 x 4 B) TMEM-copy layout
    uint8_t Bq[16 * 32];               // block-diagonal query, no swizzle, K-major
    uint8_t SFB[512];                  // its scales, TMEM-copy layout
    uint64_t full[ST], empty[ST], accfull[kAcc], accempty[kAcc], done;
    uint32_t tmem_base;
    int abort_flag;
};

template <class P>
__device__ __forceinline__ void raise_abort(P& s, int32_t* status) {
    *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
    if (status) atomicExch(status, 1);
}

template <class P>
__device__ __forceinline__ bool aborted(const P& s) { return *reinterpret_cast<const volatile int*>(&s.abort_flag) != 0; }

// One thread: barrier init.  `full_arrivals` = arrivals that fill a stage (the
// expect_tx arrive, plus 32 cp.async arrivals when the scales come by cp.async);
// `epi_arrivals` = arrivals that free an accumulator stage.
template <class P>
__device__ __forceinline__ void init_barriers(P& s, uint32_t full_arrivals, uint32_t epi_arrivals) {
    for (int i = 0; i < P::kStages; ++i) {
        tc::mbar_init(&s.full[i], full_arrivals);
        tc::mbar_init(&s.empty[i], 1);       // MMA commit
    }
    for (int i = 0; i < kAcc; ++i) {
        tc::mbar_init(&s.accfull[i], 1);     // MMA commit
        tc::mbar_init(&s.accempty[i], epi_arrivals);
    }
    tc::mbar_init(&s.done, 1);
    s.abort_flag = 0;
    tc::fence_mbar_init();
}

// Warp 1: allocate `cols` TMEM columns (the pipeline uses the first kPipeCols)
// and lay out the block-diagonal query operand.  Row n = 4h + b keeps head h's
// 8 code bytes of block b; all else zero.
template <class P>
__device__ __forceinline__ void setup_query(P& s, const uint8_t* q, const uint8_t* qs, int lane, uint32_t cols) {
    tc::tmem_alloc(&s.tmem_base, cols);
    for (int i = lane; i < 16 * 32; i += 32) s.Bq[i] = 0;
    for (int i = lane; i < 512; i += 32) s.SFB[i] = 0;
    __syncwarp();
    if (lane < 16) {
        const int n = lane, h = n >> 2, blk = n & 3;
        const int kc = blk >> 1, off = 8 * (blk & 1);
        uint8_t* row = s.Bq + (n >> 3) * 256 + kc * 128 + (n & 7) * 16 + off;
        const uint8_t* src = q + 32 * h + 8 * blk;
#pragma unroll
        for (int j = 0; j < 8; ++j) row[j] = src[j];
#pragma unroll
        for (int j = 0; j < 4; ++j) s.SFB[16 * n + j] = qs[4 * h + j];
    }
    tc::fence_proxy_async_smem();
}

// Warp 0.  MODE 0: rows [lo, hi) of the query's batch row (tiles of 128);
// MODE 1: the pool slots [lo, hi), 16 blocks of 8 rows per tile.
template <int MODE, class P>
__device__ __forceinline__ void producer(P& s, const CUtensorMap* tmap, const uint8_t* iks, int64_t row_base,
                                         int lo, int hi, int ntiles, int nstages, const int32_t* pool, int nvis,
                                         int32_t* status, int lane) {
    constexpr int kStages = P::kStages;
    int issued = 0;
    for (int t = 0; t < nstages; ++t) {
        const int slot = t % kStages;
        const uint32_t ph = (uint32_t)(t / kStages) & 1u;
        int ok = 1;
        if (lane == 0) ok = tc::mbar_wait(&s.empty[slot], ph ^ 1u);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (lane == 0 && !ok) raise_abort(s, status);
        if (__any_sync(0xFFFFFFFFu, !ok || aborted(s))) break;   // warp-uniform
        uint32_t bytes = 0;
        if (MODE == 0) {
            for (int i = 0; i < kTPS; ++i)
                if (t * kTPS + i < ntiles) bytes += kTile * 32;
        } else {
            for (int i = 0; i < kTPS; ++i) {
                const int g = t * kTPS + i;
                if (g >= ntiles) break;
                for (int j = 0; j < kPoolPerTile; ++j) {
                    const int sl = lo + g * kPoolPerTile + j;
                    if (sl < hi) {
                        const int blk = __ldg(pool + sl);
                        if (blk >= 0 && (int64_t)blk * kBlk < nvis) bytes += kBlk * 32;
                    }
                }
            }
        }
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&s.full[slot], bytes);
            for (int i = 0; i < kTPS; ++i) {
                const int g = t * kTPS + i;
                if (g >= ntiles) break;
                if (MODE == 0) {
                    tc::tma_load_2d(s.A[slot][i], tmap, 0, (int)(row_base + lo + g * kTile), &s.full[slot]);
                } else {
                    for (int j = 0; j < kPoolPerTile; ++j) {
                        const int sl = lo + g * kPoolPerTile + j;
                        if (sl >= hi) break;
                        const int blk = __ldg(pool + sl);
                        if (blk >= 0 && (int64_t)blk * kBlk < nvis)
                            tc::tma_load_2d(s.A[slot][i] + 256 * j, tmap, 0, (int)(row_base + (int64_t)blk * kBlk),
                                            &s.full[slot]);
                    }
                }
            }
        }
        // scale bytes: row m = lane + 32 j goes to byte 16 * lane + 4 * j
        for (int i = 0; i < kTPS; ++i) {
            const int g = t * kTPS + i;
            if (g >= ntiles) break;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int m = lane + 32 * j;
                int64_t e = -1;
                if (MODE == 0) {
                    const int ee = lo + g * kTile + m;
                    if (ee < hi) e = ee;
                } else {
                    const int sl = lo + g * kPoolPerTile + (m >> 3);
                    if (sl < hi) {
                        const int blk = __ldg(pool + sl);
                        const int64_t ee = (int64_t)blk * kBlk + (m & 7);
                        if (blk >= 0 && ee < nvis) e = ee;
                    }
                }
                if (e >= 0) tc::cp_async_4(&s.SF[slot][i][16 * lane + 4 * j], iks + (row_base + e) * 4);
            }
        }
        tc::cp_async_arrive_noinc(&s.full[slot]);
        ++issued;
    }
    // never leave copies in flight: wait (bounded) for the stages still pending
    if (lane == 0) {
        for (int t = max(0, issued - kStages); t < issued; ++t)
            if (!tc::mbar_wait(&s.full[t % kStages], (uint32_t)(t / kStages) & 1u)) raise_abort(s, status);
    }
}

// Warp 0, dense rows [lo, hi) with the rows of each 128-row tile permuted:
// TMEM row m of a tile holds entry 4 (m % 32) + m / 32 of it.  Under that
// order the scale bytes the MMA expects (row m at byte 16 (m % 32) + 4 (m / 32))
// are the tile's scales in their stored order, so a stage takes one TMA box per
// tile (3-D map: 32 bytes x 32 groups of 4 rows x 4 rows) and one bulk copy of
// its contiguous scale bytes.  Needs lo, the batch row base and the cache
// capacity to be multiples of 4 and 16-byte aligned scales.
template <class P>
__device__ __forceinline__ void producer_perm(P& s, const CUtensorMap* tmap3, const uint8_t* iks, int64_t row_base,
                                              int lo, int hi, int ntiles, int nstages, int32_t* status, int lane) {
    constexpr int kStages = P::kStages;
    int issued = 0;
    if (lane == 0) {
        for (int t = 0; t < nstages; ++t) {
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            if (!tc::mbar_wait(&s.empty[slot], ph ^ 1u)) {
                raise_abort(s, status);
                break;
            }
            if (aborted(s)) break;
            const int r0 = lo + t * kTPS * kTile;
            const int nrows = min(kTPS * kTile, hi - r0);
            const int ntl = (nrows + kTile - 1) / kTile;
            const uint32_t sc_bytes = (uint32_t)((nrows + 3) & ~3) * 4u;
            tc::mbar_arrive_expect_tx(&s.full[slot], (uint32_t)ntl * kTile * 32u + sc_bytes);
            for (int i = 0; i < ntl; ++i)
                tc::tma_load_3d(s.A[slot][i], tmap3, 0, (int)((row_base + r0 + i * kTile) >> 2), 0, &s.full[slot]);
            tc::bulk_load(s.SF[slot], iks + (row_base + r0) * 4, sc_bytes, &s.full[slot]);
            ++issued;
        }
        // never leave copies in flight: wait (bounded) for the stages still pending
        for (int t = max(0, issued - kStages); t < issued; ++t)
            if (!tc::mbar_wait(&s.full[t % kStages], (uint32_t)(t / kStages) & 1u)) raise_abort(s, status);
    }
    (void)ntiles;
    __syncwarp();
}

// Warp 1 (lane 0 issues).  Returns once every MMA it issued has completed.
template <class P>
__device__ __forceinline__ void mma_issuer(P& s, int ntiles, int nstages, int32_t* status, int lane) {
    constexpr int kStages = P::kStages;
    const uint32_t tbase = s.tmem_base;
    if (lane == 0) {
        tc::tc_fence_after();
        const uint32_t sa_sfb = tc::smem_u32(s.SFB);
        tc::tmem_cp_32x128_x4(tbase + kColSfb, tc::smem_desc(sa_sfb, 16, 128, tc::kLayoutNone));
        const uint64_t bdesc = tc::smem_desc(tc::smem_u32(s.Bq), 128, 256, tc::kLayoutNone);
        for (int t = 0; t < nstages; ++t) {
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            if (!tc::mbar_wait(&s.full[slot], ph) || !tc::mbar_wait(&s.accempty[a], aph ^ 1u)) {
                raise_abort(s, status);
                break;
            }
            if (aborted(s)) break;
            tc::tc_fence_after();
            tc::fence_proxy_async_smem();   // scale bytes came through cp.async (generic proxy)
            for (int i = 0; i < kTPS; ++i) {
                if (t * kTPS + i >= ntiles) break;
                const uint32_t sfa = tbase + kColSfa + (uint32_t)(a * kTPS + i) * 4;   // free once stage t - kAcc is read
                tc::tmem_cp_32x128_x4(sfa, tc::smem_desc(tc::smem_u32(s.SF[slot][i]), 16, 128, tc::kLayoutNone));
                const uint64_t adesc = tc::smem_desc(tc::smem_u32(s.A[slot][i]), 16, 256, tc::kLayoutSw32);
                tc::mma_mxf4nvf4(tbase + kColAcc + (uint32_t)(a * kTPS + i) * 16, adesc, bdesc, kIdesc, 0u, sfa,
                                 tbase + kColSfb);
            }
            tc::tc_commit(&s.empty[slot]);
            tc::tc_commit(&s.accfull[a]);
        }
        tc::tc_commit(&s.done);
        if (!tc::mbar_wait(&s.done, 0)) raise_abort(s, status);
    }
    __syncwarp();
}

// The defined score of one row from its 16 exact block products
// (column 4h + b = head h, block b).
__device__ __forceinline__ float score_of(const uint32_t (&v)[16], float w0, float w1, float w2, float w3) {
    const float* T = reinterpret_cast<const float*>(v);
    float r[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float d = __fadd_rn(__fadd_rn(__fadd_rn(T[4 * h], T[4 * h + 1]), T[4 * h + 2]), T[4 * h + 3]);
        r[h] = d > 0.0f ? d : 0.0f;
    }
    return __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(w0, r[0]), __fmul_rn(w1, r[1])), __fmul_rn(w2, r[2])),
                     __fmul_rn(w3, r[3]));
}

// Host: the indexer-K tensor map (rows of 32 bytes, box of `box_rows` rows, 32-byte swizzle).
bool encode_ik_map(CUtensorMap* map, const uint8_t* ik, int64_t rows, int box_rows);
// Host: the permuted-tile map of producer_perm (rows a multiple of 4).
bool encode_ik_map_perm(CUtensorMap* map, const uint8_t* ik, int64_t rows);

}  // namespace pipe
}  // namespace csa2
