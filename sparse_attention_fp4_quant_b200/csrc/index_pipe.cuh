// index_pipe.cuh -- the bulk-copy -> tcgen05 scoring pipeline shared by the
// index kernels (index_tc.cu: streaming Top-K per share; index_cluster.cu: one
// thread-block cluster per query with an exact radix select).
//
// Scoring as a block-scaled FP4 MMA.  A = 128 indexer-K rows (E2M1, K = 64
// channels) with unit block scales; B = the query as a block-diagonal 16 x 64
// operand with its own E4M3 block scales: column n = 4 b + h holds head h's
// codes in block b only, so accumulator column n of row t is exactly
//   (sum over 16 channels of q k) * sq[h][b]
// (at most 16 significant bits: exact in fp32 whatever the MMA's summation
// order).  The epilogue multiplies by the key's block scale sk[b] (exact: at
// most 20 significant bits), which gives the block product T[h][b], then sums
// the blocks and heads in the fixed order ((T0 + T1) + T2) + T3 and
// ((w0 r0 + w1 r1) + w2 r2) + w3 r3 on CUDA cores (score_of below): the
// defined score bit for bit.  Applying sk on CUDA cores instead of through the
// MMA's scale operand saves a TMEM scale copy per tile, which serialised with
// the MMA that read it.
//
// The indexer-K cache stores each 128-entry tile as the MMA's shared-memory
// operand image (K-major core matrices, no swizzle) and the scales row-major
// (common.cuh), so warp 0 moves whole tiles with contiguous bulk copies
// (producer_dense) or gathers 8-entry pool blocks, 256 + 32 bytes each
// (producer_pool); warp 1 owns TMEM and issues the MMAs; the epilogue warps
// read the accumulators and the stage's scales.  A ring slot is free once its
// MMAs completed and every epilogue warp read its scales.  Every mbarrier wait
// is bounded; a timeout sets the workspace status word and the CTA winds down.
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {
namespace pipe {

constexpr int kTile = 128;       // rows per MMA (M)
constexpr int kTPS = 4;          // tiles per pipeline stage
constexpr int kAcc = 2;          // accumulator stages (each with its own scale-factor slot)
constexpr int kEpiWarps = 8;     // epilogue warps (each releases a ring slot once)
constexpr uint32_t kPipeCols = 256;   // TMEM columns of the pipeline (a power of two)
constexpr uint32_t kColAcc = 0, kColSfa = kAcc * kTPS * 16, kColSfb = kColSfa + 4;
static_assert(kColSfb + 4 <= kPipeCols, "TMEM columns");
constexpr uint32_t kIdesc = tc::idesc_mxf4nvf4(128, 16);
constexpr int kPoolPerTile = kTile / kBlk;   // 16 pool blocks of 8 rows per tile

// Shared-memory part of the pipeline with ST ring stages.  Must start on a
// 1024-byte boundary.
template <int ST>
struct Pipe {
    static constexpr int kStages = ST;
    uint8_t A[ST][kTPS][kTile * 32];   // K-major core matrices, no swizzle: the cache's tile image
    uint8_t SF[ST][kTPS][kTile * 4];   // the tiles' scale bytes, row-major (read by the epilogue)
    uint8_t Bq[16 * 32];               // block-diagonal query, no swizzle, K-major
    uint8_t SFB[512];                  // its scales, in the 32 x (4 x 4 B) TMEM-copy layout
    uint8_t SFA[512];                  // unit scales (E4M3 1.0) for A, same layout
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
// producer's expect_tx arrive, or one per lane of producer_pool_async);
// `epi_arrivals` = arrivals that free an accumulator stage.
template <class P>
__device__ __forceinline__ void init_barriers(P& s, uint32_t epi_arrivals, uint32_t full_arrivals = 1) {
    for (int i = 0; i < P::kStages; ++i) {
        tc::mbar_init(&s.full[i], full_arrivals);
        tc::mbar_init(&s.empty[i], 1 + kEpiWarps);    // MMA commit + each epilogue warp
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
// and lay out the block-diagonal query operand.  Row n = 4b + h keeps head h's
// 8 code bytes of block b; all else zero.  (Block-major columns put the four
// heads of a block in adjacent accumulator registers, which score_of pairs.)
template <class P>
__device__ __forceinline__ void setup_query(P& s, const uint8_t* q, const uint8_t* qs, int lane, uint32_t cols) {
    tc::tmem_alloc(&s.tmem_base, cols);
    for (int i = lane; i < 16 * 32; i += 32) s.Bq[i] = 0;
    for (int i = lane; i < 512; i += 32) s.SFB[i] = 0;
    for (int i = lane; i < 512; i += 32) s.SFA[i] = 0x38;   // E4M3 1.0
    __syncwarp();
    if (lane < 16) {
        const int n = lane, h = n & 3, blk = n >> 2;
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

// Warp 0, dense rows [lo, hi) of the query's batch row (lo a multiple of 128):
// the cache stores each 128-entry tile as the MMA's operand image and the
// scales row-major, so a stage is one contiguous bulk copy of its tiles' codes
// and one of their scales.  Lane 0 issues.
//
// With `starve` (a test hook) the first stage's bytes are announced on its
// barrier but no copy is issued, so nothing ever completes that barrier: every
// wait on it runs out of time and the CTA winds down through its error path.
template <class P>
__device__ __forceinline__ void producer_dense(P& s, const uint8_t* ik, const uint8_t* iks, int64_t row_base, int lo,
                                               int ntiles, int nstages, int32_t* status, int lane, bool starve = false) {
    constexpr int kStages = P::kStages;
    int issued = 0;
    if (lane == 0) {
        if (starve && nstages > 0) {
            tc::mbar_arrive_expect_tx(&s.full[0], (uint32_t)min(kTPS, ntiles) * (kTile * 32u + kTile * 4u));
            issued = 1;
            nstages = 0;
        }
        for (int t = 0; t < nstages; ++t) {
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            if (!tc::mbar_wait_spin(&s.empty[slot], ph ^ 1u)) {
                raise_abort(s, status);
                break;
            }
            if (aborted(s)) break;
            const int64_t e0 = row_base + lo + (int64_t)t * kTPS * kTile;   // a tile boundary
            const int ntl = min(kTPS, ntiles - t * kTPS);
            tc::mbar_arrive_expect_tx(&s.full[slot], (uint32_t)ntl * (kTile * 32u + kTile * 4u));
            tc::bulk_load(s.A[slot], ik + ik_code_off(e0, 0), (uint32_t)ntl * kTile * 32u, &s.full[slot]);
            tc::bulk_load(s.SF[slot], iks + ik_scale_off(e0), (uint32_t)ntl * kTile * 4u, &s.full[slot]);
            ++issued;
        }
        // never leave copies in flight: wait (bounded) for the stages still pending
        for (int t = max(0, issued - kStages); t < issued; ++t)
            if (!tc::mbar_wait(&s.full[t % kStages], (uint32_t)(t / kStages) & 1u)) raise_abort(s, status);
    }
    __syncwarp();
}

// Warp 0, pool slots [lo, hi): 16 blocks of 8 entries per tile.  A block's codes
// are two core matrices, 256 contiguous bytes of the cache, copied into row
// group j of the tile; its 8 rows of scales, 32 contiguous bytes, into rows
// 8 j .. 8 j + 7 of the stage's scales.  Lanes 0..15 issue (one block each).
template <class P>
__device__ __forceinline__ void producer_pool(P& s, const uint8_t* ik, const uint8_t* iks, int64_t row_base, int lo,
                                              int hi, int ntiles, int nstages, const int32_t* pool, int nvis,
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
        // lane j < 16 of tile i: pool slot lo + (t kTPS + i) 16 + j
        int blk[kTPS];
        uint32_t live = 0;
#pragma unroll
        for (int i = 0; i < kTPS; ++i) {
            const int g = t * kTPS + i;
            const int sl = lo + g * kPoolPerTile + (lane & 15);
            blk[i] = (g < ntiles && lane < kPoolPerTile && sl < hi) ? __ldg(pool + sl) : -1;
            if (blk[i] >= 0 && (int64_t)blk[i] * kBlk >= nvis) blk[i] = -1;
            live += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, blk[i] >= 0));
        }
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.full[slot], live * (256u + 32u));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kTPS; ++i) {
            if (blk[i] < 0) continue;
            const int64_t e = row_base + (int64_t)blk[i] * kBlk;
            tc::bulk_load(s.A[slot][i] + 256 * lane, ik + ik_code_off(e, 0), 256u, &s.full[slot]);
            tc::bulk_load(s.SF[slot][i] + 32 * lane, iks + ik_scale_off(e), 32u, &s.full[slot]);
        }
        ++issued;
    }
    // never leave copies in flight: wait (bounded) for the stages still pending
    if (lane == 0) {
        for (int t = max(0, issued - kStages); t < issued; ++t)
            if (!tc::mbar_wait(&s.full[t % kStages], (uint32_t)(t / kStages) & 1u)) raise_abort(s, status);
    }
    __syncwarp();
}

// Warp 0, the same pool slots as producer_pool, copied by the 32 lanes with 16-byte
// cp.async instead of two bulk copies per block.  Each bulk copy is one request to the
// copy engine, and at 8 blocks a share of 2,048 slots issue thousands of them; here lane l
// copies half (l % 2) of the codes of block l / 2 of each tile (8 chunks) and one of the
// block's two scale chunks.  The copies write through the generic proxy, so a lane waits
// for its own copies of a stage, fences them to the async proxy (the MMA reads the codes
// there) and then arrives on the stage's barrier, which expects kPoolLanes arrivals.  The
// wait trails the issue by kLag stages so that copies of several stages are in flight.
// The pool slots are read kAhead stages before their copies are issued (a dependent
// global load per stage would otherwise sit in front of every issue), and each stage's
// block ids (-1 = no block) go to `stage_blk` ([kStages][kTPS][kPoolPerTile] in shared
// memory) before the stage's arrivals, for the epilogue to read after its wait.
constexpr uint32_t kPoolLanes = 32;
template <class P>
__device__ __forceinline__ void producer_pool_async(P& s, const uint8_t* ik, const uint8_t* iks, int64_t row_base,
                                                    int lo, int hi, int ntiles, int nstages, const int32_t* pool,
                                                    int nvis, int32_t* stage_blk, int32_t* status, int lane) {
    constexpr int kStages = P::kStages;
    constexpr int kLag = kStages > 2 ? 2 : 1;   // < kStages: stage t - kStages has arrived before t waits
    constexpr int kAhead = 2;
    const int j = lane >> 1, half = lane & 1;
    int nxt[kAhead + 1][kTPS];
    auto read_slots = [&](int t, int (&b)[kTPS]) {
#pragma unroll
        for (int i = 0; i < kTPS; ++i) {
            const int g = t * kTPS + i;
            const int sl = lo + g * kPoolPerTile + j;
            b[i] = (t < nstages && g < ntiles && sl < hi) ? __ldg(pool + sl) : -1;
        }
    };
#pragma unroll
    for (int a = 0; a < kAhead; ++a) read_slots(a, nxt[a]);
    int issued = 0, arrived = 0;
    for (int t = 0; t < nstages; ++t) {
        const int slot = t % kStages;
        const uint32_t ph = (uint32_t)(t / kStages) & 1u;
        read_slots(t + kAhead, nxt[kAhead]);
        int cur[kTPS];
#pragma unroll
        for (int i = 0; i < kTPS; ++i) {
            cur[i] = nxt[0][i];
#pragma unroll
            for (int a = 0; a < kAhead; ++a) nxt[a][i] = nxt[a + 1][i];
        }
        int ok = 1;
        if (lane == 0) ok = tc::mbar_wait_spin(&s.empty[slot], ph ^ 1u);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (lane == 0 && !ok) raise_abort(s, status);
        if (__any_sync(0xFFFFFFFFu, !ok || aborted(s))) break;   // warp-uniform
#pragma unroll
        for (int i = 0; i < kTPS; ++i) {
            int blk = cur[i];
            if (blk >= 0 && (int64_t)blk * kBlk >= nvis) blk = -1;
            if (half == 0) stage_blk[(slot * kTPS + i) * kPoolPerTile + j] = blk;
            if (blk < 0) continue;
            const int64_t e = row_base + (int64_t)blk * kBlk;
            const uint32_t dA = tc::smem_u32(s.A[slot][i] + 256 * j + 128 * half);
            const uint8_t* sA = ik + ik_code_off(e, 0) + 128 * half;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dA + 16u * c), "l"(sA + 16 * c) : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(s.SF[slot][i] + 32 * j + 16 * half)),
                         "l"(iks + ik_scale_off(e) + 16 * half)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        ++issued;
        if (issued - arrived > kLag) {
            asm volatile("cp.async.wait_group %0;" ::"n"(kLag) : "memory");
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&s.full[arrived % kStages]);
            ++arrived;
        }
    }
    // never leave copies in flight, and complete every stage that was issued
    asm volatile("cp.async.wait_all;" ::: "memory");
    tc::fence_proxy_async_smem();
    for (; arrived < issued; ++arrived) tc::mbar_arrive(&s.full[arrived % kStages]);
    __syncwarp();
}

// Warp 1 (lane 0 issues).  Returns once every MMA it issued has completed.
template <class P>
__device__ __forceinline__ void mma_issuer(P& s, int ntiles, int nstages, int32_t* status, int lane) {
    constexpr int kStages = P::kStages;
    const uint32_t tbase = s.tmem_base;
    if (lane == 0) {
        tc::tc_fence_after();
        tc::tmem_cp_32x128_x4(tbase + kColSfa, tc::smem_desc(tc::smem_u32(s.SFA), 16, 128, tc::kLayoutNone));
        tc::tmem_cp_32x128_x4(tbase + kColSfb, tc::smem_desc(tc::smem_u32(s.SFB), 16, 128, tc::kLayoutNone));
        const uint64_t bdesc = tc::smem_desc(tc::smem_u32(s.Bq), 128, 256, tc::kLayoutNone);
        for (int t = 0; t < nstages; ++t) {
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            if (!tc::mbar_wait_spin(&s.full[slot], ph) || !tc::mbar_wait_spin(&s.accempty[a], aph ^ 1u)) {
                raise_abort(s, status);
                break;
            }
            if (aborted(s)) break;
            tc::tc_fence_after();
            for (int i = 0; i < kTPS; ++i) {
                if (t * kTPS + i >= ntiles) break;
                const uint64_t adesc = tc::smem_desc(tc::smem_u32(s.A[slot][i]), 128, 256, tc::kLayoutNone);
                tc::mma_mxf4nvf4(tbase + kColAcc + (uint32_t)(a * kTPS + i) * 16, adesc, bdesc, kIdesc, 0u,
                                 tbase + kColSfa, tbase + kColSfb);
            }
            tc::tc_commit(&s.empty[slot]);
            tc::tc_commit(&s.accfull[a]);
        }
        tc::tc_commit(&s.done);
        if (!tc::mbar_wait(&s.done, 0)) raise_abort(s, status);
    }
    __syncwarp();
}

// Packed fp32 pairs: one IEEE round-to-nearest product or sum per lane.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// The row's four key block scales as (sk_b, sk_b) pairs.
struct KeyScales {
    uint64_t s2[4];
};
__device__ __forceinline__ KeyScales key_scales(uint32_t sk_bytes) {
    float sk[4];
    e4m3x4_to_f32(sk_bytes, sk);
    KeyScales k;
#pragma unroll
    for (int b = 0; b < 4; ++b) k.s2[b] = f2pack(sk[b], sk[b]);
    return k;
}

// The defined score of one row from its 16 accumulator columns (column 4b + h =
// block b of head h, without the key's scale) and the row's key scales:
//   T[h][b] = acc * sk[b];  d_h = ((T0 + T1) + T2) + T3;  r_h = max(d_h, +0);
//   score = ((w0 r0 + w1 r1) + w2 r2) + w3 r3,
// every product and sum one fp32 rounding.  Heads (0, 1) and (2, 3) run as
// packed pairs (lane by lane the same IEEE operations).  w01 = (w0, w1), w23 = (w2, w3).
// Each block product is exact in fp32 (the accumulator has at most 16
// significant bits, an E4M3 scale at most 4), so a fused multiply-add of the
// next block onto the running sum rounds exactly as the separate add of that
// product does: d_h takes one multiply and three fused multiply-adds.  The head
// products w_h r_h are not exact and keep their own rounding.
__device__ __forceinline__ float score_of(const uint32_t (&v)[16], const KeyScales& ks, uint64_t w01, uint64_t w23) {
    uint64_t d01 = f2mul(f2pack(__uint_as_float(v[0]), __uint_as_float(v[1])), ks.s2[0]);
    uint64_t d23 = f2mul(f2pack(__uint_as_float(v[2]), __uint_as_float(v[3])), ks.s2[0]);
#pragma unroll
    for (int b = 1; b < 4; ++b) {
        d01 = f2fma(f2pack(__uint_as_float(v[4 * b]), __uint_as_float(v[4 * b + 1])), ks.s2[b], d01);
        d23 = f2fma(f2pack(__uint_as_float(v[4 * b + 2]), __uint_as_float(v[4 * b + 3])), ks.s2[b], d23);
    }
    float r0, r1, r2, r3;
    f2unpack(d01, r0, r1);
    f2unpack(d23, r2, r3);
    r0 = r0 > 0.0f ? r0 : 0.0f;
    r1 = r1 > 0.0f ? r1 : 0.0f;
    r2 = r2 > 0.0f ? r2 : 0.0f;
    r3 = r3 > 0.0f ? r3 : 0.0f;
    float p0, p1, p2, p3;
    f2unpack(f2mul(w01, f2pack(r0, r1)), p0, p1);
    f2unpack(f2mul(w23, f2pack(r2, r3)), p2, p3);
    return __fadd_rn(__fadd_rn(__fadd_rn(p0, p1), p2), p3);
}

// Epilogue warp, stage t in ring slot `slot`: the 4 scale bytes of row `row` of
// tile i, read after the stage's copies are seen to have landed.
template <class P>
__device__ __forceinline__ uint32_t stage_scales(const P& s, int slot, int i, int row) {
    return *reinterpret_cast<const uint32_t*>(&s.SF[slot][i][4 * row]);
}

// Epilogue warp: wait (bounded; the phase has normally completed already) for
// the stage's copies, which makes the bulk-copied scale bytes visible here.
template <class P>
__device__ __forceinline__ bool stage_landed(P& s, int t) {
    return tc::mbar_wait(&s.full[t % P::kStages], (uint32_t)(t / P::kStages) & 1u);
}

// Epilogue warp: done with the stage's scales (lane 0 arrives once per warp).
template <class P>
__device__ __forceinline__ void release_stage(P& s, int t, int lane) {
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&s.empty[t % P::kStages]);
}

}  // namespace pipe
}  // namespace csa2
