// index_cluster.cu -- csa2_index_topk for decode-sized query counts: one
// thread-block cluster of C CTAs per query, an exact Top-K by radix select
// over the whole cluster, no merge and no sort.
//
// Each CTA scores a contiguous 1/C of the query's visible entries with the
// tcgen05 pipeline of index_pipe.cuh (a stage is one bulk copy of four tiles'
// codes and one of their scales; 8 stages in flight) and keeps every order key
// in TMEM (lane m, one column per tile: up to 32,768 keys beside the
// pipeline's 256 columns), while the epilogue counts the keys' top 11 bits
// into a 2,048-bin histogram.  The cluster sums the histograms through
// distributed shared memory and finds the bin d1 holding the K-th largest key.
// One read of the keys then marks every entry of a higher bin as selected
// (position bitmaps) and lists the entries of bin d1, the candidates.  When the
// cluster's candidates are few (the usual case) every CTA gathers all of them
// and finds the K-th key T exactly with two local radix passes (bits 20..10,
// 9..0); otherwise (many equal or close keys) two more passes over the keys in
// TMEM find T with cluster-wide histograms.  The selected set is every key
// above T plus the lowest-positioned keys equal to T (ties go to the lower
// position).  CTA r covers positions below those of CTA r + 1, so its quota of
// ties and its output offset follow from the lower-ranked CTAs' counts, and
// two block-wide prefix sums over the bitmap words give every selected
// position its place in the ascending output.
//
// Every mbarrier wait of the scoring pipeline is bounded; every thread of
// every CTA reaches each cluster barrier (and each named barrier of its warp
// group) the same number of times whatever happened before it, so no barrier
// can wait on a thread that has left.
#include "cluster.cuh"
#include "index_pipe.cuh"

namespace csa2 {
namespace {

using namespace pipe;

constexpr int kThreads = 512;              // warp 0 copies, warp 1 MMA, warps 2-9 epilogue; all 16 select
constexpr int kEpiN = 256;
constexpr int kEpiWarps = kEpiN / 32;
constexpr int kSwW = kThreads / 32;        // warps that sweep the stored keys: four per TMEM lane quarter
constexpr int kTPG = kTPS / 2;             // tiles of a stage per epilogue warp group
constexpr int kRing = 8;                   // shared-memory stages in flight
constexpr int kMaxTiles = 256;             // 32,768 entries per CTA with the keys in TMEM
constexpr int kMaxTilesG = 512;            // 65,536 entries per CTA with the keys in the workspace
constexpr uint32_t kColKeys = kPipeCols;   // key of tile g, row m: TMEM lane m, column kColKeys + g
constexpr uint32_t kTmemCols = kPipeCols + kMaxTiles;
constexpr int kWords = kMaxTilesG * kTile / 32;         // bitmap words over the CTA's entries
constexpr int kWPT = kWords / 256;                      // bitmap words per scanning thread
constexpr int kNB1 = 2048, kNB2 = 2048, kNB3 = 1024;   // radix digits: bits 31..21, 20..10, 9..0
constexpr int kSel = 256;                  // threads of the scans (warps 0-7)
constexpr int kCandPerWarp = 128;          // candidates (keys of the threshold's top bin) a sweeping warp lists
constexpr int kCandCap = kSwW * kCandPerWarp; // and a CTA
constexpr int kGatherCap = 8192;           // candidates of a cluster gathered for the local select
constexpr uint32_t kSlowPath = 0xFFFFFFFFu;
constexpr int kSelWarps = kSel / 32;
using ClPipe = Pipe<kRing>;
static_assert((kNB2 + kNB3 + 2 * kWords) * 4 + (2 * kCandCap + kGatherCap) * 8 <= (int)sizeof(ClPipe::A),
              "select scratch fits the ring");
static_assert(kTmemCols == 512, "TMEM");
static_assert(kWPT * 256 == kWords && kSel == 256, "bitmap words per scanning thread");

struct ClSmem {
    ClPipe pipe;                            // its A ring holds hist2, hist3 and two bitmaps after scoring
    alignas(16) uint32_t hist1[kNB1];
    uint32_t wsum[kSelWarps];               // scan: per-warp totals
    uint32_t res[2];                        // find_bin: (bin, keys above the bin)
    uint32_t wcnt[kSwW][2];                 // per sweeping warp: keys > T, keys == T
    alignas(8) uint32_t pub[2];             // this CTA's (entries above bin d1, candidates), read by the cluster
    alignas(8) uint32_t pub2[2];            // (> T, == T) counts of the multi-pass path, read by the cluster
    uint32_t cbase[2];                      // this CTA's tie quota and output offset
    uint32_t wcand[kSwW];                   // candidates each sweeping warp found (may exceed its list)
    alignas(8) uint32_t coarse[16][64];     // every rank's hist1 in 64 bins of 32, pushed by that rank
    uint32_t fast;                          // candidates of the cluster, or kSlowPath
    uint32_t peer[16][2];                   // per CTA: entries above bin d1, candidates of lower ranks
    uint32_t rcnt[16][2];                   // per CTA: candidates above T, equal to T
};

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// v[j] for a run-time j without indexing the array (which would move it to
// local memory): a binary select tree on the bits of j.
__device__ __forceinline__ uint32_t pick32(const uint32_t (&v)[32], uint32_t j) {
    uint32_t a[16], b[8], c[4], d[2];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = (j & 16u) ? v[i + 16] : v[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = (j & 8u) ? a[i + 8] : a[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = (j & 4u) ? b[i + 4] : b[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) d[i] = (j & 2u) ? c[i + 2] : c[i];
    return (j & 1u) ? d[1] : d[0];
}

// 32 x 32 bit transpose across the warp: in, bit j of lane l is element
// (l, j); out, bit l of lane j is element (l, j).  Five block swaps of halving
// size through shuffles.
__device__ __forceinline__ uint32_t warp_transpose_bits(uint32_t x, int lane) {
    constexpr uint32_t kMask[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        const int sh = 16 >> i;
        const uint32_t m = kMask[i];
        const uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, sh);
        x = (lane & sh) ? ((x & ~m) | ((y >> sh) & m)) : ((x & m) | ((y << sh) & ~m));
    }
    return x;
}

// Exclusive prefix of v over threads 0..255 in thread order (threads 256+ pass
// 0 and get nothing useful); *total = the sum.  All threads of the CTA call it.
__device__ __forceinline__ uint32_t block_scan_excl(ClSmem& s, uint32_t v, int tid, uint32_t* total) {
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t inc = warp_incl_scan(v, lane);
    if (lane == 31 && warp < kSelWarps) s.wsum[warp] = inc;
    __syncthreads();
    uint32_t pre = inc - v, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        if (w < warp) pre += s.wsum[w];
        tot += s.wsum[w];
    }
    *total = tot;
    __syncthreads();
    return pre;
}

// One warp: the bin d1 of hist1 (summed over the cluster's C CTAs) holding
// the R-th largest key, in two levels: the 64 coarse sums (32 bins each) give
// the coarse bin, its 32 bins the fine one.  Leaves (d1, keys above d1) in
// s.res for the CTA.
__device__ __forceinline__ void find_top_bin(ClSmem& s, uint32_t C, uint32_t R, int lane) {
    constexpr int RG = 4;   // CTAs whose loads are in flight together
    // lane l: coarse bins 2l and 2l + 1 (the highest bins on lane 31), every rank's in this CTA
    uint32_t lo = 0, hi = 0;
    for (uint32_t r = 0; r < C; ++r) {
        const uint2 x = *reinterpret_cast<const uint2*>(&s.coarse[r][2 * lane]);
        lo += x.x;
        hi += x.y;
    }
    uint32_t suf = lo + hi;   // keys in this lane's coarse bins and every higher lane's
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += y;
    }
    const uint32_t abv = suf - lo - hi;
    const int L = __ffs(__ballot_sync(0xFFFFFFFFu, abv < R && R <= suf)) - 1;
    uint32_t cb = 0, cab = 0;
    if (lane == L) {
        cb = abv + hi >= R ? 2u * lane + 1u : 2u * lane;
        cab = abv + hi >= R ? abv : abv + hi;
    }
    cb = __shfl_sync(0xFFFFFFFFu, cb, L);
    cab = __shfl_sync(0xFFFFFFFFu, cab, L);
    // lane l: bin 32 cb + l
    uint32_t f = 0;
    const uint32_t fa = tc::smem_u32(&s.hist1[32 * cb + lane]);
    for (uint32_t r0 = 0; r0 < C; r0 += RG) {
        uint32_t x[RG];
#pragma unroll
        for (int g = 0; g < RG; ++g) x[g] = r0 + g < C ? cl::ld_u32(cl::map_rank(fa, r0 + g)) : 0u;
#pragma unroll
        for (int g = 0; g < RG; ++g) f += x[g];
    }
    uint32_t fs = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, fs, o);
        if (lane + o < 32) fs += y;
    }
    const uint32_t R2 = R - cab, fab = fs - f;
    if (fab < R2 && R2 <= fs) {
        s.res[0] = 32u * cb + (uint32_t)lane;
        s.res[1] = cab + fab;
    }
}

// Sum the NB-bin histogram `hist` over the CTAs r0 .. r0 + n - 1 of the
// cluster (n = 1, r0 = own rank: this CTA's alone) and find the bin b holding
// the R-th largest key (R >= 1): keys above b < R <= keys above b + count of b.
// Leaves (b, keys above b) in s.res.  All threads of the CTA call it.
template <int NB>
__device__ __forceinline__ void find_bin(ClSmem& s, const uint32_t* hist, uint32_t r_first, uint32_t n, uint32_t R,
                                         int tid) {
    constexpr int PER = NB / kSel;   // bins per thread, highest bins on thread 0
    constexpr int NV = PER / 4;      // 16-byte loads per CTA
    constexpr int RG = 4;            // CTAs whose loads are in flight together
    static_assert(PER % 4 == 0, "vector loads");
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t h[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) h[j] = 0;
    const int b0 = NB - PER * (tid + 1);   // this thread's lowest bin
    if (tid < kSel) {
        const uint32_t la = tc::smem_u32(hist + b0);
        for (uint32_t r0 = 0; r0 < n; r0 += RG) {
            uint4 x[RG][NV];
#pragma unroll
            for (int g = 0; g < RG; ++g)
                if (r0 + g < n) {
                    const uint32_t ra = cl::map_rank(la, r_first + r0 + g);
#pragma unroll
                    for (int v = 0; v < NV; ++v) x[g][v] = cl::ld_v4(ra + 16u * v);
                }
#pragma unroll
            for (int g = 0; g < RG; ++g)
                if (r0 + g < n) {
#pragma unroll
                    for (int v = 0; v < NV; ++v) {
                        h[4 * v + 0] += x[g][v].x;
                        h[4 * v + 1] += x[g][v].y;
                        h[4 * v + 2] += x[g][v].z;
                        h[4 * v + 3] += x[g][v].w;
                    }
                }
        }
    }
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) sum += h[j];
    const uint32_t inc = warp_incl_scan(sum, lane);
    if (lane == 31 && warp < kSelWarps) s.wsum[warp] = inc;
    if (tid == 0) {
        s.res[0] = 0;
        s.res[1] = 0;
    }
    __syncthreads();
    if (tid < kSel) {
        uint32_t above = inc - sum;
        for (int w = 0; w < warp; ++w) above += s.wsum[w];
        if (above < R && R <= above + sum) {
#pragma unroll
            for (int j = PER - 1; j >= 0; --j) {
                if (above + h[j] >= R) {
                    s.res[0] = (uint32_t)(b0 + j);
                    s.res[1] = above;
                    break;
                }
                above += h[j];
            }
        }
    }
    __syncthreads();
}

// Visit every stored key of this CTA, 32 tile columns at a time: all 16 warps,
// TMEM lane quarter q = warp % 4, columns [64 h, 64 h + 64) with h = warp / 4.
// f(v, c0, q) gets the keys of columns c0 .. c0 + 31 of this lane; column c of
// lane l holds CTA-local entry 128 c + 32 q + l.
template <class F>
__device__ __forceinline__ void sweep_cols(uint32_t tbase, int warp, int ntiles, F&& f) {
    static_assert(kSwW == 16 && kMaxTiles == 4 * 64, "four warps of 64 columns per lane quarter");
    const int quarter = warp & 3, part = warp >> 2;
    const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
    for (int c0 = part * 64; c0 < min(ntiles, part * 64 + 64); c0 += 32) {
        uint32_t v[32];
        tc::tmem_ld_32x32b_x32(tbase + lanes + kColKeys + (uint32_t)c0, v);
        tc::tmem_ld_wait();
        f(v, c0, quarter);
    }
}

// The same visit when the keys sit in the workspace (key of CTA-local entry l at keys[l]):
// columns [128 h, 128 h + 128) for h = warp / 4, each lane's 32 keys of a chunk by 32
// coalesced loads (the keys were written moments before and are in L2).
template <class F>
__device__ __forceinline__ void sweep_cols_g(const uint32_t* keys, int warp, int ntiles, F&& f) {
    static_assert(kSwW == 16 && kMaxTilesG == 4 * 128, "four warps of 128 columns per lane quarter");
    const int quarter = warp & 3, part = warp >> 2, lane = threadIdx.x & 31;
    for (int c0 = part * 128; c0 < min(ntiles, part * 128 + 128); c0 += 32) {
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            v[j] = c0 + j < ntiles ? __ldcg(keys + 128 * (c0 + j) + 32 * quarter + lane) : 0u;
        f(v, c0, quarter);
    }
}

// MODE 0: index + Top-K (keys = the fixed-order scores of the visible entries);
// MODE 1: pool build (keys = the block maxima of the visible blocks, items = block ids);
// MODE 2: pool Top-K (items = the pool's slots x 8 positions, in ascending position order
//         since the pool lists its blocks ascending; keys = the scores of the visible ones).
// KG: the keys go to the workspace (p.keys, [B Q][cap]) instead of TMEM, for up to
// kMaxTilesG tiles per CTA (the index of a query with more entries than 16 CTAs hold in TMEM).
template <int MODE, bool KG = false>
__global__ void __launch_bounds__(kThreads, 1)
    index_cluster_kernel(SelectParams p) {
    pdl_enter();
    cl::arrive_relaxed();   // waited on before the first store into another CTA (every CTA has started)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    ClSmem& s = *reinterpret_cast<ClSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cl::rank(), C = cl::ctas();
    const int bq = blockIdx.y;
    const int b = bq / p.Q;
    const int k = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const int64_t row_base = (int64_t)b * p.cap;
    // the items: visible entries, or visible blocks of 8 entries (at most nb_cap)
    const int nitems = MODE == 0 ? nvis
                       : MODE == 1 ? (int)min((int64_t)((nvis + kBlk - 1) / kBlk), p.nb_cap)
                                   : p.P * kBlk;
    const int32_t* pool = MODE == 2 ? p.pool + (int64_t)bq * p.P : nullptr;
    // this CTA's items [lo, hi); the host keeps the chunk within kMaxTiles tiles
    const int chunk = ((nitems + (int)C - 1) / (int)C + kTile - 1) / kTile * kTile;
    const int lo = min(nitems, (int)rank * chunk), hi = min(nitems, lo + chunk);
    const int ntiles = (hi - lo + kTile - 1) / kTile;
    const int nstages = (ntiles + kTPS - 1) / kTPS;
    int32_t* status = p.status;
    int32_t* out = p.out + (int64_t)bq * k;
    static_assert(!KG || MODE == 0, "workspace keys: the index only");
    uint32_t* const keys = KG ? p.keys + (int64_t)bq * p.cap + lo : nullptr;   // key of CTA-local entry l at keys[l]

    // Warp 0 starts the copies as soon as the barriers exist; the other warps set up
    // the query, TMEM and the histogram meanwhile and meet on named barrier 1 (warp 0
    // only arrives there).  The pool build has no pipeline: TMEM and the histogram only.
    if constexpr (MODE == 1) {
        if (warp == 1) tc::tmem_alloc(&s.pipe.tmem_base, kTmemCols);
        for (int i = tid; i < kNB1; i += kThreads) s.hist1[i] = 0;
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    } else if (warp == 0) {
        if (lane == 0) init_barriers(s.pipe, kEpiN);
        __syncwarp();
        asm volatile("bar.arrive 1, %0;" ::"n"(kThreads) : "memory");
        if constexpr (MODE == 2)
            producer_pool(s.pipe, p.ik, p.ik_sc, row_base, lo / kBlk, hi / kBlk, ntiles, nstages, pool, nvis, status, lane);
        else
            producer_dense(s.pipe, p.ik, p.ik_sc, row_base, lo, ntiles, nstages, status, lane);
    } else {
        if (warp == 1) setup_query(s.pipe, p.q + (int64_t)bq * 128, p.q_sc + (int64_t)bq * 16, lane, kTmemCols);
        for (int i = tid - 32; i < kNB1; i += kThreads - 32) s.hist1[i] = 0;
        tc::tc_fence_before();
        asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
        tc::tc_fence_after();
    }
    uint32_t tbase = (MODE == 0 && warp == 0) ? 0u : s.pipe.tmem_base;   // warp 0 reads it after scoring

    if constexpr (MODE == 1) {
        // ------------------------------------------------------------ block maxima
        // warps 2-9: lane quarter q, columns [128 h, 128 h + 128) (h = (warp - 2) / 4); the key of
        // column c, lane l is block lo + 128 c + 32 q + l; eight loads in flight per lane
        if (warp >= 2 && warp < 2 + kEpiWarps) {
            const int quarter = warp & 3, half = (warp - 2) >> 2;
            const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
            const float* bmr = p.blockmax + (int64_t)bq * p.nb_cap;
            for (int c0 = half * 128; c0 < min(ntiles, half * 128 + 128); c0 += 8) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = lo + 128 * (c0 + j) + 32 * quarter + lane;
                    v[j] = (c0 + j < ntiles && e < hi) ? __ldg(bmr + e) : 0.0f;
                }
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    uint32_t key[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int e = lo + 128 * (c0 + j + i) + 32 * quarter + lane;
                        const bool valid = c0 + j + i < ntiles && e < hi;
                        key[i] = valid ? score_key(v[j + i]) : 0u;
                        if (valid) atomicAdd(&s.hist1[key[i] >> 21], 1u);
                    }
                    if (c0 + j + 1 < ntiles) tc::tmem_st_32x32b_x2(tbase + lanes + kColKeys + (uint32_t)(c0 + j), key[0], key[1]);
                    else if (c0 + j < ntiles) tc::tmem_st_32x32b_x1(tbase + lanes + kColKeys + (uint32_t)(c0 + j), key[0]);
                }
            }
            tc::tmem_st_wait();
        }
    } else if (warp == 0) {
    } else if (warp == 1) {
        mma_issuer(s.pipe, ntiles, nstages, status, lane);
    } else if (warp < 2 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;             // TMEM lanes this warp may read
        const int group = (warp - 2) >> 2;        // tiles 2*group, 2*group+1 of each stage
        const int eo = quarter * 32 + lane;       // this thread's TMEM row = its entry within a tile
        const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
        const uint64_t w01 = f2pack(__ldg(p.w + (int64_t)bq * 4 + 0), __ldg(p.w + (int64_t)bq * 4 + 1));
        const uint64_t w23 = f2pack(__ldg(p.w + (int64_t)bq * 4 + 2), __ldg(p.w + (int64_t)bq * 4 + 3));
        float* bm = (MODE == 0 && p.blockmax) ? p.blockmax + (int64_t)bq * p.nb_cap : nullptr;
        bool dead = false;   // this warp stopped after a failed wait (or another role's)
        for (int t = 0; t < nstages; ++t) {
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            if (!dead && __any_sync(0xFFFFFFFFu, aborted(s.pipe))) dead = true;
            if (!dead && !__all_sync(0xFFFFFFFFu, tc::mbar_wait_spin(&s.pipe.accfull[a], aph))) {   // warp-uniform
                if (lane == 0) raise_abort(s.pipe, status);
                dead = true;
            }
            if (!dead) {
                tc::tc_fence_after();
                uint32_t v[kTPG][16];
#pragma unroll
                for (int j = 0; j < kTPG; ++j)
                    tc::tmem_ld_32x32b_x16(tbase + lanes + kColAcc + (uint32_t)(a * kTPS + kTPG * group + j) * 16, v[j]);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                tc::mbar_arrive(&s.pipe.accempty[a]);
                if (!__all_sync(0xFFFFFFFFu, stage_landed(s.pipe, t))) {   // warp-uniform
                    if (lane == 0) raise_abort(s.pipe, status);
                    dead = true;
                    continue;
                }
                uint32_t skw[kTPG];
#pragma unroll
                for (int j = 0; j < kTPG; ++j) skw[j] = stage_scales(s.pipe, t % kRing, kTPG * group + j, eo);
                release_stage(s.pipe, t, lane);
                const int g0 = t * kTPS + kTPG * group;
                uint32_t key[kTPG];
#pragma unroll
                for (int j = 0; j < kTPG; ++j) {
                    const int g = g0 + j;
                    bool valid = g < ntiles && lo + g * kTile + eo < hi;
                    if (MODE == 2 && valid) {   // slot (item / 8) of the pool, position blk 8 + item % 8
                        const int item = lo + g * kTile + eo;
                        const int blk = __ldg(pool + item / kBlk);
                        valid = blk >= 0 && (int64_t)blk * kBlk + (item % kBlk) < nvis;
                    }
                    const float score = valid ? score_of(v[j], key_scales(skw[j]), w01, w23) : -INFINITY;
                    key[j] = valid ? score_key(score) : 0u;
                    if (valid) atomicAdd(&s.hist1[key[j] >> 21], 1u);
                    if (bm) {
                        const float mx = block_max8(score, lane);
                        if ((lane & (kBlk - 1)) == 0 && valid) bm[(lo + g * kTile + eo) >> 3] = mx;
                    }
                }
                if constexpr (KG) {   // every row of a live column, 128 bytes per warp
#pragma unroll
                    for (int j = 0; j < kTPG; ++j)
                        if (g0 + j < ntiles) __stcg(keys + (g0 + j) * kTile + eo, key[j]);
                } else if (g0 + 1 < ntiles) {
                    tc::tmem_st_32x32b_x2(tbase + lanes + kColKeys + (uint32_t)g0, key[0], key[1]);
                } else if (g0 < ntiles) {
                    tc::tmem_st_32x32b_x1(tbase + lanes + kColKeys + (uint32_t)g0, key[0]);
                }
            }
        }
        tc::tmem_st_wait();
        if (bm) {  // blocks with no visible position, split over the cluster
            const int64_t jb = (nvis + kBlk - 1) / kBlk;
            const int64_t rest = p.nb_cap - jb;
            if (rest > 0) {
                const int64_t cs = (rest + C - 1) / C;
                const int64_t j0 = jb + (int64_t)rank * cs, j1 = min(p.nb_cap, j0 + cs);
                for (int64_t j = j0 + (tid - 64); j < j1; j += kEpiN) bm[j] = -INFINITY;
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    tbase = s.pipe.tmem_base;
    cl::wait_acquire();
    // a visit of every stored key, from TMEM or (KG) from the workspace
    auto sweep = [&](auto&& f) {
        if constexpr (KG) sweep_cols_g(keys, warp, ntiles, f);
        else sweep_cols(tbase, warp, ntiles, f);
    };

    // ---------------------------------------------------------------- select
    uint32_t K1 = (uint32_t)min(k, nitems);   // the pool mode takes its count of valid items below
    if (MODE != 2 && K1 == 0) {   // the same for every CTA of the cluster: nothing visible
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = -1;
        if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
        return;
    }
    uint32_t* hist2 = reinterpret_cast<uint32_t*>(&s.pipe.A[0][0][0]);
    uint32_t* hist3 = hist2 + kNB2;
    uint32_t* selbm = hist3 + kNB3;   // entries above T (then also the ties taken)
    uint32_t* tiebm = selbm + kWords; // entries equal to T
    uint2* cand = reinterpret_cast<uint2*>(tiebm + kWords);   // this CTA's keys of bin d1: (key, entry)
    uint2* wlist = cand + kCandCap;                            // each sweeping warp's, before compaction
    uint2* gath = wlist + kCandCap;                            // the cluster's, gathered: (key, entry | rank << 16)
    for (int i = tid; i < kNB2 + kNB3 + 2 * kWords; i += kThreads) hist2[i] = 0;
    if (tid < 32) s.rcnt[tid >> 1][tid & 1] = 0;
    {   // hist1 in coarse bins of 32, pushed to every rank for the cluster's two-level search
        static_assert(kSwW * 4 == 64, "four coarse bins per warp");
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int cb = 4 * warp + i;
            const uint32_t x = __reduce_add_sync(0xFFFFFFFFu, s.hist1[32 * cb + lane]);
            if ((uint32_t)lane < C) cl::st_u32(cl::map_rank(tc::smem_u32(&s.coarse[rank][cb]), (uint32_t)lane), x);
        }
    }

    cl::sync();                                   // every CTA's hist1 is complete
    if constexpr (MODE == 2) {   // the cluster's valid items: the sum of every rank's coarse bins
        if (warp == 0) {
            uint32_t t = 0;
            for (uint32_t r = 0; r < C; ++r) t += s.coarse[r][2 * lane] + s.coarse[r][2 * lane + 1];
            t = __reduce_add_sync(0xFFFFFFFFu, t);
            if (lane == 0) s.res[0] = t;
        }
        __syncthreads();
        K1 = min((uint32_t)k, s.res[0]);
        __syncthreads();
        if (K1 == 0) {   // the same for every CTA of the cluster (the same totals)
            if (rank == 0)
                for (int i = tid; i < k; i += kThreads) out[i] = -1;
            if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
            return;
        }
    }
    if (warp == 0) find_top_bin(s, C, K1, lane);
    __syncthreads();
    const uint32_t d1 = s.res[0];
    const uint32_t R = K1 - s.res[1];             // keys still to take from bin d1 (1 <= R)

    // One read of the keys: an entry of a bin above d1 is selected whatever T
    // is (marked in the bitmaps: one word per column and lane quarter, built by
    // a bit transpose of the lanes' column masks); an entry of bin d1 is a
    // candidate, appended to this CTA's list.
    uint32_t above = 0, nlist = 0;   // nlist: this warp's candidates (warp-uniform)
    uint2* mylist = wlist + warp * kCandPerWarp;
    const uint32_t top = ((d1 + 1u) << 21) - 1u;   // keys above bin d1 are > top (none when d1 = 2047)
    const uint32_t bot = d1 << 21;                 // keys of bin d1: key - bot < 2^21
    sweep([&](const uint32_t(&v)[32], int c0, int q) {
        uint32_t ma4[4] = {0u, 0u, 0u, 0u}, mc4[4] = {0u, 0u, 0u, 0u};   // four short chains
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            ma4[j & 3] |= (uint32_t)(v[j] > top) << j;
            mc4[j & 3] |= (uint32_t)(v[j] - bot < (1u << 21)) << j;
        }
        // bit j: the key of column c0 + j is above bin d1 / in bin d1
        uint32_t ma = (ma4[0] | ma4[1]) | (ma4[2] | ma4[3]), mc = (mc4[0] | mc4[1]) | (mc4[2] | mc4[3]);
        if (ntiles - c0 < 32) {   // columns past the last tile hold no keys
            const uint32_t cm = (1u << (ntiles - c0)) - 1u;
            ma &= cm;
            mc &= cm;
        }
        const uint32_t word = warp_transpose_bits(ma, lane);   // column c0 + lane; bit l: lane l
        if (c0 + lane < ntiles) selbm[4 * (c0 + lane) + q] = word;
        above += __popc(word);
        if (__any_sync(0xFFFFFFFFu, mc != 0u)) {
            const uint32_t n = __popc(mc);
            const uint32_t incl = warp_incl_scan(n, lane);
            const uint32_t base = nlist + incl - n;
            nlist += __shfl_sync(0xFFFFFFFFu, incl, 31);
            const uint32_t e0 = 128u * (uint32_t)c0 + 32u * (uint32_t)q + (uint32_t)lane;
            // a lane has few candidates: visit its set bits, picking the key by a
            // five-level select on the column's bits (the keys stay in registers)
            uint32_t m = mc, slot = base;
            while (__any_sync(0xFFFFFFFFu, m != 0u)) {
                if (m != 0u) {
                    const uint32_t j = (uint32_t)__ffs(m) - 1u;
                    m &= m - 1u;
                    if (slot < (uint32_t)kCandPerWarp) mylist[slot] = make_uint2(pick32(v, j), e0 + 128u * j);
                    ++slot;
                }
            }
        }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xFFFFFFFFu, above, o);
    if (lane == 0) {
        s.wcnt[warp][0] = above;
        s.wcand[warp] = nlist;
    }
    tc::tc_fence_before();
    __syncthreads();
    {   // compact the warps' lists into this CTA's list, in warp order
        uint32_t base = 0;
        for (int w = 0; w < warp; ++w) base += min(s.wcand[w], (uint32_t)kCandPerWarp);
        const uint32_t n = min(nlist, (uint32_t)kCandPerWarp);
        for (uint32_t i = lane; i < n; i += 32) cand[base + i] = mylist[i];
    }
    if (tid == 0) {
        uint32_t a = 0, n = 0;
        bool over = false;
        for (int w = 0; w < kSwW; ++w) {
            a += s.wcnt[w][0];
            n += s.wcand[w];
            over = over || s.wcand[w] > (uint32_t)kCandPerWarp;
        }
        s.pub[0] = a;
        s.pub[1] = over ? (uint32_t)kCandCap + 1u : n;   // above the capacity: too many to gather
    }
    cl::sync();                                   // every CTA's counts and candidates are published
    if (warp == 0) {
        uint2 x = make_uint2(0u, 0u);
        if ((uint32_t)lane < C) x = cl::ld_v2(cl::map_rank(tc::smem_u32(s.pub), (uint32_t)lane));
        const uint32_t cincl = warp_incl_scan(x.y, lane);
        const bool over = __any_sync(0xFFFFFFFFu, x.y > (uint32_t)kCandCap);
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, cincl, 31);
        if ((uint32_t)lane < C) {
            s.peer[lane][0] = x.x;            // entries above bin d1
            s.peer[lane][1] = cincl - x.y;    // candidates of lower-ranked CTAs
        }
        if (lane == 0) s.fast = (!over && total <= (uint32_t)kGatherCap) ? total : kSlowPath;
    }
    __syncthreads();

    const uint32_t ncg = s.fast;
    if (ncg != kSlowPath) {
        // ---- the threshold bin is small: gather it and finish the select locally
        if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);   // no TMEM reads past this point
        constexpr int kU = 8;   // distributed loads in flight per thread
        for (uint32_t i0 = 0; i0 < ncg; i0 += kU * kThreads) {
            uint2 x[kU];
            uint32_t rr[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint32_t i = i0 + (uint32_t)(u * kThreads + tid);
                rr[u] = 0;
                x[u] = make_uint2(0u, 0u);
                if (i < ncg) {
                    uint32_t r = 0;
                    while (r + 1 < C && s.peer[r + 1][1] <= i) ++r;
                    rr[u] = r;
                    x[u] = cl::ld_v2(cl::map_rank(tc::smem_u32(&cand[i - s.peer[r][1]]), r));
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint32_t i = i0 + (uint32_t)(u * kThreads + tid);
                if (i < ncg) gath[i] = make_uint2(x[u].x, x[u].y | (rr[u] << 16));
            }
        }
        __syncthreads();
        for (uint32_t i = tid; i < ncg; i += kThreads) atomicAdd(&hist2[(gath[i].x >> 10) & (kNB2 - 1)], 1u);
        __syncthreads();
        find_bin<kNB2>(s, hist2, rank, 1, R, tid);
        const uint32_t p2 = (d1 << 11) | s.res[0];
        const uint32_t R3 = R - s.res[1];
        for (uint32_t i = tid; i < ncg; i += kThreads) {
            const uint32_t key = gath[i].x;
            if ((key >> 10) == p2) atomicAdd(&hist3[key & (kNB3 - 1)], 1u);
        }
        __syncthreads();
        find_bin<kNB3>(s, hist3, rank, 1, R3, tid);
        const uint32_t T = (p2 << 10) | s.res[0];
        const uint32_t Rt = R3 - s.res[1];   // keys equal to T to take, lowest positions first (1 <= Rt)
        // every CTA's counts above and at T; this CTA's own candidates into the bitmaps
        for (uint32_t i = (uint32_t)(warp * 32 + lane); i - (uint32_t)lane < ncg; i += kThreads) {
            const bool ok = i < ncg;
            const uint2 x = ok ? gath[i] : make_uint2(0u, 0u);
            const uint32_t r = ok ? (x.y >> 16) : 0xFFFFu;
            const bool gt = ok && x.x > T, eq = ok && x.x == T;
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, r);
            const uint32_t bg = __ballot_sync(0xFFFFFFFFu, gt) & peers, be = __ballot_sync(0xFFFFFFFFu, eq) & peers;
            if (ok && lane == __ffs(peers) - 1) {
                if (bg != 0u) atomicAdd(&s.rcnt[r][0], (uint32_t)__popc(bg));
                if (be != 0u) atomicAdd(&s.rcnt[r][1], (uint32_t)__popc(be));
            }
            if (r == rank && (gt || eq)) {
                const uint32_t e = x.y & 0xFFFFu;
                atomicOr(&(gt ? selbm : tiebm)[e >> 5], 1u << (e & 31));
            }
        }
        __syncthreads();
        if (tid == 0) {   // CTA r covers positions below CTA r + 1: ties go to the lower ranks first
            uint32_t tb = 0, ob = 0;
            for (uint32_t r = 0; r < C; ++r) {
                const uint32_t e = s.rcnt[r][1];
                const uint32_t take = tb < Rt ? min(e, Rt - tb) : 0u;
                if (r == rank) {
                    s.cbase[0] = take;
                    s.cbase[1] = ob;
                }
                tb += e;
                ob += s.peer[r][0] + s.rcnt[r][0] + take;
            }
        }
    } else {
        // ---- a threshold bin too large to gather (many equal or close keys):
        // two more radix passes over the keys in TMEM, each with a cluster-wide find
        uint32_t Rs = R;
        sweep([&](const uint32_t(&v)[32], int c0, int) {
            uint32_t m = 0;   // bit j: column c0 + j matches (independent compares, then a short loop)
#pragma unroll
            for (int j = 0; j < 32; ++j) m |= (uint32_t)(c0 + j < ntiles && (v[j] >> 21) == d1) << j;
            while (m != 0u) {
                const int j = __ffs(m) - 1;
                m &= m - 1u;
                atomicAdd(&hist2[(pick32(v, (uint32_t)j) >> 10) & (kNB2 - 1)], 1u);
            }
        });
        cl::sync();
        find_bin<kNB2>(s, hist2, 0, C, Rs, tid);
        const uint32_t p2 = (d1 << 11) | s.res[0];
        Rs -= s.res[1];
        sweep([&](const uint32_t(&v)[32], int c0, int) {
            uint32_t m = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) m |= (uint32_t)(c0 + j < ntiles && (v[j] >> 10) == p2) << j;
            while (m != 0u) {
                const int j = __ffs(m) - 1;
                m &= m - 1u;
                atomicAdd(&hist3[pick32(v, (uint32_t)j) & (kNB3 - 1)], 1u);
            }
        });
        cl::sync();
        find_bin<kNB3>(s, hist3, 0, C, Rs, tid);
        const uint32_t T = (p2 << 10) | s.res[0];
        Rs -= s.res[1];   // ties at T still to take, lowest positions first (1 <= Rs)
        // keys > T and == T: counted, and marked in position bitmaps (column c of lane l
        // is entry 128 c + 32 q + l: bitmap word 4 c + q, bit l)
        uint32_t gt = 0, eq = 0;
        sweep([&](const uint32_t(&v)[32], int c0, int q) {
            uint32_t mg = 0, me = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const bool valid = c0 + j < ntiles;
                mg |= (uint32_t)(valid && v[j] > T) << j;
                me |= (uint32_t)(valid && v[j] == T) << j;
            }
            gt += __popc(mg);
            eq += __popc(me);
            const uint32_t bit = 1u << lane;
            const int w0 = 4 * c0 + q;
            while (mg != 0u) {
                const int j = __ffs(mg) - 1;
                mg &= mg - 1u;
                atomicOr(&selbm[w0 + 4 * j], bit);
            }
            while (me != 0u) {
                const int j = __ffs(me) - 1;
                me &= me - 1u;
                atomicOr(&tiebm[w0 + 4 * j], bit);
            }
        });
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xFFFFFFFFu, gt, o);
            eq += __shfl_xor_sync(0xFFFFFFFFu, eq, o);
        }
        if (lane == 0) {
            s.wcnt[warp][0] = gt;
            s.wcnt[warp][1] = eq;
        }
        tc::tc_fence_before();
        __syncthreads();
        if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);   // no TMEM reads past this point
        if (tid == 0) {
            uint32_t g = 0, e = 0;
            for (int w = 0; w < kSwW; ++w) {
                g += s.wcnt[w][0];
                e += s.wcnt[w][1];
            }
            s.pub2[0] = g;
            s.pub2[1] = e;
        }
        cl::sync();                               // every CTA's counts are published
        if (warp == 0) {
            uint32_t g = 0, e = 0;
            if ((uint32_t)lane < C) {
                const uint2 x = cl::ld_v2(cl::map_rank(tc::smem_u32(s.pub2), (uint32_t)lane));
                g = x.x;
                e = x.y;
            }
            const uint32_t tb = warp_incl_scan(e, lane) - e;             // ties in lower-ranked CTAs
            const uint32_t take = tb < Rs ? min(e, Rs - tb) : 0u;
            const uint32_t ob = warp_incl_scan(g + take, lane) - (g + take);
            const uint32_t my_take = __shfl_sync(0xFFFFFFFFu, take, (int)rank);
            const uint32_t my_ob = __shfl_sync(0xFFFFFFFFu, ob, (int)rank);
            if (lane == 0) {
                s.cbase[0] = my_take;
                s.cbase[1] = my_ob;
            }
        }
    }
    __syncthreads();
    // take the lowest-positioned `quota` ties: thread t owns bitmap words kWPT t .. kWPT t + kWPT - 1
    const uint32_t quota = s.cbase[0];
    uint32_t tw[kWPT] = {}, nt = 0;
    if (tid < kSel) {
#pragma unroll
        for (int j = 0; j < kWPT; ++j) {
            tw[j] = tiebm[kWPT * tid + j];
            nt += __popc(tw[j]);
        }
    }
    uint32_t total;
    uint32_t tpre = block_scan_excl(s, nt, tid, &total);
    uint32_t sw[kWPT] = {}, ns = 0;
    if (tid < kSel) {
#pragma unroll
        for (int j = 0; j < kWPT; ++j) {
            uint32_t m = tw[j], keep = 0;
            while (m != 0u && tpre < quota) {
                const uint32_t low = m & (0u - m);
                keep |= low;
                m ^= low;
                ++tpre;
            }
            sw[j] = selbm[kWPT * tid + j] | keep;
            ns += __popc(sw[j]);
        }
    }
    uint32_t o = s.cbase[1] + block_scan_excl(s, ns, tid, &total);
    if (tid < kSel) {
#pragma unroll
        for (int j = 0; j < kWPT; ++j) {
            uint32_t m = sw[j];
            while (m != 0u) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                if (o < (uint32_t)k) {
                    const int item = lo + 32 * (kWPT * tid + j) + bit;
                    out[o] = MODE == 2 ? __ldg(pool + item / kBlk) * kBlk + item % kBlk : item;
                }
                ++o;
            }
        }
    }
    if (rank == 0)
        for (int i = (int)K1 + tid; i < k; i += kThreads) out[i] = -1;
    cl::sync();                                   // no CTA leaves while the cluster may read it
}

int smem_bytes() { return (int)sizeof(ClSmem) + 1024; }

DeviceOnce g_attr;
bool g_nonportable[kMaxDevices];

// Shared-memory size and (where allowed) 16-CTA clusters of both modes, once per device.
bool set_attributes() {
    return g_attr.run([] {
        cudaError_t e =
            cudaFuncSetAttribute(index_cluster_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(index_cluster_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(index_cluster_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(index_cluster_kernel<0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem_bytes());
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return e;
        }
        const int d = current_device();
        g_nonportable[d] =
            cudaFuncSetAttribute(index_cluster_kernel<0>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess &&
            cudaFuncSetAttribute(index_cluster_kernel<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess &&
            cudaFuncSetAttribute(index_cluster_kernel<2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess &&
            cudaFuncSetAttribute(index_cluster_kernel<0, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess;
        if (!g_nonportable[d]) (void)cudaGetLastError();
        return cudaSuccess;
    }) == cudaSuccess;
}

bool nonportable() {
    const int d = current_device();
    return d >= 0 && d < kMaxDevices && g_nonportable[d];
}

struct ClusterOcc {
    int n[17];
};
DeviceValue<ClusterOcc> g_occ;

// Clusters of C CTAs that can be resident at once on the current device (0 if refused);
// both modes have the same block and shared-memory size and one CTA per SM.
int max_active_clusters(int C) {
    const ClusterOcc occ = g_occ.get(
        [] {
            ClusterOcc o{};
            for (int c = 1; c <= (nonportable() ? 16 : 8); c <<= 1) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3(c, 1);
                cfg.blockDim = dim3(kThreads);
                cfg.dynamicSmemBytes = smem_bytes();
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = c;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                if (cudaOccupancyMaxActiveClusters(&o.n[c], index_cluster_kernel<0>, &cfg) != cudaSuccess) {
                    (void)cudaGetLastError();
                    o.n[c] = 0;
                }
            }
            return o;
        },
        ClusterOcc{});
    return occ.n[C];
}

}  // namespace

namespace {
// Largest cluster whose CTAs each hold at most `tiles` tiles of `items` items per query.
int cluster_size_for(const SelectParams& p, int64_t items, int tiles = kMaxTiles) {
    const int bq = p.B * p.Q;
    if (bq <= 0 || !set_attributes()) return 0;
    const int sms = device_sm_count();
    for (int C = nonportable() ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > sms) continue;
        const int64_t chunk = ((items + C - 1) / C + kTile - 1) / kTile * kTile;
        if (chunk > (int64_t)tiles * kTile) return 0;   // a smaller cluster only lengthens the chunk
        if (max_active_clusters(C) >= bq) return C;
    }
    return 0;
}
}  // namespace

int index_cluster_size(const SelectParams& p, bool* keys_in_ws) {
    if (keys_in_ws) *keys_in_ws = false;
    const int C = cluster_size_for(p, p.cap);
    if (C > 0 || !p.keys || !keys_in_ws) return C;
    const int Cg = cluster_size_for(p, p.cap, kMaxTilesG);   // the keys in the workspace
    *keys_in_ws = Cg > 0;
    return Cg;
}

cudaError_t launch_index_cluster(SelectParams& p, int C, bool keys_in_ws, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    if (keys_in_ws)
        return launch_ex(index_cluster_kernel<0, true>, dim3(C, p.B * p.Q), dim3(kThreads), smem_bytes(), st, C, p);
    return launch_ex(index_cluster_kernel<0>, dim3(C, p.B * p.Q), dim3(kThreads), smem_bytes(), st, C, p);
}

size_t cluster_keys_bytes(int B, int Q, int64_t cap) {
    const int64_t bq = (int64_t)B * Q;
    if (bq < 1 || bq * 16 > kSplitSMs) return 0;                       // one 16-CTA cluster per query
    if (cap <= 16ll * kMaxTiles * kTile || cap > 16ll * kMaxTilesG * kTile) return 0;
    return ((size_t)(bq * cap * 4) + 255) & ~(size_t)255;
}

int pool_build_cluster_size(const SelectParams& p) { return cluster_size_for(p, p.nb_cap); }

int pool_topk_cluster_size(const SelectParams& p) { return cluster_size_for(p, (int64_t)p.P * kBlk); }

cudaError_t launch_pool_topk_cluster(SelectParams& p, int C, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    return launch_ex(index_cluster_kernel<2>, dim3(C, p.B * p.Q), dim3(kThreads), smem_bytes(), st, C, p);
}

cudaError_t launch_pool_build_cluster(SelectParams& p, int C, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    return launch_ex(index_cluster_kernel<1>, dim3(C, p.B * p.Q), dim3(kThreads), smem_bytes(), st, C, p);
}

}  // namespace csa2
