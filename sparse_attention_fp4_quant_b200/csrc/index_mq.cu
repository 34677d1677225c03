// index_mq.cu -- csa2_index_topk for many queries per batch row (prefill
// chunks): the indexer keys are scored once for 8 queries at a time, then one
// CTA per query selects its Top-K.
//
// Scoring (mq_score_kernel, one CTA per 8 consecutive queries of a batch row
// and share of its entry range (shares when the groups alone leave SMs idle,
// their histograms added in the workspace); 16 epilogue warps, two queries each, so that four warps share each SM
// sub-partition and hide each other's latency).  The block-scaled FP4 MMA of index_pipe.cuh with B = 8 block-diagonal
// query operands side by side (N = 128: column 16 g + 4 h + b holds query g's
// head h codes of block b only), so every key tile crosses shared memory once
// for 8 queries and each accumulator column is still one exact block product
// (without the key's scale, which the epilogue applies).  The epilogue forms
// each (query, entry) score in the defined fixed order, counts its order key's
// top 11 bits into the query's 2,048-bin histogram and stores the key's top 16
// bits ([query][entry] u16 in the workspace); block maxima when asked.
//
// Selection (mq_select_kernel, one CTA per query).  From the histogram, the
// bin d1 of the K-th key; one read of the stored prefixes marks every entry of
// a higher bin in a position bitmap and lists the entries of bin d1; their
// exact keys are recomputed on CUDA cores (score_cc.cuh: the same defined
// score) and two radix passes over them give the threshold T.  The selection
// is every key above T plus the lowest-positioned keys equal to T, written in
// ascending position order.  A threshold bin larger than the list is narrowed by
// a second read to the sub-bin of the prefix's next 5 bits (counted in the first
// read) that holds the K-th key; one still too large (many equal or close keys)
// is resolved by passes that re-score its entries.
#include "index_pipe.cuh"
#include "score_cc.cuh"

namespace csa2 {
namespace {

using namespace pipe;

constexpr int kG = 8;                         // queries per scoring CTA
constexpr int kN = 16 * kG;                   // MMA N
constexpr int kMqRing = 4;                    // shared-memory stages (4 tiles each)
constexpr int kAccT = 3;                      // accumulator tiles in TMEM
constexpr uint32_t kMqCols = 512;             // TMEM columns allocated
constexpr uint32_t kColSA = kAccT * kN;       // unit scales of A
constexpr uint32_t kColSB = kColSA + 4;       // the queries' scales
static_assert(kColSB + 4 <= kMqCols, "TMEM columns");
constexpr uint32_t kIdescN = tc::idesc_mxf4nvf4(128, kN);
constexpr int kEpiW = 16;                     // epilogue warps: four per TMEM lane quarter
constexpr int kQPW = kG * 4 / kEpiW;          // queries per epilogue warp
constexpr int kMqEpi = 32 * kEpiW;
constexpr int kMqThreads = 64 + kMqEpi;       // warp 0 copies, warp 1 MMA, the rest epilogue
static_assert(kQPW * kEpiW == 4 * kG, "every (lane quarter, query) pair has one warp");
constexpr int kNB1 = 2048;                    // top-11-bit histogram bins

struct MqSmem {
    static constexpr int kStages = kMqRing;
    uint8_t A[kMqRing][kTPS][kTile * 32];     // code tiles, the cache's MMA operand image
    uint8_t SF[kMqRing][kTPS][kTile * 4];     // their scales, row-major
    uint8_t Bq[kN * 32];                      // 8 block-diagonal queries, no swizzle, K-major
    uint8_t SFB[512];                         // their scales, TMEM-copy layout (row n at 16 (n % 32) + 4 (n / 32))
    uint8_t SFA[512];                         // unit scales (E4M3 1.0)
    uint32_t hist[kG][kNB1];
    uint64_t full[kMqRing], empty[kMqRing], accfull[kAccT], accempty[kAccT], done;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kMqThreads, 1) mq_score_kernel(SelectParams p, uint16_t* prefix, uint32_t* hist_out) {
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MqSmem& s = *reinterpret_cast<MqSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int q0 = blockIdx.x * kG;
    const int share = blockIdx.z, S = gridDim.z;
    const int ng = min(kG, p.Q - q0);          // queries of this CTA (the rest of B is zero)
    const int64_t bq0 = (int64_t)b * p.Q + q0;
    const int64_t row_base = (int64_t)b * p.cap;
    int nmax = 0;
    for (int g = 0; g < ng; ++g) nmax = max(nmax, n_visible(p.q_pos[bq0 + g], p.n_entries[b], p.m, p.cap));
    // this share's tiles [t_lo, t_lo + ntiles) of the group's range, whole stages
    const int ntiles_all = (nmax + kTile - 1) / kTile;
    const int chunk = ((ntiles_all + S - 1) / S + kTPS - 1) / kTPS * kTPS;
    const int t_lo = min(ntiles_all, share * chunk);
    const int ntiles = min(ntiles_all, t_lo + chunk) - t_lo;
    const int nstages = (ntiles + kTPS - 1) / kTPS;
    const int lo = t_lo * kTile;               // first entry of the share
    int32_t* status = p.status;

    if (tid == 0) {
        for (int i = 0; i < kMqRing; ++i) {
            tc::mbar_init(&s.full[i], 1);
            tc::mbar_init(&s.empty[i], 1 + kEpiW);   // MMA commit + each epilogue warp (scales read)
        }
        for (int i = 0; i < kAccT; ++i) {
            tc::mbar_init(&s.accfull[i], 1);
            tc::mbar_init(&s.accempty[i], kMqEpi);
        }
        tc::mbar_init(&s.done, 1);
        s.abort_flag = 0;
        tc::fence_mbar_init();
    }
    for (int i = tid; i < kG * kNB1; i += kMqThreads) (&s.hist[0][0])[i] = 0u;
    if (warp == 1) {   // TMEM and the query operand
        tc::tmem_alloc(&s.tmem_base, kMqCols);
        for (int i = lane; i < kN * 32; i += 32) s.Bq[i] = 0;
        for (int i = lane; i < 512; i += 32) {
            s.SFB[i] = 0;
            s.SFA[i] = 0x38;   // E4M3 1.0
        }
        __syncwarp();
        for (int n = lane; n < 16 * ng; n += 32) {
            const int g = n >> 4, h = n & 3, blk = (n >> 2) & 3;   // column 16 g + 4 blk + h
            const uint8_t* q = p.q + (bq0 + g) * 128;
            const uint8_t* qs = p.q_sc + (bq0 + g) * 16;
            uint8_t* row = s.Bq + (n >> 3) * 256 + (blk >> 1) * 128 + (n & 7) * 16 + 8 * (blk & 1);
#pragma unroll
            for (int j = 0; j < 8; ++j) row[j] = q[32 * h + 8 * blk + j];
#pragma unroll
            for (int j = 0; j < 4; ++j) s.SFB[16 * (n & 31) + 4 * (n >> 5) + j] = qs[4 * h + j];
        }
        tc::fence_proxy_async_smem();
    }
    __syncthreads();
    const uint32_t tbase = s.tmem_base;

    if (warp == 0) {
        producer_dense(s, p.ik, p.ik_sc, row_base, lo, ntiles, nstages, status, lane);
    } else if (warp == 1) {
        if (lane == 0) {
            tc::tc_fence_after();
            tc::tmem_cp_32x128_x4(tbase + kColSA, tc::smem_desc(tc::smem_u32(s.SFA), 16, 128, tc::kLayoutNone));
            tc::tmem_cp_32x128_x4(tbase + kColSB, tc::smem_desc(tc::smem_u32(s.SFB), 16, 128, tc::kLayoutNone));
            const uint64_t bdesc = tc::smem_desc(tc::smem_u32(s.Bq), 128, 256, tc::kLayoutNone);
            int u = 0;   // tiles issued
            bool stop = false;
            for (int t = 0; t < nstages && !stop; ++t) {
                const int slot = t % kMqRing;
                if (!tc::mbar_wait_spin(&s.full[slot], (uint32_t)(t / kMqRing) & 1u)) {
                    raise_abort(s, status);
                    break;
                }
                const int ntl = min(kTPS, ntiles - t * kTPS);
                for (int i = 0; i < ntl; ++i, ++u) {
                    const int a = u % kAccT;
                    if (!tc::mbar_wait_spin(&s.accempty[a], ((uint32_t)(u / kAccT) & 1u) ^ 1u)) {
                        raise_abort(s, status);
                        stop = true;
                        break;
                    }
                    if (aborted(s)) {
                        stop = true;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t adesc = tc::smem_desc(tc::smem_u32(s.A[slot][i]), 128, 256, tc::kLayoutNone);
                    tc::mma_mxf4nvf4(tbase + (uint32_t)(a * kN), adesc, bdesc, kIdescN, 0u, tbase + kColSA,
                                     tbase + kColSB);
                    tc::tc_commit(&s.accfull[a]);
                }
                tc::tc_commit(&s.empty[slot]);
            }
            tc::tc_commit(&s.done);
            if (!tc::mbar_wait(&s.done, 0)) raise_abort(s, status);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may read
        const int gb = kQPW * ((warp - 2) >> 2);      // queries gb .. gb + kQPW - 1
        const int row = 32 * quarter + lane;
        const uint32_t lanes = (uint32_t)(32 * quarter) << 16;
        uint64_t w01[kQPW], w23[kQPW];
        int nv[kQPW];
#pragma unroll
        for (int j = 0; j < kQPW; ++j) {
            const int g = gb + j;
            nv[j] = g < ng ? n_visible(p.q_pos[bq0 + g], p.n_entries[b], p.m, p.cap) : 0;
            float wq[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) wq[h] = g < ng ? __ldg(p.w + (bq0 + g) * 4 + h) : 0.0f;
            w01[j] = f2pack(wq[0], wq[1]);
            w23[j] = f2pack(wq[2], wq[3]);
        }
        bool dead = false;
        int u = 0;
        for (int t = 0; t < nstages; ++t) {
            const int ntl = min(kTPS, ntiles - t * kTPS);
            for (int i = 0; i < ntl; ++i, ++u) {
                const int a = u % kAccT;
                if (!dead && __any_sync(0xFFFFFFFFu, aborted(s))) dead = true;
                if (!dead && !__all_sync(0xFFFFFFFFu, tc::mbar_wait_spin(&s.accfull[a], (uint32_t)(u / kAccT) & 1u))) {
                    if (lane == 0) raise_abort(s, status);
                    dead = true;
                }
                if (dead) continue;
                tc::tc_fence_after();
                uint32_t v[kQPW][16];
#pragma unroll
                for (int j = 0; j < kQPW; ++j)
                    tc::tmem_ld_32x32b_x16(tbase + lanes + (uint32_t)(a * kN + 16 * (gb + j)), v[j]);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                tc::mbar_arrive(&s.accempty[a]);
                if (i == 0 && !__all_sync(0xFFFFFFFFu, stage_landed(s, t))) {   // the stage's scales
                    if (lane == 0) raise_abort(s, status);
                    dead = true;
                    continue;
                }
                const KeyScales ks = key_scales(stage_scales(s, t % kMqRing, i, row));   // shared by the queries
                if (i == ntl - 1) release_stage(s, t, lane);
                const int e = lo + u * kTile + row;
#pragma unroll
                for (int j = 0; j < kQPW; ++j) {
                    const int g = gb + j;
                    if (g >= ng) break;   // warp-uniform
                    const bool valid = e < nv[j];
                    const float score = valid ? score_of(v[j], ks, w01[j], w23[j]) : -INFINITY;
                    const uint32_t key = score_key(score);
                    if (valid) {
                        atomicAdd(&s.hist[g][key >> 21], 1u);
                        prefix[(bq0 + g) * p.cap + e] = (uint16_t)(key >> 16);
                    }
                    if (p.blockmax) {
                        const float mx = block_max8(score, lane);
                        if ((lane & (kBlk - 1)) == 0 && valid) p.blockmax[(bq0 + g) * p.nb_cap + (e >> 3)] = mx;
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tbase, kMqCols);
    if (aborted(s)) return;
    if (S == 1) {
        for (int i = tid; i < ng * kNB1; i += kMqThreads) hist_out[bq0 * kNB1 + i] = (&s.hist[0][0])[i];
    } else {   // the shares add into the zeroed workspace histograms
        for (int i = tid; i < ng * kNB1; i += kMqThreads) {
            const uint32_t c = (&s.hist[0][0])[i];
            if (c) atomicAdd(&hist_out[bq0 * kNB1 + i], c);
        }
    }
    if (p.blockmax && share == 0) {   // blocks with no visible position
        for (int g = 0; g < ng; ++g) {
            const int nvg = n_visible(p.q_pos[bq0 + g], p.n_entries[b], p.m, p.cap);
            for (int64_t j = (nvg + kBlk - 1) / kBlk + tid; j < p.nb_cap; j += kMqThreads)
                p.blockmax[(bq0 + g) * p.nb_cap + j] = -INFINITY;
        }
    }
}

// ---------------------------------------------------------------------------- selection
constexpr int kMaxVis = 262144;               // entries a query may see on this path
constexpr int kSmallVis = 65536;              // the smaller selector (two CTAs per SM)
constexpr int kCandMax = 4096;                // threshold-bin entries listed
constexpr int kNB2 = 2048, kNB3 = 1024;
constexpr int kPB = 8;                        // prefix loads of a thread in flight together

template <int MAXVIS>
struct SelSmem {
    // threads of a selecting CTA: the large selector runs alone on its SM (its bitmaps),
    // with twice the threads to keep as many prefix loads in flight
    static constexpr int kST = MAXVIS > kSmallVis ? 512 : 256;
    static constexpr int kSW = MAXVIS / 32;   // bitmap words
    static constexpr int kWPT = kSW / kST;    // bitmap words per thread
    uint32_t hist[kNB1];
    uint32_t hist2[kNB2];
    uint32_t hist3[kNB3];
    uint32_t selbm[kSW];                      // entries above T (and the ties taken)
    uint32_t tiebm[kSW];                      // entries equal to T
    uint32_t h16[kST / 32][32];               // bin d1's entries by the prefix's low 5 bits, per warp
    int32_t cpos[kCandMax];                   // the threshold bin's entries
    uint32_t ckey[kCandMax];                  // and their exact keys
    uint32_t wsum[kST / 32];
    uint32_t res[2];
    uint32_t ncand;
};

__device__ __forceinline__ uint32_t warp_incl_scan_u(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Exclusive prefix of v over the CTA's threads in order; *total = the sum.
template <class SelSmem>
__device__ __forceinline__ uint32_t scan_excl(SelSmem& s, uint32_t v, int tid, uint32_t* total) {
    constexpr int kST = SelSmem::kST;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t inc = warp_incl_scan_u(v, lane);
    if (lane == 31) s.wsum[warp] = inc;
    __syncthreads();
    uint32_t pre = inc - v, tot = 0;
#pragma unroll
    for (int w = 0; w < kST / 32; ++w) {
        if (w < warp) pre += s.wsum[w];
        tot += s.wsum[w];
    }
    *total = tot;
    __syncthreads();
    return pre;
}

// The bin b of the NB-bin histogram holding the R-th largest key (R >= 1):
// keys above b < R <= keys above b + count of b.  Leaves (b, keys above b) in
// s.res.  All threads call it.
template <int NB, class SelSmem>
__device__ __forceinline__ void find_bin_local(SelSmem& s, const uint32_t* hist, uint32_t R, int tid) {
    constexpr int kST = SelSmem::kST;
    constexpr int PER = NB / kST;             // bins per thread, the highest on thread 0
    const int b0 = NB - PER * (tid + 1);
    uint32_t h[PER], sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        h[j] = hist[b0 + j];
        sum += h[j];
    }
    uint32_t total;
    uint32_t above = scan_excl(s, sum, tid, &total);
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
    __syncthreads();
}

template <int MAXVIS>
__global__ void __launch_bounds__(SelSmem<MAXVIS>::kST, MAXVIS > kSmallVis ? 1 : 3)
    mq_select_kernel(SelectParams p, const uint16_t* prefix, const uint32_t* hist_in) {
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    using SelSmem = csa2::SelSmem<MAXVIS>;
    constexpr int kSW = SelSmem::kSW, kWPT = SelSmem::kWPT, kST = SelSmem::kST;
    SelSmem& s = *reinterpret_cast<SelSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t bq = blockIdx.x;
    const int b = (int)(bq / p.Q);
    const int k = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const uint32_t K1 = (uint32_t)min(k, nvis);
    int32_t* out = p.out + bq * k;
    if (K1 == 0) {
        for (int i = tid; i < k; i += kST) out[i] = -1;
        return;
    }
    for (int i = tid; i < kNB1; i += kST) s.hist[i] = hist_in[bq * kNB1 + i];
    for (int i = tid; i < kNB2 + kNB3 + 2 * kSW + kST; i += kST) s.hist2[i] = 0u;   // hist2, hist3, both bitmaps, h16
    if (tid == 0) s.ncand = 0;
    __syncthreads();
    find_bin_local<kNB1>(s, s.hist, K1, tid);
    const uint32_t d1 = s.res[0];
    uint32_t R = K1 - s.res[1];   // keys to take from bin d1 (1 <= R)

    // reads of the prefixes, kPB loads of a thread in flight together (a uniform trip count,
    // for the warp scans): classify(prefix) = 1 puts the entry into the bitmap (above the
    // threshold bin), 2 lists it (in the bin), 0 neither
    const uint16_t* pre = prefix + bq * p.cap;
    const int n8 = (nvis + 7) >> 3;
    auto sweep = [&](auto classify) {
        for (int base = 0; base < n8; base += kPB * kST) {
            uint4 xs[kPB];
#pragma unroll
            for (int r = 0; r < kPB; ++r) {
                const int c = base + r * kST + tid;
                xs[r] = c < n8 ? __ldcg(reinterpret_cast<const uint4*>(pre) + c) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int r = 0; r < kPB; ++r) {
                const int e0 = 8 * (base + r * kST + tid);
                const uint32_t w[4] = {xs[r].x, xs[r].y, xs[r].z, xs[r].w};
                uint32_t ma = 0, mc = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t p16 = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
                    const int c = e0 + j < nvis ? classify(p16) : 0;
                    ma |= (uint32_t)(c == 1) << j;
                    mc |= (uint32_t)(c == 2) << j;
                }
                if (ma) atomicOr(&s.selbm[e0 >> 5], ma << (e0 & 31));
                const uint32_t n = __popc(mc);
                const uint32_t incl = warp_incl_scan_u(n, lane);
                uint32_t cbase = 0;
                if (lane == 31 && incl) cbase = atomicAdd(&s.ncand, incl);
                cbase = __shfl_sync(0xFFFFFFFFu, cbase, 31) + incl - n;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t slot = cbase + (uint32_t)__popc(mc & ((1u << j) - 1u));
                    if (((mc >> j) & 1u) && slot < (uint32_t)kCandMax) s.cpos[slot] = e0 + j;
                }
            }
        }
    };
    // first read: bins above d1 into the bitmap, bin d1 listed and counted by the prefix's
    // low 5 bits
    sweep([&](uint32_t p16) -> int {
        const uint32_t bin = p16 >> 5;
        if (bin == d1) {
            atomicAdd(&s.h16[tid >> 5][p16 & 31u], 1u);
            return 2;
        }
        return bin > d1 ? 1 : 0;
    });
    __syncthreads();
    uint32_t nc = s.ncand;
    uint32_t pmask = 0xFFE0u, pval = d1 << 5;   // the prefixes of the threshold bin
    if (nc > (uint32_t)kCandMax) {
        // too many to list (a far tail of close keys): a second read keeps the sub-bin of the
        // prefix's low 5 bits that holds the R-th key, marks the sub-bins above it
        if (tid == 0) {
            uint32_t above = 0;
            int bb = 31;
            for (; bb > 0; --bb) {
                uint32_t c = 0;
                for (int w = 0; w < kST / 32; ++w) c += s.h16[w][bb];
                if (above + c >= R) break;
                above += c;
            }
            s.res[0] = (uint32_t)bb;
            s.res[1] = above;
            s.ncand = 0;
        }
        __syncthreads();
        const uint32_t d1b = s.res[0];
        R -= s.res[1];
        pmask = 0xFFFFu;
        pval = (d1 << 5) | d1b;
        sweep([&](uint32_t p16) -> int {
            if ((p16 >> 5) != d1) return 0;
            const uint32_t lo5 = p16 & 31u;
            return lo5 > d1b ? 1 : (lo5 == d1b ? 2 : 0);
        });
        __syncthreads();
        nc = s.ncand;
    }
    QReg Rq;
    load_query(Rq, p.q + bq * 128, p.q_sc + bq * 16, p.w + bq * 4);
    const uint8_t* ik = p.ik + (int64_t)b * p.cap * 32;
    const uint8_t* iks = p.ik_sc + (int64_t)b * p.cap * 4;
    uint32_t T, Rt;
    if (nc <= (uint32_t)kCandMax) {
        // exact keys of the listed entries, then two radix passes over them
        for (uint32_t i = tid; i < nc; i += kST) {
            const uint32_t key = score_key(entry_score_at(Rq, ik, iks, s.cpos[i]));
            s.ckey[i] = key;
            atomicAdd(&s.hist2[(key >> 10) & (kNB2 - 1)], 1u);
        }
        __syncthreads();
        find_bin_local<kNB2>(s, s.hist2, R, tid);
        const uint32_t p2 = (d1 << 11) | s.res[0];
        const uint32_t R3 = R - s.res[1];
        for (uint32_t i = tid; i < nc; i += kST) {
            const uint32_t key = s.ckey[i];
            if ((key >> 10) == p2) atomicAdd(&s.hist3[key & (kNB3 - 1)], 1u);
        }
        __syncthreads();
        find_bin_local<kNB3>(s, s.hist3, R3, tid);
        T = (p2 << 10) | s.res[0];
        Rt = R3 - s.res[1];
        for (uint32_t i = tid; i < nc; i += kST) {
            const uint32_t key = s.ckey[i];
            const int e = s.cpos[i];
            if (key > T) atomicOr(&s.selbm[e >> 5], 1u << (e & 31));
            else if (key == T) atomicOr(&s.tiebm[e >> 5], 1u << (e & 31));
        }
    } else {
        // still too many (many equal or close keys): passes that re-score the bin's entries
        for (int e = tid; e < nvis; e += kST) {
            if (((uint32_t)pre[e] & pmask) != pval) continue;
            const uint32_t key = score_key(entry_score_at(Rq, ik, iks, e));
            atomicAdd(&s.hist2[(key >> 10) & (kNB2 - 1)], 1u);
        }
        __syncthreads();
        find_bin_local<kNB2>(s, s.hist2, R, tid);
        const uint32_t p2 = (d1 << 11) | s.res[0];
        const uint32_t R3 = R - s.res[1];
        for (int e = tid; e < nvis; e += kST) {
            if (((uint32_t)pre[e] & pmask) != pval) continue;
            const uint32_t key = score_key(entry_score_at(Rq, ik, iks, e));
            if ((key >> 10) == p2) atomicAdd(&s.hist3[key & (kNB3 - 1)], 1u);
        }
        __syncthreads();
        find_bin_local<kNB3>(s, s.hist3, R3, tid);
        T = (p2 << 10) | s.res[0];
        Rt = R3 - s.res[1];
        for (int e = tid; e < nvis; e += kST) {
            if (((uint32_t)pre[e] & pmask) != pval) continue;
            const uint32_t key = score_key(entry_score_at(Rq, ik, iks, e));
            if (key > T) atomicOr(&s.selbm[e >> 5], 1u << (e & 31));
            else if (key == T) atomicOr(&s.tiebm[e >> 5], 1u << (e & 31));
        }
    }
    __syncthreads();

    // the lowest-positioned Rt ties, then every selected position in ascending order:
    // thread t owns bitmap words [kWPT t, kWPT t + kWPT)
    uint32_t tw[kWPT], nt = 0;
#pragma unroll
    for (int j = 0; j < kWPT; ++j) {
        tw[j] = s.tiebm[kWPT * tid + j];
        nt += __popc(tw[j]);
    }
    uint32_t total;
    uint32_t tpre = scan_excl(s, nt, tid, &total);
    uint32_t sw[kWPT], ns = 0;
#pragma unroll
    for (int j = 0; j < kWPT; ++j) {
        uint32_t m = tw[j], keep = 0;
        while (m != 0u && tpre < Rt) {
            const uint32_t low = m & (0u - m);
            keep |= low;
            m ^= low;
            ++tpre;
        }
        sw[j] = s.selbm[kWPT * tid + j] | keep;
        ns += __popc(sw[j]);
    }
    uint32_t o = scan_excl(s, ns, tid, &total);
#pragma unroll
    for (int j = 0; j < kWPT; ++j) {
        uint32_t m = sw[j];
        while (m != 0u) {
            const int bit = __ffs(m) - 1;
            m &= m - 1u;
            if (o < (uint32_t)k) out[o] = 32 * (kWPT * tid + j) + bit;
            ++o;
        }
    }
    for (int i = (int)K1 + tid; i < k; i += kST) out[i] = -1;
}

DeviceOnce g_mq_attr;

}  // namespace

bool index_mq_eligible(int B, int Q, int64_t cap) {
    return (int64_t)B * Q > kSplitSMs && Q >= kG && cap <= kMaxVis;
}

// Entry-range shares of the scoring (one CTA per SM): the count that minimises waves x
// tiles per CTA, each CTA also paying its set-up (TMEM, the query operands, the histogram
// flush: about kSetupTiles tiles' time).  A last wave that leaves most SMs idle costs
// as much as a full one.
static int mq_shares(int B, int Q, int64_t cap) {
    constexpr int64_t kSetupTiles = 8;
    const int dev_sms = device_sm_count();   // a grid choice only: the workspace does not depend on it
    const int64_t sms = dev_sms > 0 ? dev_sms : kSplitSMs;
    const int64_t groups = (int64_t)((Q + kG - 1) / kG) * B;
    const int64_t tiles = (cap + kTile - 1) / kTile;
    int best = 1;
    int64_t best_cost = -1;
    for (int S = 1; S <= 16; ++S) {
        const int64_t waves = (groups * S + sms - 1) / sms;
        const int64_t cost = waves * ((tiles + S - 1) / S + kSetupTiles);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = S;
        }
    }
    return best;
}

size_t index_mq_ws_bytes(int B, int Q, int64_t cap) {
    const size_t bq = (size_t)B * Q;
    return align256(bq * (size_t)cap * 2) + align256(bq * kNB1 * 4);
}

cudaError_t launch_index_mq(SelectParams& p, void* mq_ws, cudaStream_t st) {
    const size_t bq = (size_t)p.B * p.Q;
    uint16_t* prefix = (uint16_t*)mq_ws;
    uint32_t* hist = (uint32_t*)((char*)mq_ws + align256(bq * (size_t)p.cap * 2));
    const int smem1 = (int)sizeof(MqSmem) + 1024;
    const int smem_small = (int)sizeof(SelSmem<kSmallVis>), smem_large = (int)sizeof(SelSmem<kMaxVis>);
    cudaError_t e = g_mq_attr.run([&] {
        cudaError_t r = cudaFuncSetAttribute(mq_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(mq_select_kernel<kSmallVis>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_small);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(mq_select_kernel<kMaxVis>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_large);
        return r;
    });
    if (e != cudaSuccess) return e;
    const int S = mq_shares(p.B, p.Q, p.cap);
    if (S > 1) {   // the shares add their histograms
        e = cudaMemsetAsync(hist, 0, bq * kNB1 * sizeof(uint32_t), st);
        if (e != cudaSuccess) return e;
    }
    e = launch_ex(mq_score_kernel, dim3((p.Q + kG - 1) / kG, p.B, S), dim3(kMqThreads), smem1, st, 0, p, prefix, hist);
    if (e != cudaSuccess) return e;
    if (p.cap <= kSmallVis)
        return launch_ex(mq_select_kernel<kSmallVis>, dim3((unsigned)bq), dim3(SelSmem<kSmallVis>::kST), smem_small, st, 0, p,
                         (const uint16_t*)prefix, (const uint32_t*)hist);
    return launch_ex(mq_select_kernel<kMaxVis>, dim3((unsigned)bq), dim3(SelSmem<kMaxVis>::kST), smem_large, st, 0, p,
                     (const uint16_t*)prefix, (const uint32_t*)hist);
}

}  // namespace csa2
