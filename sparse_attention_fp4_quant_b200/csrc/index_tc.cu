// index_tc.cu -- FP4 index scoring on the tcgen05 tensor cores (index_pipe.cuh),
// fused with an exact Top-K (Full layers: csa2_index_topk for shapes the cluster
// and many-query kernels do not take; Reindex layers: csa2_pool_topk, and
// csa2_layer_step's Reindex for many queries).
//
// One CTA = one share of one query's candidates.  Warps 0 and 1 run the
// scoring pipeline; warps 2-9 finish the scores and select (named barrier 1).
// Modes 0 and 1 (dense range, pool) stream the scores through a threshold
// filter into a buffer that an exact radix select compacts.  Modes 2 (an
// ascending pool, one CTA per query) and 3 (dense range) keep every order key
// in the workspace and count its top 11 bits while scoring, then offer only the
// items at or above the bin that holds the k-th key to the exact Top-K: no
// per-stage barrier, and typically no compaction before the last.  With several
// shares the last CTA of a query merges their best k through a histogram of all
// their keys.
#include "index_pipe.cuh"
#include "topk.cuh"

namespace csa2 {
namespace {

using namespace pipe;

constexpr int kEpiT0 = 64, kEpiN = 256;   // 8 epilogue warps: two per TMEM lane quarter
constexpr int kThreads = kEpiT0 + kEpiN;
constexpr int kTPG = kTPS / 2;   // tiles of a stage per epilogue warp group

constexpr int kRing = 4;   // shared-memory stages in flight
constexpr int kHistBits = 11, kHistBins = 1 << kHistBits;   // mode 2: bins of the keys' top bits

template <int CAP>
struct TcSmem {
    Pipe<kRing> pipe;
    int32_t stage_blk[kRing][kTPS][kPoolPerTile];   // pool modes: each stage's block ids (-1 = none)
    int last;
    uint32_t sel_bin, sel_count;    // mode 2: the bin of the k-th key, entries in it or above
    uint32_t warp_sum[kEpiN / 32];  // mode 2: per-warp histogram sums
    union {
        typename TopK<kEpiN, CAP, 1, kEpiT0>::Smem topk;
        uint32_t hist[kHistBins];   // mode 2, while scoring (the Top-K takes the space afterwards)
    };
};
static_assert(sizeof(uint32_t) * kHistBins <= sizeof(typename TopK<kEpiN, 2048, 1, kEpiT0>::Smem), "histogram fits");

// One shared-memory add per entry (bin < 0: none).  Lanes that hit the same bin are
// serialised by the hardware; grouping them first (match.any) cost more than it saved
// on pool scores.
__device__ __forceinline__ void hist_add(uint32_t hist_base, int bin) {
    if (bin >= 0) shm::red_add(hist_base + 4u * (uint32_t)bin, 1u);
}

// OR of `v` over the epilogue warps, through named barrier 1 (every epilogue
// thread gets the same answer, so they all leave or all stay).
__device__ __forceinline__ bool epilogue_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kEpiN)
        : "memory");
    return r != 0;
}

// Epilogue warps: from the histogram of the keys' top bits in s.hist, the bin that holds
// the k-th largest key (bins scanned from the top; bin 0 when there are at most k keys)
// into s.sel_bin, and the number of keys in it or above into s.sel_count.  After it no
// thread reads the histogram, whose space the Top-K may take.
template <int CAP>
__device__ __forceinline__ void threshold_bin(TcSmem<CAP>& s, int k, int lane, int warp) {
    using TKE = TopK<kEpiN, CAP, 1, kEpiT0>;
    const int et = (int)threadIdx.x - kEpiT0, ew = warp - kEpiT0 / 32;
    constexpr int kPer = kHistBins / kEpiN;   // bins per thread, highest first
    uint32_t c[kPer], tot = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        c[j] = s.hist[kHistBins - 1 - (kPer * et + j)];
        tot += c[j];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s.warp_sum[ew] = incl;
    TKE::sync();
    uint32_t before = incl - tot, total = 0;
#pragma unroll
    for (int w = 0; w < kEpiN / 32; ++w) {
        const uint32_t v = s.warp_sum[w];
        if (w < ew) before += v;
        total += v;
    }
    const uint32_t kk = (uint32_t)k;
    if (total <= kk) {
        if (et == 0) {
            s.sel_bin = 0;
            s.sel_count = total;
        }
    } else if (before < kk && kk <= before + tot) {
        uint32_t run = before;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            if (run + c[j] >= kk) {
                s.sel_bin = (uint32_t)(kHistBins - 1 - (kPer * et + j));
                s.sel_count = run + c[j];
                break;
            }
            run += c[j];
        }
    }
    TKE::sync();
}

// Epilogue warps, modes 2 and 3, after scoring: the bin d that holds the k-th largest
// key, then one read of the keys offers each item i in bin d or above to the exact Top-K
// as position pos0 + i (mode 3: the share's entries from pos0; mode 2: the entry index of
// an ascending pool, which orders like the position).  When those items fit the buffer
// nothing is compacted before the final select; otherwise the buffer makes room as it
// fills, which is exact too, only slower.
template <int CAP>
__device__ __forceinline__ void keys_select(TcSmem<CAP>& s, TopK<kEpiN, CAP, 1, kEpiT0>& tk, const uint32_t* qkeys,
                                            int n_items, int pos0, int k, int lane, int warp) {
    const int et = (int)threadIdx.x - kEpiT0;
    threshold_bin<CAP>(s, k, lane, warp);
    const uint32_t d = s.sel_bin;
    const bool fast = s.sel_count <= (uint32_t)CAP;
    tk.init();
    constexpr int kBatch = 8;   // rounds of 4 keys a thread whose loads are in flight together
    for (int base = 0; base < n_items; base += kBatch * 4 * kEpiN) {   // uniform trip count
        uint4 kv[kBatch];
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
            const int i0 = base + r * 4 * kEpiN + 4 * et;   // n_items is a multiple of 4
            kv[r] = i0 < n_items ? __ldcg(reinterpret_cast<const uint4*>(qkeys + i0)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
            const int i0 = base + r * 4 * kEpiN + 4 * et;
            const uint32_t key4[4] = {kv[r].x, kv[r].y, kv[r].z, kv[r].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (!fast) tk.make_room(k, kEpiN);
                const bool take = key4[q] != 0u && (key4[q] >> (32 - kHistBits)) >= d;
                tk.offer(take, key4[q], pos0 + i0 + q);
            }
        }
    }
    tk.finish(k);
}

// The last CTA of a query, once every share has written its best k (padded to k with key
// 0, which no finite score maps to): the histogram of all S k keys' top 11 bits gives the
// bin of the k-th best, and only the keys in it or above are offered to the exact Top-K.
// Offering all of them compacted the buffer every few hundred offers.  Every batch of
// loads is in flight together.
template <int CAP>
__device__ __forceinline__ void merge_shares(TcSmem<CAP>& s, TopK<kEpiN, CAP, 1, kEpiT0>& tk, const uint32_t* keys,
                                             const int32_t* poss, int total, int k, int lane, int warp) {
    using TKE = TopK<kEpiN, CAP, 1, kEpiT0>;
    constexpr int kB = 16;
    const int et = (int)threadIdx.x - kEpiT0;
    const uint32_t hist_base = tc::smem_u32(&s.hist[0]);
    for (int i = et; i < kHistBins; i += kEpiN) shm::st(hist_base + 4u * (uint32_t)i, 0u);
    TKE::sync();
    for (int base = 0; base < total; base += kB * kEpiN) {
        uint32_t kv[kB];
#pragma unroll
        for (int r = 0; r < kB; ++r) {
            const int g = base + r * kEpiN + et;
            kv[r] = g < total ? __ldcg(keys + g) : 0u;
        }
#pragma unroll
        for (int r = 0; r < kB; ++r)
            if (kv[r] != 0u) shm::red_add(hist_base + 4u * (kv[r] >> (32 - kHistBits)), 1u);
    }
    TKE::sync();
    threshold_bin<CAP>(s, k, lane, warp);
    const uint32_t d = s.sel_bin;
    const bool fast = s.sel_count <= (uint32_t)CAP;
    tk.init();
    for (int base = 0; base < total; base += kB * kEpiN) {   // uniform trip count
        uint32_t kv[kB];
        int32_t pv[kB];
#pragma unroll
        for (int r = 0; r < kB; ++r) {
            const int g = base + r * kEpiN + et;
            kv[r] = g < total ? __ldcg(keys + g) : 0u;
        }
#pragma unroll
        for (int r = 0; r < kB; ++r) {
            const int g = base + r * kEpiN + et;
            const bool take = kv[r] != 0u && (kv[r] >> (32 - kHistBits)) >= d;
            pv[r] = take ? __ldcg(poss + g) : 0;
            if (!take) kv[r] = 0u;
        }
#pragma unroll
        for (int r = 0; r < kB; ++r) {
            if (!fast) tk.make_room(k, kEpiN);
            tk.offer(kv[r] != 0u, kv[r], pv[r]);
        }
    }
    tk.finish(k);
}

// MODE 0 = dense range (index Top-K), 1 = pool blocks (pool Top-K), 2 = pool blocks of an
// ascending pool with the keys kept in the workspace (one share per query), 3 = dense range
// with the keys kept in the workspace ([B Q][cap])
template <int MODE, int CAP>
__global__ void __launch_bounds__(kThreads, 2)
    index_tc_kernel(SelectParams p) {
    pdl_enter();
    using TKE = TopK<kEpiN, CAP, 1, kEpiT0>;
    using TcSmem = csa2::TcSmem<CAP>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align by pointer arithmetic on the shared array (an integer round trip would
    // hide the address space and turn every shared access into a generic one)
    TcSmem& s = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bq = blockIdx.y, share = blockIdx.x, S = gridDim.x;
    const int b = bq / p.Q;
    const int k = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const int64_t row_base = (int64_t)b * p.cap;

    constexpr bool kDense = MODE == 0 || MODE == 3, kKeys = MODE >= 2;
    // this share's candidates: dense = entries [lo, hi); pool = pool slots [lo, hi)
    int lo, hi, ntiles;
    if (kDense) {
        int chunk = (((nvis + S - 1) / S) + (kTPS * kTile - 1)) / (kTPS * kTile) * (kTPS * kTile);
        lo = min(nvis, share * chunk);
        hi = min(nvis, lo + chunk);
        ntiles = (hi - lo + kTile - 1) / kTile;
    } else {
        int chunk = (((p.P + S - 1) / S) + (kTPS * kPoolPerTile - 1)) / (kTPS * kPoolPerTile) * (kTPS * kPoolPerTile);
        lo = min(p.P, share * chunk);
        hi = min(p.P, lo + chunk);
        ntiles = (hi - lo + kPoolPerTile - 1) / kPoolPerTile;
    }
    const int nstages = (ntiles + kTPS - 1) / kTPS;
    const int32_t* pool = kDense ? nullptr : p.pool + (int64_t)bq * p.P;
    // this share's order keys, one per (tile, row): mode 2 item i = slot * 8 + row of the
    // query's pool; mode 3 item i = entry lo + i of the query's [cap] row
    uint32_t* qkeys = MODE == 2 ? p.keys + (int64_t)bq * ntiles * kTile
                                : (MODE == 3 ? p.keys + (int64_t)bq * p.cap + lo : nullptr);

    if (tid == 0) init_barriers(s.pipe, kEpiN, kDense ? 1u : kPoolLanes);
    if (warp == 1) setup_query(s.pipe, p.q + (int64_t)bq * 128, p.q_sc + (int64_t)bq * 16, lane, kPipeCols);
    __syncthreads();
    const uint32_t tbase = s.pipe.tmem_base;
    int32_t* status = p.status;

    if (warp == 0) {
        if constexpr (kDense)
            producer_dense(s.pipe, p.ik, p.ik_sc, row_base, lo, ntiles, nstages, status, lane, p.test_starve != 0);
        else
            producer_pool_async(s.pipe, p.ik, p.ik_sc, row_base, lo, hi, ntiles, nstages, pool, nvis, &s.stage_blk[0][0][0],
                                status, lane);
    } else if (warp == 1) {
        mma_issuer(s.pipe, ntiles, nstages, status, lane);
    } else {
        // ------------------------------------------------------------ epilogue
        TKE tk(s.topk);
        const uint32_t hist_base = tc::smem_u32(&s.hist[0]);
        if constexpr (kKeys) {
            for (int i = tid - kEpiT0; i < kHistBins; i += kEpiN) shm::st(hist_base + 4u * (uint32_t)i, 0u);
            TKE::sync();
        } else {
            tk.init();
        }
        const int quarter = warp & 3;             // TMEM lanes this warp may read
        const int group = (warp - 2) >> 2;        // tiles 2*group, 2*group+1 of each stage
        const int row = quarter * 32 + lane;
        const uint64_t w01 = f2pack(__ldg(p.w + (int64_t)bq * 4 + 0), __ldg(p.w + (int64_t)bq * 4 + 1));
        const uint64_t w23 = f2pack(__ldg(p.w + (int64_t)bq * 4 + 2), __ldg(p.w + (int64_t)bq * 4 + 3));
        float* bm = (kDense && p.blockmax) ? p.blockmax + (int64_t)bq * p.nb_cap : nullptr;
        bool stop = false;
        for (int t = 0; t < nstages && !stop; ++t) {
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            const bool ok = __all_sync(0xFFFFFFFFu, tc::mbar_wait_spin(&s.pipe.accfull[a], aph));  // warp-uniform
            if (!ok && lane == 0) raise_abort(s.pipe, status);
            tc::tc_fence_after();
            uint32_t v[kTPG][16];
#pragma unroll
            for (int j = 0; j < kTPG; ++j) {
                const int i = kTPG * group + j;
                if (ok) {
                    tc::tmem_ld_32x32b_x16(tbase + ((uint32_t)(quarter * 32) << 16) + kColAcc + (uint32_t)(a * kTPS + i) * 16,
                                           v[j]);
                }
            }
            if (ok) tc::tmem_ld_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(&s.pipe.accempty[a]);
            const bool landed = ok && __all_sync(0xFFFFFFFFu, stage_landed(s.pipe, t));   // warp-uniform
            if (ok && !landed && lane == 0) raise_abort(s.pipe, status);
            uint32_t skw[kTPG];
            int sblk[kTPG];   // pool mode: the row's block id (read before the stage is released)
#pragma unroll
            for (int j = 0; j < kTPG; ++j) {
                skw[j] = landed ? stage_scales(s.pipe, t % kRing, kTPG * group + j, row) : 0u;
                sblk[j] = (!kDense && landed) ? s.stage_blk[t % kRing][kTPG * group + j][row >> 3] : -1;
            }
            if (landed) release_stage(s.pipe, t, lane);
            if constexpr (kKeys) {
                if (!landed) {   // warp-uniform; the warps meet again after the loop
                    stop = true;
                    break;
                }
#pragma unroll
                for (int j = 0; j < kTPG; ++j) {
                    const int g = t * kTPS + kTPG * group + j;
                    if (g >= ntiles) break;   // warp-uniform
                    int64_t e = -1;
                    if (MODE == 3) {
                        const int ee = lo + g * kTile + row;
                        if (ee < hi) e = ee;
                    } else if (sblk[j] >= 0) {
                        const int64_t ee = (int64_t)sblk[j] * kBlk + (row & 7);
                        if (ee < nvis) e = ee;
                    }
                    const bool valid = e >= 0;
                    const float score = valid ? score_of(v[j], key_scales(skw[j]), w01, w23) : -INFINITY;
                    if (MODE == 3 && bm) {
                        const float m8 = block_max8(score, lane);
                        if ((lane & 7) == 0 && valid) bm[e >> 3] = m8;
                    }
                    // key 0 marks "no entry": a finite score's key is never 0
                    const uint32_t key = valid ? score_key(score) : 0u;
                    __stcg(qkeys + g * kTile + row, key);
                    hist_add(hist_base, valid ? (int)(key >> (32 - kHistBits)) : -1);
                }
                continue;
            }
            if (epilogue_any(aborted(s.pipe))) {   // also the barrier that orders the previous offers
                stop = true;
                break;
            }
            if (tk.count() > CAP - kTPS * kTile) tk.compact(k);
            const auto th = tk.threshold();
#pragma unroll
            for (int j = 0; j < kTPG; ++j) {
                const int g = t * kTPS + kTPG * group + j;
                int64_t e = -1;
                if (g < ntiles) {
                    if (MODE == 0) {
                        const int ee = lo + g * kTile + row;
                        if (ee < hi) e = ee;
                    } else if (sblk[j] >= 0) {   // the producer wrote -1 past the share and for unseen blocks
                        const int64_t ee = (int64_t)sblk[j] * kBlk + (row & 7);
                        if (ee < nvis) e = ee;
                    }
                }
                const bool valid = e >= 0;
                const float score = valid ? score_of(v[j], key_scales(skw[j]), w01, w23) : -INFINITY;
                if (MODE == 0 && bm && g < ntiles) {
                    const float m8 = block_max8(score, lane);
                    if ((lane & 7) == 0 && valid) bm[e >> 3] = m8;
                }
                tk.offer(th, valid, score_key(valid ? score : 0.0f), (int32_t)(valid ? e : 0));
            }
        }
        if (!stop && kDense && bm) {  // blocks with no visible position
            const int64_t jb = (nvis + kBlk - 1) / kBlk;
            const int64_t rest = p.nb_cap - jb;
            if (rest > 0) {
                const int64_t cs = (rest + S - 1) / S;
                const int64_t j0 = jb + (int64_t)share * cs, j1 = min(p.nb_cap, j0 + cs);
                for (int64_t j = j0 + (tid - kEpiT0); j < j1; j += kEpiN) bm[j] = -INFINITY;
            }
        }
        if constexpr (kKeys) {
            stop = epilogue_any(stop || aborted(s.pipe));
            if (!stop) keys_select<CAP>(s, tk, qkeys, ntiles * kTile, MODE == 3 ? lo : 0, k, lane, warp);
        } else {
            if (!stop) tk.finish(k);
        }
    }
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tbase, kPipeCols);
    if (warp < 2 || aborted(s.pipe)) return;

    // ---------------------------------------------------------------- output
    TKE tk(s.topk);
    const int et = tid - kEpiT0;
    if (S > 1) {
        const int cnt = tk.count();
        const int64_t off = ((int64_t)bq * S + share) * k;
        for (int i = et; i < k; i += kEpiN) {   // padded to k with key 0 (no entry)
            p.cand_key[off + i] = i < cnt ? tk.key_at(i) : 0u;
            if (i < cnt) p.cand_pos[off + i] = tk.pos_at(i);
        }
        if (et == 0) p.cand_cnt[(int64_t)bq * S + share] = cnt;
        __threadfence();
        TKE::sync();
        if (et == 0) s.last = (atomicAdd(&p.counters[bq], 1) == S - 1);
        TKE::sync();
        if (!s.last) return;
        __threadfence();
        merge_shares<CAP>(s, tk, p.cand_key + (int64_t)bq * S * k, p.cand_pos + (int64_t)bq * S * k, S * k, k, lane, warp);
        if (et == 0) p.counters[bq] = 0;
    }
    const int cnt = tk.count();
    tk.sort_positions(cnt);
    if constexpr (MODE == 2) {   // entry index -> position (ascending pool: the same order)
        for (int i = et; i < k; i += kEpiN) {
            int32_t r = -1;
            if (i < cnt) {
                const int32_t it = tk.pos_at(i);
                r = __ldg(pool + (it >> 3)) * kBlk + (it & 7);
            }
            p.out[(int64_t)bq * k + i] = r;
        }
    } else {
        for (int i = et; i < k; i += kEpiN) p.out[(int64_t)bq * k + i] = i < cnt ? tk.pos_at(i) : -1;
    }
}

// two CTAs per SM for the usual k (the k > 1536 variant runs one)
static_assert(sizeof(TcSmem<2048>) + 1024 <= 113 * 1024, "shared memory of two CTAs per SM");

}  // namespace

bool index_tc_supported(const SelectParams& p) {
    return (((uintptr_t)p.ik) & 15u) == 0 && (((uintptr_t)p.ik_sc) & 15u) == 0 && p.cap % kTile == 0 &&
           (int64_t)p.B * p.cap < (int64_t(1) << 31);
}

size_t pool_keys_bytes(int B, int Q, int P) { return (size_t)B * Q * (size_t)((P + kPoolPerTile - 1) / kPoolPerTile) * kTile * 4; }

template <int MODE, int CAP>
cudaError_t launch_tc(SelectParams& p, int S, cudaStream_t st) {
    const int smem = (int)sizeof(TcSmem<CAP>) + 1024;
    static DeviceOnce attr;
    cudaError_t e = attr.run(
        [&] { return cudaFuncSetAttribute(index_tc_kernel<MODE, CAP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
    if (e != cudaSuccess) return e;
    dim3 grid(S, p.B * p.Q);
    return launch_ex(index_tc_kernel<MODE, CAP>, grid, dim3(kThreads), smem, st, 0, p);
}

cudaError_t launch_index_tc(int op, SelectParams& p, int S, cudaStream_t st) {
    // with the keys in the workspace: a pool search (the caller vouches for an ascending
    // pool, one share per query) or a dense index
    const int mode = (op == CSA2_OP_POOL_TOPK) ? ((p.keys && S == 1) ? 2 : 1) : (p.keys ? 3 : 0);
    // the buffer must hold k survivors plus one stage of offers
    if (p.k <= 2048 - kTPS * kTile) {
        switch (mode) {
            case 0: return launch_tc<0, 2048>(p, S, st);
            case 1: return launch_tc<1, 2048>(p, S, st);
            case 2: return launch_tc<2, 2048>(p, S, st);
            default: return launch_tc<3, 2048>(p, S, st);
        }
    }
    switch (mode) {
        case 0: return launch_tc<0, 4096>(p, S, st);
        case 1: return launch_tc<1, 4096>(p, S, st);
        case 2: return launch_tc<2, 4096>(p, S, st);
        default: return launch_tc<3, 4096>(p, S, st);
    }
}

}  // namespace csa2
