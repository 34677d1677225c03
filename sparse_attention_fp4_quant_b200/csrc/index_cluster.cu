// index_cluster.cu -- csa2_index_topk for decode-sized query counts: one
// thread-block cluster of C CTAs per query, an exact Top-K by radix select
// over the whole cluster, no merge and no sort.
//
// Each CTA scores a contiguous 1/C of the query's visible entries with the
// tcgen05 pipeline of index_pipe.cuh (permuted tiles: TMEM row m of a tile is
// entry 4 (m % 32) + m / 32, so a stage is one TMA box per tile plus one bulk
// copy of its scales) and keeps every order key in shared memory (at most
// 32,768 per CTA, in TMEM-row order), while the epilogue counts the keys' top
// 11 bits into a 2,048-bin histogram.  The cluster then finds the K-th largest
// key T exactly in three radix passes (bits 31..21, 20..10, 9..0): each pass
// sums the CTAs' histograms through distributed shared memory and locates the
// bin holding the K-th key from the top.  After the first pass one ordered
// sweep over the CTA's keys copies every key at or above the first-pass bin
// (with its position) into a short per-warp list, which the later passes and
// the output read instead of the whole key array (a list that would overflow
// sends its CTA back to the whole array; the results are the same).  The
// selected set is every key above T plus the lowest-positioned keys equal to T
// (ties go to the lower position).  CTA r covers positions below those of CTA
// r + 1 and each warp a contiguous run of its CTA, so writing each run's
// survivors at a prefix-summed offset yields the positions in ascending order.
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

constexpr int kThreads = 320;              // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int kEpiN = 256;
constexpr int kTPG = kTPS / 2;             // tiles of a stage per epilogue warp group
constexpr int kMaxKeys = 32768;            // order keys one CTA keeps in shared memory
constexpr int kNB1 = 2048, kNB2 = 2048, kNB3 = 1024;   // radix digits: bits 31..21, 20..10, 9..0
constexpr int kSel = 256;                  // threads of the select phase (warps 0-7)
constexpr int kSelWarps = kSel / 32;
constexpr int kSegCap = 512;               // candidate list capacity per select warp
static_assert((kNB2 + kNB3) * 4 + kSelWarps * kSegCap * 8 <= (int)sizeof(Pipe::A), "select scratch fits the ring");

struct ClSmem {
    Pipe pipe;                              // its A ring holds hist2, hist3 and the candidate lists after scoring
    alignas(16) uint32_t hist1[kNB1];
    alignas(16) uint32_t keys[kMaxKeys];    // key of TMEM row m of tile g at g * 128 + m (0 past the CTA's range)
    float bmx[2][2][kTPG][kTile];           // block-max staging: [group][stage parity][tile][entry in tile]
    uint32_t wsum[kSelWarps];               // scan: per-warp totals
    uint32_t res[2];                        // scan: (bin, keys above the bin)
    uint32_t segn[kSelWarps];               // candidates found per select warp (may exceed kSegCap)
    uint32_t wgt[kSelWarps], weq[kSelWarps];   // per-warp counts of keys > T and == T
    alignas(8) uint32_t pub[2];             // this CTA's (> T, == T) counts, read by the cluster
    uint32_t wbase[kSelWarps][2];           // per-warp (tie rank, output offset) at the start of its run
};

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__device__ __forceinline__ uint32_t lanemask_lt(int lane) { return (1u << lane) - 1u; }

__device__ __forceinline__ void group_bar(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(2 + group) : "memory");
}

// Sum the NB-bin histogram `hist` over the cluster's CTAs and find the bin b
// holding the R-th largest key (R >= 1): keys above b < R <= keys above b +
// count of b.  Leaves (b, keys above b) in s.res.  All threads of the CTA call it.
template <int NB>
__device__ __forceinline__ void find_bin(ClSmem& s, const uint32_t* hist, uint32_t C, uint32_t R, int tid) {
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
        for (uint32_t r0 = 0; r0 < C; r0 += RG) {
            uint4 x[RG][NV];
#pragma unroll
            for (int g = 0; g < RG; ++g)
                if (r0 + g < C) {
                    const uint32_t ra = cl::map_rank(la, r0 + g);
#pragma unroll
                    for (int v = 0; v < NV; ++v) x[g][v] = cl::ld_v4(ra + 16u * v);
                }
#pragma unroll
            for (int g = 0; g < RG; ++g)
                if (r0 + g < C) {
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

__global__ void __launch_bounds__(kThreads, 1)
    index_cluster_kernel(SelectParams p, const __grid_constant__ CUtensorMap tmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    ClSmem& s = *reinterpret_cast<ClSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cl::rank(), C = cl::ctas();
    const int bq = blockIdx.y;
    const int b = bq / p.Q;
    const int k = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const int64_t row_base = (int64_t)b * p.cap;
    // this CTA's entries [lo, hi); the host keeps the chunk within kMaxKeys
    const int chunk = ((nvis + (int)C - 1) / (int)C + kTile - 1) / kTile * kTile;
    const int lo = min(nvis, (int)rank * chunk), hi = min(nvis, lo + chunk);
    const int ntiles = (hi - lo + kTile - 1) / kTile;
    const int nstages = (ntiles + kTPS - 1) / kTPS;
    const int npad = ntiles * kTile;
    int32_t* status = p.status;
    int32_t* out = p.out + (int64_t)bq * k;

    if (tid == 0) init_barriers(s.pipe, 1, kEpiN);
    if (warp == 1) setup_query(s.pipe, p.q + (int64_t)bq * 128, p.q_sc + (int64_t)bq * 16, lane);
    for (int i = tid; i < kNB1; i += kThreads) s.hist1[i] = 0;
    __syncthreads();
    const uint32_t tbase = s.pipe.tmem_base;

    if (warp == 0) {
        producer_perm(s.pipe, &tmap, p.ik_sc, row_base, lo, hi, ntiles, nstages, status, lane);
    } else if (warp == 1) {
        mma_issuer(s.pipe, ntiles, nstages, status, lane);
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;             // TMEM lanes this warp may read
        const int group = (warp - 2) >> 2;        // tiles 2*group, 2*group+1 of each stage
        const int m = quarter * 32 + lane;        // TMEM row
        const int eo = 4 * lane + quarter;        // its entry within the tile
        const float w0 = __ldg(p.w + (int64_t)bq * 4 + 0), w1 = __ldg(p.w + (int64_t)bq * 4 + 1);
        const float w2 = __ldg(p.w + (int64_t)bq * 4 + 2), w3 = __ldg(p.w + (int64_t)bq * 4 + 3);
        float* bm = p.blockmax ? p.blockmax + (int64_t)bq * p.nb_cap : nullptr;
        bool dead = false;   // this warp stopped after a failed wait (or another role's)
        for (int t = 0; t < nstages; ++t) {
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            if (!dead && __any_sync(0xFFFFFFFFu, aborted(s.pipe))) dead = true;
            if (!dead && !__all_sync(0xFFFFFFFFu, tc::mbar_wait(&s.pipe.accfull[a], aph))) {   // warp-uniform
                if (lane == 0) raise_abort(s.pipe, status);
                dead = true;
            }
            if (!dead) {
                tc::tc_fence_after();
                uint32_t v[kTPG][16];
#pragma unroll
                for (int j = 0; j < kTPG; ++j)
                    tc::tmem_ld_32x32b_x16(tbase + ((uint32_t)(quarter * 32) << 16) + kColAcc +
                                               (uint32_t)(a * kTPS + kTPG * group + j) * 16,
                                           v[j]);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                tc::mbar_arrive(&s.pipe.accempty[a]);
#pragma unroll
                for (int j = 0; j < kTPG; ++j) {
                    const int g = t * kTPS + kTPG * group + j;
                    if (g >= ntiles) continue;   // warp-uniform
                    const bool valid = lo + g * kTile + eo < hi;
                    const float score = valid ? score_of(v[j], w0, w1, w2, w3) : -INFINITY;
                    const uint32_t key = valid ? score_key(score) : 0u;
                    s.keys[g * kTile + m] = key;
                    if (valid) atomicAdd(&s.hist1[key >> 21], 1u);
                    if (bm) s.bmx[group][t & 1][j][eo] = score;
                }
            }
            if (bm) {
                // block maxima in position order: the first strictly larger score wins
                group_bar(group);
                if (!dead && warp == 2 + 4 * group) {   // one warp of the group
                    const int j = lane >> 4, c = lane & 15;
                    const int g = t * kTPS + kTPG * group + j;
                    const int e0 = lo + g * kTile + 8 * c;
                    if (g < ntiles && e0 < hi) {
                        const float* sc = &s.bmx[group][t & 1][j][8 * c];
                        float mx = sc[0];
                        for (int e = 1; e < kBlk && e0 + e < hi; ++e)
                            if (sc[e] > mx) mx = sc[e];
                        bm[e0 >> 3] = mx;
                    }
                }
            }
        }
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
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);

    // ---------------------------------------------------------------- select
    const uint32_t K1 = (uint32_t)min(k, nvis);
    if (K1 == 0) {   // the same for every CTA of the cluster: nothing visible
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    uint32_t* hist2 = reinterpret_cast<uint32_t*>(&s.pipe.A[0][0][0]);
    uint32_t* hist3 = hist2 + kNB2;
    uint2* seg = reinterpret_cast<uint2*>(hist3 + kNB3) + (warp < kSelWarps ? warp : 0) * kSegCap;
    for (int i = tid; i < kNB2 + kNB3; i += kThreads) hist2[i] = 0;
    // warp w < 8 owns keys [wlo, whi) of this CTA (whole tiles), in position order
    const int Lw = ((npad + kSelWarps - 1) / kSelWarps + kTile - 1) / kTile * kTile;
    const int wlo = min(npad, warp * Lw), whi = min(npad, wlo + Lw);

    cl::sync();                                   // every CTA's hist1 is complete
    find_bin<kNB1>(s, s.hist1, C, K1, tid);
    const uint32_t d1 = s.res[0];
    uint32_t R = K1 - s.res[1];

    // one ordered sweep: the candidates (first digit >= d1) into this warp's list,
    // the second-digit histogram of the keys whose first digit is d1
    if (warp < kSelWarps) {
        uint32_t n = 0;
        for (int base = wlo; base < whi; base += kTile) {
            uint32_t kk[4], c = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kk[j] = s.keys[base + 32 * j + lane];   // entry base + 4 lane + j
                const uint32_t d = kk[j] >> 21;
                if (d == d1) atomicAdd(&hist2[(kk[j] >> 10) & (kNB2 - 1)], 1u);
                c += (uint32_t)(d >= d1);
            }
            if (__ballot_sync(0xFFFFFFFFu, c != 0) == 0) continue;   // warp-uniform
            const uint32_t inc = warp_incl_scan(c, lane);
            uint32_t o = n + inc - c;
            n += __shfl_sync(0xFFFFFFFFu, inc, 31);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if ((kk[j] >> 21) >= d1) {
                    if (o < (uint32_t)kSegCap) seg[o] = make_uint2(kk[j], (uint32_t)(base + 4 * lane + j));
                    ++o;
                }
            }
        }
        if (lane == 0) s.segn[warp] = n;
    }
    cl::sync();
    find_bin<kNB2>(s, hist2, C, R, tid);
    const uint32_t p2 = (d1 << 11) | s.res[0];
    R -= s.res[1];
    bool whole = false;   // some list overflowed: this CTA reads its whole key array
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) whole |= s.segn[w] > (uint32_t)kSegCap;
    const uint32_t nseg = warp < kSelWarps ? min(s.segn[warp], (uint32_t)kSegCap) : 0u;

    if (whole) {
        for (int i = tid; i < npad; i += kThreads) {
            const uint32_t key = s.keys[i];
            if ((key >> 10) == p2) atomicAdd(&hist3[key & (kNB3 - 1)], 1u);
        }
    } else if (warp < kSelWarps) {
        for (uint32_t i = lane; i < nseg; i += 32) {
            const uint32_t key = seg[i].x;
            if ((key >> 10) == p2) atomicAdd(&hist3[key & (kNB3 - 1)], 1u);
        }
    }
    cl::sync();
    find_bin<kNB3>(s, hist3, C, R, tid);
    const uint32_t T = (p2 << 10) | s.res[0];
    R -= s.res[1];   // ties at T still to take, in position order (1 <= R)

    // ---------------------------------------------------------------- output
    if (warp < kSelWarps) {
        uint32_t gt = 0, eq = 0;
        if (whole) {
            for (int base = wlo; base < whi; base += kTile)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t key = s.keys[base + 32 * j + lane];
                    gt += (uint32_t)(key > T);
                    eq += (uint32_t)(key == T);
                }
        } else {
            for (uint32_t i = lane; i < nseg; i += 32) {
                const uint32_t key = seg[i].x;
                gt += (uint32_t)(key > T);
                eq += (uint32_t)(key == T);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xFFFFFFFFu, gt, o);
            eq += __shfl_xor_sync(0xFFFFFFFFu, eq, o);
        }
        if (lane == 0) {
            s.wgt[warp] = gt;
            s.weq[warp] = eq;
        }
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kSelWarps; ++w) {
            g += s.wgt[w];
            e += s.weq[w];
        }
        s.pub[0] = g;
        s.pub[1] = e;
    }
    cl::sync();                                   // every CTA's counts are published
    if (warp == 0) {
        uint32_t g = 0, e = 0;
        if ((uint32_t)lane < C) {
            const uint2 x = cl::ld_v2(cl::map_rank(tc::smem_u32(s.pub), (uint32_t)lane));
            g = x.x;
            e = x.y;
        }
        const uint32_t tb = warp_incl_scan(e, lane) - e;             // ties in lower-ranked CTAs
        const uint32_t take = tb < R ? min(e, R - tb) : 0u;
        const uint32_t ob = warp_incl_scan(g + take, lane) - (g + take);
        uint32_t t = __shfl_sync(0xFFFFFFFFu, tb, (int)rank), o = __shfl_sync(0xFFFFFFFFu, ob, (int)rank);
        if (lane == 0) {
            for (int w = 0; w < kSelWarps; ++w) {
                s.wbase[w][0] = t;
                s.wbase[w][1] = o;
                const uint32_t tw = t < R ? min(s.weq[w], R - t) : 0u;
                t += s.weq[w];
                o += s.wgt[w] + tw;
            }
        }
    }
    __syncthreads();
    if (warp < kSelWarps) {
        uint32_t tie = s.wbase[warp][0], ob = s.wbase[warp][1];
        if (whole) {
            for (int base = wlo; base < whi; base += kTile) {
                uint32_t kk[4];
                uint32_t ne = 0, any = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    kk[j] = s.keys[base + 32 * j + lane];   // entry base + 4 lane + j
                    ne += (uint32_t)(kk[j] == T);
                    any |= (uint32_t)(kk[j] >= T);
                }
                if (__ballot_sync(0xFFFFFFFFu, any) == 0) continue;   // warp-uniform
                const uint32_t ne_inc = warp_incl_scan(ne, lane);
                uint32_t tr = tie + ne_inc - ne;
                tie += __shfl_sync(0xFFFFFFFFu, ne_inc, 31);
                uint32_t sel = 0, ns = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (kk[j] > T) {
                        sel |= 1u << j;
                    } else if (kk[j] == T) {
                        if (tr < R) sel |= 1u << j;
                        ++tr;
                    }
                    ns += (sel >> j) & 1u;
                }
                const uint32_t ns_inc = warp_incl_scan(ns, lane);
                uint32_t o = ob + ns_inc - ns;
                ob += __shfl_sync(0xFFFFFFFFu, ns_inc, 31);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if ((sel >> j) & 1u) {
                        if (o < (uint32_t)k) out[o] = lo + base + 4 * lane + j;
                        ++o;
                    }
                }
            }
        } else {
            for (uint32_t i0 = 0; i0 < nseg; i0 += 32) {
                const uint32_t i = i0 + lane;
                const uint2 ce = i < nseg ? seg[i] : make_uint2(0u, 0u);
                const bool gt = i < nseg && ce.x > T, eq = i < nseg && ce.x == T;
                const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
                const uint32_t tr = tie + __popc(eqb & lanemask_lt(lane));
                tie += __popc(eqb);
                const bool sel = gt || (eq && tr < R);
                const uint32_t sb = __ballot_sync(0xFFFFFFFFu, sel);
                const uint32_t o = ob + __popc(sb & lanemask_lt(lane));
                ob += __popc(sb);
                if (sel && o < (uint32_t)k) out[o] = lo + (int)ce.y;
            }
        }
    }
    if (rank == 0)
        for (int i = (int)K1 + tid; i < k; i += kThreads) out[i] = -1;
    cl::sync();                                   // no CTA leaves while the cluster may read it
}

int g_max_active[17];
bool g_max_active_known[17];

// Clusters of C CTAs that can be resident at once (0 if the size is refused).
int max_active_clusters(int C, int bq, int smem) {
    if (g_max_active_known[C]) return g_max_active[C];
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, bq);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, index_cluster_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    g_max_active[C] = n;
    g_max_active_known[C] = true;
    return n;
}

int smem_bytes() { return (int)sizeof(ClSmem) + 1024; }

bool g_attr_done = false;
bool g_nonportable = false;

bool set_attributes() {
    if (g_attr_done) return true;
    if (cudaFuncSetAttribute(index_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes()) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    g_nonportable = cudaFuncSetAttribute(index_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                    cudaSuccess;
    if (!g_nonportable) (void)cudaGetLastError();
    g_attr_done = true;
    return true;
}

}  // namespace

int index_cluster_size(const SelectParams& p) {
    const int bq = p.B * p.Q;
    // permuted tiles: rows in groups of 4, 16-byte aligned scale rows
    if (bq <= 0 || (p.cap & 3) != 0 || (((uintptr_t)p.ik_sc) & 15u) != 0 || !set_attributes()) return 0;
    for (int C = g_nonportable ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > kNumSMs) continue;
        const int64_t chunk = ((p.cap + C - 1) / C + kTile - 1) / kTile * kTile;
        if (chunk > kMaxKeys) return 0;   // a smaller cluster only lengthens the chunk
        if (max_active_clusters(C, bq, smem_bytes()) >= bq) return C;
    }
    return 0;
}

cudaError_t launch_index_cluster(SelectParams& p, int C, cudaStream_t st) {
    CUtensorMap map;
    if (!pipe::encode_ik_map_perm(&map, p.ik, (int64_t)p.B * p.cap)) return cudaErrorInvalidValue;
    if (!set_attributes()) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, p.B * p.Q);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, index_cluster_kernel, p, map);
}

}  // namespace csa2
