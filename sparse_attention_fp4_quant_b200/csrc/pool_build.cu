// pool_build.cu -- csa2_pool_build for many queries: one CTA per query, an
// exact radix select over the query's block maxima.
//
// The hierarchical indexer ([Blog] "分层稀疏索引器") keeps, per query, the P
// blocks of 8 entries whose block maximum (the largest index score of the
// block's visible entries) is highest, listed in ascending block order; equal
// maxima go to the lower block.  The order key of a block is the monotone
// uint32 image of its maximum, and the select is a plain radix select on it:
//
//   1. one read of the maxima counts the keys' top 11 bits: the bin d1 of the
//      K-th largest key (K = min(P, visible blocks));
//   2. a read counting bits 20..10 of the keys in bin d1: the bin d2;
//   3. a read counting bits 9..0 of the keys in (d1, d2): the exact threshold
//      key T and the number of keys equal to T to take;
//   4. a read marking every key above T in one position bitmap and every key
//      equal to T in another; the lowest-positioned ties are taken, and two
//      prefix scans over the bitmap words write the blocks in ascending order.
//
// Each read moves the query's maxima from L2 (the index kernel wrote them just
// before) with every load of a batch in flight; no candidate buffer is ever
// compacted, and no sort is needed.  Used when one CTA per query fills the GPU
// (the streaming per-share select compacts its buffer every few thousand
// offers); decode-sized query counts take the cluster select.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {
namespace {

constexpr int kBT = 256;                 // threads of a CTA
constexpr int kMaxBlocks = 131072;       // blocks a query may have on this path
constexpr int kWords = kMaxBlocks / 32;  // bitmap words
constexpr int kWPT = kWords / kBT;       // bitmap words per thread
constexpr int kNB1 = 2048, kNB2 = 2048, kNB3 = 1024;
constexpr int kBatch = 8;                // float4 loads of a thread in flight together

struct BuildSmem {
    uint32_t h1[kNB1];
    uint32_t h2[kNB2];
    uint32_t h3[kNB3];
    uint32_t sel[kWords];   // blocks above T (and, after the tie step, the ties taken)
    uint32_t tie[kWords];   // blocks equal to T
    uint32_t wsum[kBT / 32];
    uint32_t res[2];
};

__device__ __forceinline__ void red_add_shared(uint32_t* a, uint32_t v) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(a)), "r"(v) : "memory");
}

// Exclusive prefix of v over the CTA's threads in order; *total = the sum.
__device__ __forceinline__ uint32_t scan_excl(BuildSmem& s, uint32_t v, int tid, uint32_t* total) {
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s.wsum[warp] = inc;
    __syncthreads();
    uint32_t pre = inc - v, tot = 0;
#pragma unroll
    for (int w = 0; w < kBT / 32; ++w) {
        if (w < warp) pre += s.wsum[w];
        tot += s.wsum[w];
    }
    *total = tot;
    __syncthreads();
    return pre;
}

// The bin b of an NB-bin histogram that holds the R-th largest key (1 <= R <= total):
// keys above b < R <= keys above b + count of b.  Leaves (b, keys above b) in s.res.
template <int NB>
__device__ __forceinline__ void find_bin(BuildSmem& s, const uint32_t* hist, uint32_t R, int tid) {
    constexpr int PER = NB / kBT;   // bins per thread, the highest on thread 0
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

// f(j, key) for every block j < nblk, the loads of kBatch float4 per thread in flight together.
template <class F>
__device__ __forceinline__ void for_each_key(const float* bm, int nblk, int tid, F&& f) {
    const int n4 = (nblk + 3) >> 2;
    const float4* b4 = reinterpret_cast<const float4*>(bm);
    for (int base = 0; base < n4; base += kBatch * kBT) {
        float4 v[kBatch];
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
            const int c = base + r * kBT + tid;
            v[r] = c < n4 ? __ldcg(b4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
            const int c = base + r * kBT + tid;
            if (c >= n4) break;
            const float x[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (4 * c + q < nblk) f(4 * c + q, score_key(x[q]));
        }
    }
}

__global__ void __launch_bounds__(kBT) pool_build_kernel(SelectParams p) {
    pdl_enter();
    extern __shared__ __align__(16) uint8_t build_smem[];
    BuildSmem& s = *reinterpret_cast<BuildSmem*>(build_smem);
    const int tid = threadIdx.x;
    const int64_t bq = blockIdx.x;
    const int b = (int)(bq / p.Q);
    const int P = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    int nblk = (nvis + kBlk - 1) / kBlk;
    if (nblk > p.nb_cap) nblk = (int)p.nb_cap;
    int32_t* out = p.out + bq * P;
    const float* bm = p.blockmax + bq * p.nb_cap;
    if (nblk <= P) {   // every visible block, in order
        for (int i = tid; i < P; i += kBT) out[i] = i < nblk ? i : -1;
        return;
    }
    for (int i = tid; i < kNB1 + kNB2 + kNB3 + 2 * kWords; i += kBT) s.h1[i] = 0u;   // the histograms, both bitmaps
    __syncthreads();

    // 1. top 11 bits
    for_each_key(bm, nblk, tid, [&](int, uint32_t key) { red_add_shared(&s.h1[key >> 21], 1u); });
    __syncthreads();
    find_bin<kNB1>(s, s.h1, (uint32_t)P, tid);
    const uint32_t d1 = s.res[0];
    const uint32_t R2 = (uint32_t)P - s.res[1];   // keys still to take from bin d1 (>= 1)
    // 2. bits 20..10 of bin d1
    for_each_key(bm, nblk, tid, [&](int, uint32_t key) {
        if ((key >> 21) == d1) red_add_shared(&s.h2[(key >> 10) & (kNB2 - 1)], 1u);
    });
    __syncthreads();
    find_bin<kNB2>(s, s.h2, R2, tid);
    const uint32_t p2 = (d1 << 11) | s.res[0];
    const uint32_t R3 = R2 - s.res[1];
    // 3. bits 9..0 of (d1, d2): the threshold key
    for_each_key(bm, nblk, tid, [&](int, uint32_t key) {
        if ((key >> 10) == p2) red_add_shared(&s.h3[key & (kNB3 - 1)], 1u);
    });
    __syncthreads();
    find_bin<kNB3>(s, s.h3, R3, tid);
    const uint32_t T = (p2 << 10) | s.res[0];
    const uint32_t Rt = R3 - s.res[1];   // keys equal to T to take, the lowest blocks first (>= 1)
    // 4. mark
    for_each_key(bm, nblk, tid, [&](int j, uint32_t key) {
        if (key > T) atomicOr(&s.sel[j >> 5], 1u << (j & 31));
        else if (key == T) atomicOr(&s.tie[j >> 5], 1u << (j & 31));
    });
    __syncthreads();

    // the Rt lowest ties, then every selected block in ascending order: thread t owns
    // bitmap words [kWPT t, kWPT t + kWPT)
    uint32_t tw[kWPT], nt = 0;
#pragma unroll
    for (int j = 0; j < kWPT; ++j) {
        tw[j] = s.tie[kWPT * tid + j];
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
        sw[j] = s.sel[kWPT * tid + j] | keep;
        ns += __popc(sw[j]);
    }
    uint32_t o = scan_excl(s, ns, tid, &total);
#pragma unroll
    for (int j = 0; j < kWPT; ++j) {
        uint32_t m = sw[j];
        while (m != 0u) {
            const int bit = __ffs(m) - 1;
            m &= m - 1u;
            if (o < (uint32_t)P) out[o] = 32 * (kWPT * tid + j) + bit;
            ++o;
        }
    }
}

DeviceOnce g_build_attr;

}  // namespace

bool pool_build_radix_ok(const SelectParams& p) {
    return p.nb_cap <= kMaxBlocks && (((uintptr_t)p.blockmax) & 15u) == 0 && p.nb_cap % 4 == 0;
}

cudaError_t launch_pool_build_radix(SelectParams& p, cudaStream_t st) {
    const int smem = (int)sizeof(BuildSmem);
    cudaError_t e = g_build_attr.run(
        [&] { return cudaFuncSetAttribute(pool_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
    if (e != cudaSuccess) return e;
    return launch_ex(pool_build_kernel, dim3((unsigned)(p.B * p.Q)), dim3(kBT), smem, st, 0, p);
}

}  // namespace csa2
