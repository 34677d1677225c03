// topk.cuh -- exact block-wide Top-K selection in shared memory.
//
// Order: key descending, then position ascending (keys are the monotone uint32
// images of fp32 scores, so equal scores tie and the lower position wins).
// Candidates stream through a threshold filter into a buffer of CAP slots;
// when the buffer nears full, an exact radix select keeps the best k and the
// k-th best (key, pos) becomes the new admission threshold.  Offer order does
// not matter: the composite threshold admits a later candidate that ties the
// threshold score only if its position is lower.
//
// The NT participating threads are threads [T0, T0 + NT) of the CTA (whole
// warps).  BAR = 0 synchronises with __syncthreads (NT must be the block);
// BAR > 0 uses named barrier BAR for the NT threads only, so a warp-specialised
// kernel can run the selection in its consumer warps.
//
// All shared-memory traffic goes through explicit ld/st/atom/red.shared on
// 32-bit shared addresses: the engine is reached through a reference, and a
// generic address would route every access (atomics included) through the
// much slower generic path.
#pragma once
#include <stddef.h>

#include "common.cuh"

namespace csa2 {

template <int BAR, int NT>
__device__ __forceinline__ void group_sync() {
    if constexpr (BAR == 0) {
        __syncthreads();
    } else {
        asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
    }
}

namespace shm {
__device__ __forceinline__ uint32_t ld(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void st(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add(uint32_t a, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add(uint32_t a, uint32_t v) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void red_max_s32(uint32_t a, int32_t v) {
    asm volatile("red.shared.max.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
}  // namespace shm

template <int NT, int CAP, int BAR = 0, int T0 = 0>
struct TopK {
    static_assert(CAP % NT == 0, "CAP must be a multiple of the block size");

    // Two buffers: compact() reads the current one and writes the survivors to
    // the other, so it needs no register copy of the candidates (keeps the code
    // small; a fully unrolled register version thrashes the instruction cache).
    struct Smem {
        uint32_t key[2][CAP];
        int32_t pos[2][CAP];
        uint32_t hist[256];
        int cur;
        int count;
        int new_count;
        int has_thr;
        uint32_t thr_key;
        int32_t thr_pos;
        uint32_t sel_prefix;
        int sel_remaining;
        int sel_found;
        int32_t worst_pos;
    };

    uint32_t base;  // shared address of the Smem block

    __device__ explicit TopK(Smem& sm) : base((uint32_t)__cvta_generic_to_shared(&sm)) {}

    __device__ __forceinline__ uint32_t cur() const { return shm::ld(base + (uint32_t)offsetof(Smem, cur)); }
    __device__ __forceinline__ uint32_t a_key_of(uint32_t c) const { return base + (uint32_t)offsetof(Smem, key) + c * 4u * CAP; }
    __device__ __forceinline__ uint32_t a_pos_of(uint32_t c) const { return base + (uint32_t)offsetof(Smem, pos) + c * 4u * CAP; }
    __device__ __forceinline__ uint32_t a_key() const { return a_key_of(cur()); }
    __device__ __forceinline__ uint32_t a_pos() const { return a_pos_of(cur()); }
    __device__ __forceinline__ uint32_t a_hist() const { return base + (uint32_t)offsetof(Smem, hist); }
    __device__ __forceinline__ uint32_t a_(size_t off) const { return base + (uint32_t)off; }

    __device__ __forceinline__ static int ltid() { return (int)threadIdx.x - T0; }
    __device__ __forceinline__ static void sync() { group_sync<BAR, NT>(); }

    __device__ __forceinline__ int count() const { return (int)shm::ld(a_(offsetof(Smem, count))); }
    __device__ __forceinline__ uint32_t key_at(int i) const { return shm::ld(a_key() + 4u * (uint32_t)i); }
    __device__ __forceinline__ int32_t pos_at(int i) const { return (int32_t)shm::ld(a_pos() + 4u * (uint32_t)i); }

    __device__ __forceinline__ void init() {
        if (ltid() == 0) {
            shm::st(a_(offsetof(Smem, cur)), 0u);
            shm::st(a_(offsetof(Smem, count)), 0u);
            shm::st(a_(offsetof(Smem, has_thr)), 0u);
            shm::st(a_(offsetof(Smem, thr_key)), 0u);
            shm::st(a_(offsetof(Smem, thr_pos)), 0x7FFFFFFFu);
        }
        sync();
    }

    // The admission threshold; read once per batch of offers (it only changes in compact()).
    struct Thr {
        bool on;
        uint32_t key;
        int32_t pos;
    };
    __device__ __forceinline__ Thr threshold() const {
        Thr t;
        t.on = shm::ld(a_(offsetof(Smem, has_thr))) != 0u;
        t.key = shm::ld(a_(offsetof(Smem, thr_key)));
        t.pos = (int32_t)shm::ld(a_(offsetof(Smem, thr_pos)));
        return t;
    }

    // Warp-collective: every lane of the warp must call it (valid may be false).
    __device__ __forceinline__ void offer(const Thr& t, bool valid, uint32_t key, int32_t pos) {
        const bool take = valid && (!t.on || key > t.key || (key == t.key && pos < t.pos));
        const unsigned ball = __ballot_sync(0xFFFFFFFFu, take);
        if (ball == 0) return;
        const int lane = lane_id();
        const int leader = __ffs(ball) - 1;
        uint32_t slot0 = 0;
        if (lane == leader) slot0 = shm::atom_add(a_(offsetof(Smem, count)), (uint32_t)__popc(ball));
        slot0 = __shfl_sync(0xFFFFFFFFu, slot0, leader);
        if (take) {
            const uint32_t slot = slot0 + (uint32_t)__popc(ball & ((1u << lane) - 1u));
            shm::st(a_key() + 4u * slot, key);
            shm::st(a_pos() + 4u * slot, (uint32_t)pos);
        }
    }
    __device__ __forceinline__ void offer(bool valid, uint32_t key, int32_t pos) { offer(threshold(), valid, key, pos); }

    // Group-collective.  Guarantees room for `room` more offers.
    __device__ __forceinline__ void make_room(int k, int room) {
        sync();
        if (count() > CAP - room) compact(k);
    }

    // Group-collective.  After it, count <= k and the buffer holds the best k.
    __device__ __forceinline__ void finish(int k) {
        sync();
        if (count() > k) compact(k);
    }

    // Histogram update with one shared atomic per distinct bin per warp:
    // clustered keys (similar scores share their top bits) would otherwise
    // serialise on a single address.  Warp-collective; `bin` < 0 = no update.
    __device__ __forceinline__ void hist_add(int bin) {
        const unsigned act = __ballot_sync(0xFFFFFFFFu, bin >= 0);
        if (bin >= 0) {
            const unsigned peers = __match_any_sync(act, bin);
            if ((int)(__ffs(peers) - 1) == lane_id()) shm::red_add(a_hist() + 4u * (uint32_t)bin, (uint32_t)__popc(peers));
        }
    }

    // The first 32 participating threads scan the 256-bin histogram for the bin
    // holding the `remaining`-th element, from high to low bins (desc) or low
    // to high (!desc).
    __device__ __forceinline__ void scan_hist(bool desc, int shift) {
        if (ltid() < 32) {
            const int lane = ltid();
            const int rem = (int)shm::ld(a_(offsetof(Smem, sel_remaining)));
            uint32_t c[8];
            uint32_t tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int bin = desc ? 255 - (8 * lane + j) : 8 * lane + j;
                c[j] = shm::ld(a_hist() + 4u * (uint32_t)bin);
                tot += c[j];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t before = incl - tot;
            if (before < (uint32_t)rem && (uint32_t)rem <= incl) {
                uint32_t run = before;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= (uint32_t)rem) {
                        const int bin = desc ? 255 - (8 * lane + j) : 8 * lane + j;
                        const uint32_t ap = a_(offsetof(Smem, sel_prefix));
                        shm::st(ap, shm::ld(ap) | ((uint32_t)bin << shift));
                        shm::st(a_(offsetof(Smem, sel_remaining)), (uint32_t)(rem - (int)run));
                        shm::st(a_(offsetof(Smem, sel_found)), c[j]);
                        break;
                    }
                    run += c[j];
                }
            }
        }
        sync();
    }

    // Exact: keep the k best of count > k buffered candidates.
    __device__ __noinline__ void compact(int k) {
        const int tid = ltid();
        const int n = count();
        const uint32_t src = cur();
        const uint32_t sk = a_key_of(src), sp = a_pos_of(src);
        const int iters = (n + NT - 1) / NT;   // uniform trip count: hist_add is warp-collective
        if (tid == 0) {
            shm::st(a_(offsetof(Smem, sel_prefix)), 0u);
            shm::st(a_(offsetof(Smem, sel_remaining)), (uint32_t)k);
        }
        // 1. radix select of the k-th largest key (4 digits of 8 bits, high first)
        uint32_t mask = 0;
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) shm::st(a_hist() + 4u * (uint32_t)i, 0u);
            sync();
            const uint32_t prefix = shm::ld(a_(offsetof(Smem, sel_prefix)));
#pragma unroll 1
            for (int it = 0; it < iters; it += 4) {
                uint32_t u[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {   // independent loads first (overlap their latency)
                    const int i = (it + q) * NT + tid;
                    u[q] = (it + q < iters && i < n) ? shm::ld(sk + 4u * (uint32_t)i) : 0u;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (it + q >= iters) break;   // uniform
                    const int i = (it + q) * NT + tid;
                    int bin = -1;
                    if (i < n && (u[q] & mask) == prefix) bin = (int)((u[q] >> shift) & 255u);
                    hist_add(bin);
                }
            }
            sync();
            scan_hist(true, shift);
            mask |= 255u << shift;
        }
        const uint32_t tau = shm::ld(a_(offsetof(Smem, sel_prefix)));
        const int need = (int)shm::ld(a_(offsetof(Smem, sel_remaining)));   // how many with key == tau to keep
        const int n_eq = (int)shm::ld(a_(offsetof(Smem, sel_found)));
        sync();
        // 2. among key == tau, the `need` lowest positions (only if some must go)
        int32_t pi = 0x7FFFFFFF;
        if (n_eq > need) {
            if (tid == 0) {
                shm::st(a_(offsetof(Smem, sel_prefix)), 0u);
                shm::st(a_(offsetof(Smem, sel_remaining)), (uint32_t)need);
            }
            uint32_t pmask = 0;
#pragma unroll 1
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = tid; i < 256; i += NT) shm::st(a_hist() + 4u * (uint32_t)i, 0u);
                sync();
                const uint32_t prefix = shm::ld(a_(offsetof(Smem, sel_prefix)));
#pragma unroll 1
                for (int it = 0; it < iters; ++it) {
                    const int i = it * NT + tid;
                    int bin = -1;
                    if (i < n && shm::ld(sk + 4u * (uint32_t)i) == tau) {
                        const uint32_t p = shm::ld(sp + 4u * (uint32_t)i);
                        if ((p & pmask) == prefix) bin = (int)((p >> shift) & 255u);
                    }
                    hist_add(bin);
                }
                sync();
                scan_hist(false, shift);
                pmask |= 255u << shift;
            }
            pi = (int32_t)shm::ld(a_(offsetof(Smem, sel_prefix)));
        }
        // 3. write the survivors (exactly k of them) to the other buffer
        const uint32_t dk = a_key_of(src ^ 1u), dp = a_pos_of(src ^ 1u);
        if (tid == 0) {
            shm::st(a_(offsetof(Smem, new_count)), 0u);
            shm::st(a_(offsetof(Smem, worst_pos)), 0xFFFFFFFFu);
        }
        sync();
#pragma unroll 1
        for (int it = 0; it < iters; ++it) {
            const int i = it * NT + tid;
            uint32_t kv = 0u;
            int32_t pv = 0;
            bool keep = false;
            if (i < n) {
                kv = shm::ld(sk + 4u * (uint32_t)i);
                keep = kv > tau || kv == tau;
                if (keep) {
                    pv = (int32_t)shm::ld(sp + 4u * (uint32_t)i);
                    keep = kv > tau || pv <= pi;
                }
            }
            const unsigned ball = __ballot_sync(0xFFFFFFFFu, keep);
            if (ball) {
                const int lane = lane_id();
                const int leader = __ffs(ball) - 1;
                uint32_t slot0 = 0;
                if (lane == leader) slot0 = shm::atom_add(a_(offsetof(Smem, new_count)), (uint32_t)__popc(ball));
                slot0 = __shfl_sync(0xFFFFFFFFu, slot0, leader);
                if (keep) {
                    const uint32_t slot = slot0 + (uint32_t)__popc(ball & ((1u << lane) - 1u));
                    shm::st(dk + 4u * slot, kv);
                    shm::st(dp + 4u * slot, (uint32_t)pv);
                    if (kv == tau) shm::red_max_s32(a_(offsetof(Smem, worst_pos)), pv);
                }
            }
        }
        sync();
        if (tid == 0) {
            shm::st(a_(offsetof(Smem, cur)), src ^ 1u);
            shm::st(a_(offsetof(Smem, count)), shm::ld(a_(offsetof(Smem, new_count))));
            shm::st(a_(offsetof(Smem, has_thr)), 1u);
            shm::st(a_(offsetof(Smem, thr_key)), tau);
            shm::st(a_(offsetof(Smem, thr_pos)), shm::ld(a_(offsetof(Smem, worst_pos))));
        }
        sync();
    }

    // Group-collective: sort the first `n` positions ascending in place
    // (bitonic over the next power of two, padding with INT_MAX).
    __device__ __noinline__ void sort_positions(int n) {
        int np2 = 1;
        while (np2 < n) np2 <<= 1;
        const uint32_t ap = a_pos();
        for (int i = n + ltid(); i < np2; i += NT) shm::st(ap + 4u * (uint32_t)i, 0x7FFFFFFFu);
        sync();
        for (int size = 2; size <= np2; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int t = ltid(); t < np2 / 2; t += NT) {
                    const int i = 2 * t - (t & (stride - 1));
                    const int j = i + stride;
                    const bool up = ((i & size) == 0);
                    const int32_t a = (int32_t)shm::ld(ap + 4u * (uint32_t)i), b = (int32_t)shm::ld(ap + 4u * (uint32_t)j);
                    if ((a > b) == up) {
                        shm::st(ap + 4u * (uint32_t)i, (uint32_t)b);
                        shm::st(ap + 4u * (uint32_t)j, (uint32_t)a);
                    }
                }
                sync();
            }
        }
    }
};

}  // namespace csa2
