// topk.cuh -- exact block-wide Top-K selection in shared memory.
//
// Order: key descending, then position ascending (keys are the monotone uint32
// images of fp32 scores, so equal scores tie and the lower position wins).
// Candidates stream through a threshold filter into a buffer of CAP slots;
// when the buffer nears full, an exact radix select keeps the best k and the
// k-th best (key, pos) becomes the new admission threshold.  Offer order does
// not matter: the composite threshold admits a later candidate that ties the
// threshold score only if its position is lower.
#pragma once
#include "common.cuh"

namespace csa2 {

template <int NT, int CAP>
struct TopK {
    static_assert(CAP % NT == 0, "CAP must be a multiple of the block size");
    static constexpr int PER = CAP / NT;

    struct Smem {
        uint32_t key[CAP];
        int32_t pos[CAP];
        uint32_t hist[256];
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

    Smem& s;
    __device__ explicit TopK(Smem& sm) : s(sm) {}

    __device__ void init() {
        if (threadIdx.x == 0) {
            s.count = 0;
            s.has_thr = 0;
            s.thr_key = 0;
            s.thr_pos = 0x7FFFFFFF;
        }
        __syncthreads();
    }

    // Does (key, pos) beat the current threshold?
    __device__ __forceinline__ bool admits(uint32_t key, int32_t pos) const {
        if (!s.has_thr) return true;
        uint32_t tk = s.thr_key;
        return key > tk || (key == tk && pos < s.thr_pos);
    }

    // Warp-collective: every lane of the warp must call it (valid may be false).
    __device__ __forceinline__ void offer(bool valid, uint32_t key, int32_t pos) {
        bool take = valid && admits(key, pos);
        unsigned ball = __ballot_sync(0xFFFFFFFFu, take);
        if (ball == 0) return;
        int lane = lane_id();
        int leader = __ffs(ball) - 1;
        int base = 0;
        if (lane == leader) base = atomicAdd(&s.count, __popc(ball));
        base = __shfl_sync(0xFFFFFFFFu, base, leader);
        if (take) {
            int slot = base + __popc(ball & ((1u << lane) - 1u));
            s.key[slot] = key;
            s.pos[slot] = pos;
        }
    }

    // Block-collective.  Guarantees room for `room` more offers.
    __device__ void make_room(int k, int room) {
        __syncthreads();
        if (s.count > CAP - room) compact(k);
    }

    // Block-collective.  After it, count <= k and the buffer holds the best k.
    __device__ void finish(int k) {
        __syncthreads();
        if (s.count > k) compact(k);
    }

    // Warp 0 scans the 256-bin histogram for the bin holding the `remaining`-th
    // element, scanning bins from high to low (desc) or low to high (!desc).
    __device__ void scan_hist(bool desc, int shift, uint32_t bits_mask) {
        if (threadIdx.x < 32) {
            int lane = threadIdx.x;
            int rem = s.sel_remaining;
            uint32_t c[8];
            uint32_t tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int bin = desc ? 255 - (8 * lane + j) : 8 * lane + j;
                c[j] = s.hist[bin];
                tot += c[j];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            uint32_t before = incl - tot;
            if (before < (uint32_t)rem && (uint32_t)rem <= incl) {
                uint32_t run = before;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= (uint32_t)rem) {
                        int bin = desc ? 255 - (8 * lane + j) : 8 * lane + j;
                        s.sel_prefix |= (uint32_t)bin << shift;
                        s.sel_remaining = rem - (int)run;
                        s.sel_found = (int)c[j];
                        break;
                    }
                    run += c[j];
                }
            }
        }
        __syncthreads();
    }

    // Exact: keep the k best of count > k buffered candidates.
    __device__ void compact(int k) {
        const int tid = threadIdx.x;
        const int n = s.count;
        if (tid == 0) {
            s.sel_prefix = 0;
            s.sel_remaining = k;
        }
        // 1. radix select of the k-th largest key (4 digits of 8 bits, high first)
        uint32_t mask = 0;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) s.hist[i] = 0;
            __syncthreads();
            uint32_t prefix = s.sel_prefix;
            for (int i = tid; i < n; i += NT) {
                uint32_t u = s.key[i];
                if ((u & mask) == prefix) atomicAdd(&s.hist[(u >> shift) & 255u], 1u);
            }
            __syncthreads();
            scan_hist(true, shift, mask);
            mask |= 255u << shift;
        }
        const uint32_t tau = s.sel_prefix;
        const int need = s.sel_remaining;   // how many with key == tau to keep
        const int n_eq = s.sel_found;
        __syncthreads();
        // 2. among key == tau, the `need` lowest positions (only if some must go)
        int32_t pi = 0x7FFFFFFF;
        if (n_eq > need) {
            if (tid == 0) {
                s.sel_prefix = 0;
                s.sel_remaining = need;
            }
            uint32_t pmask = 0;
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = tid; i < 256; i += NT) s.hist[i] = 0;
                __syncthreads();
                uint32_t prefix = s.sel_prefix;
                for (int i = tid; i < n; i += NT) {
                    if (s.key[i] != tau) continue;
                    uint32_t p = (uint32_t)s.pos[i];
                    if ((p & pmask) == prefix) atomicAdd(&s.hist[(p >> shift) & 255u], 1u);
                }
                __syncthreads();
                scan_hist(false, shift, pmask);
                pmask |= 255u << shift;
            }
            pi = (int32_t)s.sel_prefix;
        }
        // 3. compact the survivors (exactly k of them)
        uint32_t kk[PER];
        int32_t pp[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            int i = tid + j * NT;
            kk[j] = 0;
            pp[j] = 0;
            if (i < n) {
                kk[j] = s.key[i];
                pp[j] = s.pos[i];
            }
        }
        if (tid == 0) {
            s.new_count = 0;
            s.worst_pos = -1;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            int i = tid + j * NT;
            bool keep = (i < n) && (kk[j] > tau || (kk[j] == tau && pp[j] <= pi));
            unsigned ball = __ballot_sync(0xFFFFFFFFu, keep);
            if (ball) {
                int lane = lane_id();
                int leader = __ffs(ball) - 1;
                int base = 0;
                if (lane == leader) base = atomicAdd(&s.new_count, __popc(ball));
                base = __shfl_sync(0xFFFFFFFFu, base, leader);
                if (keep) {
                    int slot = base + __popc(ball & ((1u << lane) - 1u));
                    s.key[slot] = kk[j];
                    s.pos[slot] = pp[j];
                    if (kk[j] == tau) atomicMax(&s.worst_pos, pp[j]);
                }
            }
        }
        __syncthreads();
        if (tid == 0) {
            s.count = s.new_count;
            s.has_thr = 1;
            s.thr_key = tau;
            s.thr_pos = s.worst_pos;
        }
        __syncthreads();
    }

    // Block-collective: sort the first `n` positions ascending in place
    // (bitonic over the next power of two, padding with INT_MAX).
    __device__ void sort_positions(int n) {
        int np2 = 1;
        while (np2 < n) np2 <<= 1;
        for (int i = n + threadIdx.x; i < np2; i += NT) s.pos[i] = 0x7FFFFFFF;
        __syncthreads();
        for (int size = 2; size <= np2; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int t = threadIdx.x; t < np2 / 2; t += NT) {
                    int i = 2 * t - (t & (stride - 1));
                    int j = i + stride;
                    bool up = ((i & size) == 0);
                    int32_t a = s.pos[i], b = s.pos[j];
                    if ((a > b) == up) {
                        s.pos[i] = b;
                        s.pos[j] = a;
                    }
                }
                __syncthreads();
            }
        }
    }
};

}  // namespace csa2
