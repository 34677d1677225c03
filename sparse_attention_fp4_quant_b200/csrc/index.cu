// index.cu -- FP4 index scoring + exact Top-K (Full layers), pool Top-K
// (Reindex layers) and pool build (hierarchical sparse indexer).
//
// One CTA scores a contiguous share of one query's candidates, keeps its local
// best k in shared memory (topk.cuh) and writes them to the workspace; the
// last CTA of the query (atomic ticket) merges the shares and writes the
// ascending positions.  With one share per query the CTA writes directly.
#include "common.cuh"
#include "kernels.h"
#include "score_cc.cuh"
#include "topk.cuh"

namespace csa2 {

constexpr int kNT = 256;
constexpr int kCap = 4096;
using TK = TopK<kNT, kCap>;

enum { MODE_DENSE = 0, MODE_POOL = 1, MODE_BUILD = 2 };

// Merge the S shares of query bq from the workspace (last CTA only), then write
// the ascending positions.  Block-collective.
__device__ void finalize(TK& tk, const SelectParams& p, int bq, int S, int k, int32_t* out) {
    const int tid = threadIdx.x;
    if (S > 1) {
        int cnt = tk.count();
        int64_t off = ((int64_t)bq * S + blockIdx.x) * k;
        for (int i = tid; i < cnt; i += kNT) {
            p.cand_key[off + i] = tk.key_at(i);
            p.cand_pos[off + i] = tk.pos_at(i);
        }
        if (tid == 0) p.cand_cnt[(int64_t)bq * S + blockIdx.x] = cnt;
        __threadfence();
        __syncthreads();
        __shared__ int s_last;
        if (tid == 0) s_last = (atomicAdd(&p.counters[bq], 1) == S - 1);
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        tk.init();
        for (int c = 0; c < S; ++c) {
            int n = __ldcg(&p.cand_cnt[(int64_t)bq * S + c]);
            int64_t coff = ((int64_t)bq * S + c) * k;
            for (int base = 0; base < n; base += kNT) {
                tk.make_room(k, kNT);
                int i = base + tid;
                bool valid = i < n;
                uint32_t key = valid ? __ldcg(&p.cand_key[coff + i]) : 0u;
                int32_t pos = valid ? __ldcg(&p.cand_pos[coff + i]) : 0;
                tk.offer(valid, key, pos);
            }
        }
        tk.finish(k);
        if (tid == 0) p.counters[bq] = 0;
    }
    int cnt = tk.count();
    tk.sort_positions(cnt);
    for (int i = tid; i < k; i += kNT) out[(int64_t)bq * k + i] = i < cnt ? tk.pos_at(i) : -1;
}

template <int MODE>
__global__ void __launch_bounds__(kNT, 2) select_kernel(SelectParams p) {
    pdl_enter();
    extern __shared__ __align__(16) uint8_t select_smem[];
    TK tk(*reinterpret_cast<TK::Smem*>(select_smem));
    const int tid = threadIdx.x;
    const int bq = blockIdx.y;
    const int s = blockIdx.x, S = gridDim.x;
    const int b = bq / p.Q;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const int k = p.k;
    tk.init();

    if (MODE == MODE_BUILD) {
        const int64_t nbcap = p.nb_cap;
        int nblk = (nvis + kBlk - 1) / kBlk;
        if (nblk > nbcap) nblk = (int)nbcap;
        int chunk = (nblk + S - 1) / S;
        int lo = min(nblk, s * chunk), hi = min(nblk, lo + chunk);
        const float* bm = p.blockmax + (int64_t)bq * nbcap;
        for (int base = lo; base < hi; base += kNT) {
            tk.make_room(k, kNT);
            int j = base + tid;
            bool valid = j < hi;
            float v = valid ? __ldg(bm + j) : 0.0f;
            tk.offer(valid, score_key(v), j);
        }
        tk.finish(k);
        finalize(tk, p, bq, S, k, p.out);
        return;
    }

    QReg R;
    load_query(R, p.q + (int64_t)bq * 128, p.q_sc + (int64_t)bq * 16, p.w + (int64_t)bq * 4);
    const uint8_t* ik = p.ik + (int64_t)b * p.cap * 32;
    const uint8_t* iks = p.ik_sc + (int64_t)b * p.cap * 4;

    if (MODE == MODE_DENSE) {
        int chunk = (((nvis + S - 1) / S) + 7) & ~7;
        int lo = min(nvis, s * chunk), hi = min(nvis, lo + chunk);
        float* bm = p.blockmax ? p.blockmax + (int64_t)bq * p.nb_cap : nullptr;
        for (int base = lo; base < hi; base += 2 * kNT) {
            tk.make_room(k, 2 * kNT);
            int e0 = base + tid, e1 = base + kNT + tid;
            bool v0 = e0 < hi, v1 = e1 < hi;
            float s0 = -INFINITY, s1 = -INFINITY;
            if (v0) s0 = entry_score_at(R, ik, iks, e0);
            if (v1) s1 = entry_score_at(R, ik, iks, e1);
            if (bm) {
                const float m0 = block_max8(s0, tid & 31), m1 = block_max8(s1, tid & 31);
                if ((tid & 7) == 0) {
                    if (v0) bm[e0 >> 3] = m0;
                    if (v1) bm[e1 >> 3] = m1;
                }
            }
            tk.offer(v0, score_key(s0), e0);
            tk.offer(v1, score_key(s1), e1);
        }
        if (bm) {  // blocks with no visible position
            int64_t jb = (nvis + kBlk - 1) / kBlk;
            int64_t rest = p.nb_cap - jb;
            if (rest > 0) {
                int64_t cs = (rest + S - 1) / S;
                int64_t j0 = jb + (int64_t)s * cs, j1 = min(p.nb_cap, j0 + cs);
                for (int64_t j = j0 + tid; j < j1; j += kNT) bm[j] = -INFINITY;
            }
        }
    } else {  // MODE_POOL
        const int P = p.P;
        int ps = (P + S - 1) / S;
        int lo = min(P, s * ps), hi = min(P, lo + ps);
        const int32_t* pool = p.pool + (int64_t)bq * P;
        for (int sb = lo; sb < hi; sb += kNT / kBlk) {
            tk.make_room(k, kNT);
            int slot = sb + tid / kBlk;
            int blk = slot < hi ? __ldg(pool + slot) : -1;
            int64_t e = (int64_t)blk * kBlk + (tid & (kBlk - 1));
            bool valid = blk >= 0 && e < nvis;
            float sc = valid ? entry_score_at(R, ik, iks, e) : 0.0f;
            tk.offer(valid, score_key(sc), (int32_t)e);
        }
    }
    tk.finish(k);
    finalize(tk, p, bq, S, k, p.out);
}

// ---- host side -------------------------------------------------------------

static int slots() { return 2 * kSplitSMs; }

int select_splits(int op, int B, int Q, int64_t cap, int k, int P) {
    int64_t bq = (int64_t)B * Q;
    int64_t by_cta = slots() / (bq > 0 ? bq : 1);
    int64_t want;
    if (op == CSA2_OP_INDEX_TOPK) want = (cap + 2047) / 2048;
    else if (op == CSA2_OP_POOL_TOPK) want = ((int64_t)P * kBlk + 4095) / 4096;
    else want = ((cap + kBlk - 1) / kBlk + 16383) / 16384;
    int64_t S = want < by_cta ? want : by_cta;
    if (S < 1) S = 1;
    if (S > 1024) S = 1024;
    return (int)S;
}

size_t select_ws_bytes(int op, int B, int Q, int64_t cap, int k, int P, bool mq) {
    int S = select_splits(op, B, Q, cap, k, P);
    size_t bq = (size_t)B * Q;
    size_t bytes = align256(bq * 4);                 // counters
    bytes += 256;                                    // status word
    if (S > 1) {
        bytes += align256(bq * S * 4);               // share counts
        bytes += 2 * align256(bq * S * (size_t)k * 4);  // keys, positions
    }
    if (mq && op == CSA2_OP_INDEX_TOPK && index_mq_eligible(B, Q, cap)) bytes += index_mq_ws_bytes(B, Q, cap);
    return bytes;
}

void select_carve_ws(SelectParams& p, int S, void* ws, int B, int Q, int k, bool mq) {
    size_t bq = (size_t)B * Q;
    char* c = (char*)ws;
    p.counters = (int32_t*)c;
    c += align256(bq * 4);
    p.status = (int32_t*)c;
    c += 256;
    if (S > 1) {
        p.cand_cnt = (int32_t*)c;
        c += align256(bq * S * 4);
        p.cand_key = (uint32_t*)c;
        c += align256(bq * S * (size_t)k * 4);
        p.cand_pos = (int32_t*)c;
        c += align256(bq * S * (size_t)k * 4);
    }
    p.mq_ws = (mq && index_mq_eligible(B, Q, p.cap)) ? (void*)c : nullptr;
}

cudaError_t launch_select(int op, SelectParams& p, int S, cudaStream_t st) {
    if ((op == CSA2_OP_INDEX_TOPK || op == CSA2_OP_POOL_TOPK) && index_tc_supported(p)) {
        if (op == CSA2_OP_INDEX_TOPK && p.mq_ws) return launch_index_mq(p, p.mq_ws, st);
        if (op == CSA2_OP_INDEX_TOPK) {
            bool keys_in_ws = false;
            const int C = index_cluster_size(p, &keys_in_ws);
            if (C > 0) return launch_index_cluster(p, C, keys_in_ws, st);
        }
        return launch_index_tc(op, p, S, st);
    }
    dim3 grid(S, p.B * p.Q);
    const int smem = (int)sizeof(TK::Smem);
    static DeviceOnce attr[3];
    const int mode = op == CSA2_OP_INDEX_TOPK ? 0 : (op == CSA2_OP_POOL_TOPK ? 1 : 2);
    cudaError_t e = attr[mode].run([&] {
        return mode == 0   ? cudaFuncSetAttribute(select_kernel<MODE_DENSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
               : mode == 1 ? cudaFuncSetAttribute(select_kernel<MODE_POOL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
                           : cudaFuncSetAttribute(select_kernel<MODE_BUILD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    if (mode == 0) return launch_ex(select_kernel<MODE_DENSE>, grid, dim3(kNT), smem, st, 0, p);
    if (mode == 1) return launch_ex(select_kernel<MODE_POOL>, grid, dim3(kNT), smem, st, 0, p);
    return launch_ex(select_kernel<MODE_BUILD>, grid, dim3(kNT), smem, st, 0, p);
}

}  // namespace csa2
