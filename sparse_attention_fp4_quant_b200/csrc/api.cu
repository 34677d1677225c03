// api.cu -- the extern "C" entry points of libcsa2.so: argument validation,
// workspace sizing, launch, and the per-layer mode dispatch.
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/csa2.h"
#include "kernels.h"

using namespace csa2;

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_test_starve{0};

csa2_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return CSA2_OK;
    g_last_cuda_error = (int)e;
    return CSA2_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool kv_ok(const csa2_kv* kv) {
    return kv && kv->n_entries && kv->cap >= 1 && (kv->m == 1 || kv->m == 2) && kv->cap <= (int64_t(1) << 31) / 8;
}

bool kv_index_ok(const csa2_kv* kv) {
    return kv_ok(kv) && kv->ik && kv->ik_sc && aligned16(kv->ik) && aligned16(kv->ik_sc) && kv->cap % 128 == 0;
}

bool kv_latent_ok(const csa2_kv* kv) {
    return kv_ok(kv) && kv->lat && kv->lat_sc && aligned16(kv->lat) && aligned16(kv->lat_sc);
}

SelectParams select_params(const csa2_kv* kv, const int32_t* q_pos, int B, int Q, int k) {
    SelectParams p{};
    p.ik = kv->ik;
    p.ik_sc = kv->ik_sc;
    p.n_entries = kv->n_entries;
    p.cap = kv->cap;
    p.m = kv->m;
    p.q_pos = q_pos;
    p.B = B;
    p.Q = Q;
    p.k = k;
    p.nb_cap = (kv->cap + CSA2_BLOCK - 1) / CSA2_BLOCK;
    return p;
}

}  // namespace

namespace csa2 {
void record_cuda_error(int e) { g_last_cuda_error = e; }
int test_starve_copies() { return g_test_starve.load(std::memory_order_relaxed); }
}  // namespace csa2

extern "C" {

const char* csa2_status_str(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "CSA2_OK";
        case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG";
        case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED";
        case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE";
        case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
        case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
    }
    return "CSA2_ERR_UNKNOWN";
}

int csa2_last_cuda_error(void) { return g_last_cuda_error; }

void csa2_test_starve_copies(int32_t enable) { g_test_starve.store(enable ? 1 : 0, std::memory_order_relaxed); }

csa2_status csa2_quant_nvfp4(const void* x, int64_t rows, int32_t ch, uint8_t* codes, uint8_t* scales,
                             const int64_t* dst_rows, int64_t out_rows, void* stream) {
    if (rows < 0 || ch < 16 || ch > 4096 || ch % 16 != 0) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    if (!x || !codes || !scales || !aligned16(x) || ((uintptr_t)codes & 7u)) return CSA2_ERR_INVALID_ARG;
    if (out_rows < 0 || (!dst_rows && out_rows < rows)) return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_quant(x, rows, ch, codes, scales, dst_rows, out_rows, (cudaStream_t)stream));
}

csa2_status csa2_index_k_proj(const void* x, int64_t rows, const float* W, uint8_t* k_codes, uint8_t* k_scales,
                              const int64_t* dst_rows, int64_t out_rows, void* stream) {
    if (rows < 0) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    if (!x || !W || !k_codes || !k_scales || !aligned16(x) || !aligned16(W) || ((uintptr_t)k_codes & 7u))
        return CSA2_ERR_INVALID_ARG;
    if (out_rows < 0 || out_rows % 128 != 0 || (!dst_rows && out_rows < rows)) return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_index_k_proj(x, rows, W, k_codes, k_scales, dst_rows, out_rows, (cudaStream_t)stream));
}

csa2_status csa2_append_tokens(const void* x, int64_t rows, const float* W, uint8_t* lat_codes, uint8_t* lat_scales,
                               uint8_t* k_codes, uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows,
                               void* stream) {
    if (rows < 0) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    if (!x || !W || !lat_codes || !lat_scales || !k_codes || !k_scales || !aligned16(x) || !aligned16(W) ||
        ((uintptr_t)lat_codes & 7u) || ((uintptr_t)k_codes & 7u))
        return CSA2_ERR_INVALID_ARG;
    if (out_rows < 0 || out_rows % 128 != 0 || (!dst_rows && out_rows < rows)) return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_append(x, rows, W, lat_codes, lat_scales, k_codes, k_scales, dst_rows, out_rows,
                                     (cudaStream_t)stream));
}

csa2_status csa2_device_status(void* ws, int32_t B, int32_t Q, int32_t clear, void* stream) {
    if (!ws || B < 1 || Q < 1) return CSA2_ERR_INVALID_ARG;
    char* flag_ptr = static_cast<char*>(ws) + CSA2_STATUS_OFFSET(B, Q);
    int32_t flag = 0;
    cudaError_t e = cudaMemcpyAsync(&flag, flag_ptr, sizeof(flag), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess && flag && clear) e = cudaMemsetAsync(flag_ptr, 0, sizeof(flag), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
    return flag ? CSA2_ERR_TIMEOUT : CSA2_OK;
}

size_t csa2_workspace_bytes(csa2_op op, int32_t B, int32_t Q, int64_t cap, int32_t k, int32_t P) {
    if (B < 1 || Q < 1) return 0;
    switch (op) {
        case CSA2_OP_INDEX_TOPK:
            return ((select_ws_bytes((int)op, B, Q, cap, k, P) + 255) & ~(size_t)255) + cluster_keys_bytes(B, Q, cap);
        case CSA2_OP_POOL_BUILD:
        case CSA2_OP_POOL_TOPK: return select_ws_bytes((int)op, B, Q, cap, k, P);
        case CSA2_OP_SPARSE_ATTN: return attn_ws_bytes(B, Q, k, CSA2_MAX_WINDOW);
        case CSA2_OP_LAYER: {
            size_t a = ((select_ws_bytes(CSA2_OP_INDEX_TOPK, B, Q, cap, k, P) + 255) & ~(size_t)255) +
                       cluster_keys_bytes(B, Q, cap);
            size_t b = select_ws_bytes(CSA2_OP_POOL_BUILD, B, Q, cap, P > 0 ? P : 1, P);
            size_t c = select_ws_bytes(CSA2_OP_POOL_TOPK, B, Q, cap, k, P);
            if (P > 0 && select_splits(CSA2_OP_POOL_TOPK, B, Q, cap, k, P) == 1)   // Reindex keeps its keys
                c = ((c + 255) & ~(size_t)255) + pool_keys_bytes(B, Q, P);
            size_t d = attn_ws_bytes(B, Q, k, CSA2_MAX_WINDOW);
            size_t m = a;
            if (b > m) m = b;
            if (c > m) m = c;
            if (d > m) m = d;
            return m;
        }
    }
    return 0;
}

csa2_status csa2_front_end(const void* x, int64_t rows, const float* rope_cos, const float* rope_sin,
                           const float* norm_w, float eps, const float* W, uint8_t* lat_codes, uint8_t* lat_scales,
                           uint8_t* k_codes, uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows, void* y_out,
                           void* stream) {
    if (rows < 0) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    if (!x || !rope_cos || !rope_sin || !W || !lat_codes || !lat_scales || !k_codes || !k_scales || !aligned16(x) ||
        !aligned16(W) || ((uintptr_t)lat_codes & 7u) || ((uintptr_t)k_codes & 7u) || ((uintptr_t)rope_cos & 3u) ||
        ((uintptr_t)rope_sin & 3u) || ((uintptr_t)norm_w & 3u) || (y_out && !aligned16(y_out)))
        return CSA2_ERR_INVALID_ARG;
    if (!(eps == eps)) return CSA2_ERR_INVALID_ARG;
    if (out_rows < 0 || out_rows % 128 != 0 || (!dst_rows && out_rows < rows)) return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_front_end(x, rows, rope_cos, rope_sin, norm_w, eps, W, lat_codes, lat_scales, k_codes,
                                        k_scales, dst_rows, out_rows, y_out, (cudaStream_t)stream));
}

csa2_status csa2_index_topk(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv,
                            const int32_t* q_pos, int32_t B, int32_t Q, int32_t k, int32_t* idx_out,
                            float* blockmax_out, void* ws, size_t ws_bytes, void* stream) {
    if (B < 1 || Q < 1 || (int64_t)B * Q > 65535 || k < 1 || k > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (!q || !q_sc || !w || !q_pos || !idx_out || !kv_index_ok(kv) || !aligned16(q)) return CSA2_ERR_INVALID_ARG;
    if (((uintptr_t)q_sc & 3u) || ((uintptr_t)w & 3u)) return CSA2_ERR_INVALID_ARG;
    if (!ws || ws_bytes < select_ws_bytes(CSA2_OP_INDEX_TOPK, B, Q, kv->cap, k, 0)) return CSA2_ERR_WORKSPACE;
    SelectParams p = select_params(kv, q_pos, B, Q, k);
    p.q = q;
    p.q_sc = q_sc;
    p.w = w;
    p.out = idx_out;
    p.blockmax = blockmax_out;
    p.test_starve = test_starve_copies();
    int S = select_splits(CSA2_OP_INDEX_TOPK, B, Q, kv->cap, k, 0);
    select_carve_ws(p, S, ws, B, Q, k);
    // the cluster index keeps its keys in the workspace when they outgrow TMEM and the
    // workspace has room for them (csa2_workspace_bytes counts it; the minimum does not)
    const size_t need = select_ws_bytes(CSA2_OP_INDEX_TOPK, B, Q, kv->cap, k, 0);
    const size_t kb = cluster_keys_bytes(B, Q, kv->cap);
    const size_t off = (need + 255) & ~(size_t)255;
    if (kb > 0 && ws_bytes >= off + kb) p.keys = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + off);
    return cuda_status(launch_select(CSA2_OP_INDEX_TOPK, p, S, (cudaStream_t)stream));
}

csa2_status csa2_pool_build(const float* blockmax, const csa2_kv* kv, const int32_t* q_pos, int32_t B, int32_t Q,
                            int32_t max_blocks, int32_t* pool_out, void* ws, size_t ws_bytes, void* stream) {
    if (B < 1 || Q < 1 || (int64_t)B * Q > 65535 || max_blocks < 1 || max_blocks > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (!blockmax || !q_pos || !pool_out || !kv_ok(kv)) return CSA2_ERR_INVALID_ARG;
    if (!ws || ws_bytes < select_ws_bytes(CSA2_OP_POOL_BUILD, B, Q, kv->cap, max_blocks, 0)) return CSA2_ERR_WORKSPACE;
    SelectParams p = select_params(kv, q_pos, B, Q, max_blocks);
    p.blockmax = const_cast<float*>(blockmax);
    p.out = pool_out;
    int S = select_splits(CSA2_OP_POOL_BUILD, B, Q, kv->cap, max_blocks, 0);
    select_carve_ws(p, S, ws, B, Q, max_blocks);
    const int C = pool_build_cluster_size(p);   // decode-sized query counts: the cluster radix select
    if (C > 0) return cuda_status(launch_pool_build_cluster(p, C, (cudaStream_t)stream));
    // one CTA per query fills the GPU: the per-query radix select
    if (S == 1 && pool_build_radix_ok(p)) return cuda_status(launch_pool_build_radix(p, (cudaStream_t)stream));
    return cuda_status(launch_select(CSA2_OP_POOL_BUILD, p, S, (cudaStream_t)stream));
}

namespace {
// The pool Top-K; `ascending`: the pool lists its valid blocks in ascending id order (as
// csa2_pool_build writes it), which the cluster select needs (it orders and breaks ties by
// pool slot); any other pool takes the per-share select, which sorts by position.
csa2_status pool_topk(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv, const int32_t* pool,
                      int32_t P, const int32_t* q_pos, int32_t B, int32_t Q, int32_t k, int32_t* idx_out, void* ws,
                      size_t ws_bytes, void* stream, bool ascending) {
    if (B < 1 || Q < 1 || (int64_t)B * Q > 65535 || k < 1 || k > CSA2_MAX_K || P < 1 || P > 65536) return CSA2_ERR_INVALID_ARG;
    if (!q || !q_sc || !w || !pool || !q_pos || !idx_out || !kv_index_ok(kv) || !aligned16(q))
        return CSA2_ERR_INVALID_ARG;
    if (((uintptr_t)q_sc & 3u) || ((uintptr_t)w & 3u)) return CSA2_ERR_INVALID_ARG;
    if (!ws || ws_bytes < select_ws_bytes(CSA2_OP_POOL_TOPK, B, Q, kv->cap, k, P)) return CSA2_ERR_WORKSPACE;
    SelectParams p = select_params(kv, q_pos, B, Q, k);
    p.q = q;
    p.q_sc = q_sc;
    p.w = w;
    p.pool = pool;
    p.P = P;
    p.out = idx_out;
    int S = select_splits(CSA2_OP_POOL_TOPK, B, Q, kv->cap, k, P);
    select_carve_ws(p, S, ws, B, Q, k);
    const int C = ascending ? pool_topk_cluster_size(p) : 0;   // decode-sized query counts: the cluster select
    if (C > 0) return cuda_status(launch_pool_topk_cluster(p, C, (cudaStream_t)stream));
    if (ascending && S == 1) {   // one CTA per query: keep the keys when the workspace has room for them
        const size_t off = (select_ws_bytes(CSA2_OP_POOL_TOPK, B, Q, kv->cap, k, P) + 255) & ~(size_t)255;
        if (ws_bytes >= off + pool_keys_bytes(B, Q, P)) p.keys = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + off);
    }
    return cuda_status(launch_select(CSA2_OP_POOL_TOPK, p, S, (cudaStream_t)stream));
}
}  // namespace

csa2_status csa2_pool_topk(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv,
                           const int32_t* pool, int32_t P, const int32_t* q_pos, int32_t B, int32_t Q, int32_t k,
                           int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
    return pool_topk(q, q_sc, w, kv, pool, P, q_pos, B, Q, k, idx_out, ws, ws_bytes, stream, false);
}

csa2_status csa2_sparse_attn(const void* q, const csa2_kv* kv, const int32_t* idx, int32_t k, const uint8_t* swa,
                             const float* swa_sc, const int32_t* swa_pos0, int32_t T, int32_t window,
                             const int32_t* replay_start, const int32_t* q_pos, int32_t B, int32_t Q,
                             float sm_scale, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    if (B < 1 || Q < 1 || (int64_t)B * Q > 65535 || k < 0 || k > CSA2_MAX_K || T < 0 || window < 1 || window > CSA2_MAX_WINDOW)
        return CSA2_ERR_INVALID_ARG;
    if (!q || !out || !q_pos || !swa_pos0 || !kv_latent_ok(kv) || !aligned16(q) || ((uintptr_t)out & 3u))
        return CSA2_ERR_INVALID_ARG;
    if (k > 0 && !idx) return CSA2_ERR_INVALID_ARG;
    if (T > 0 && (!swa || !swa_sc || !aligned16(swa))) return CSA2_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale)) return CSA2_ERR_INVALID_ARG;
    if (!ws || ws_bytes < attn_ws_bytes(B, Q, k, window)) return CSA2_ERR_WORKSPACE;
    AttnParams p{};
    p.q = static_cast<const uint16_t*>(q);
    p.lat = kv->lat;
    p.lat_sc = kv->lat_sc;
    p.n_entries = kv->n_entries;
    p.cap = kv->cap;
    p.idx = idx;
    p.k = k;
    p.swa = swa;
    p.swa_sc = swa_sc;
    p.swa_pos0 = swa_pos0;
    p.T = T;
    p.window = window;
    p.replay_start = replay_start;
    p.q_pos = q_pos;
    p.B = B;
    p.Q = Q;
    p.sm_scale = sm_scale;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.slots_total = k + window;
    int S = attn_splits(B, Q, k, window, &p.tiles_per_split);
    attn_carve_ws(p, S, ws);
    const int C = attn_cluster_size(B, Q, k, window, &p.main_per_cta, &p.swa_per_cta);
    if (C > 0) return cuda_status(launch_attn_cluster(p, C, (cudaStream_t)stream));
    return cuda_status(launch_attn(p, S, (cudaStream_t)stream));
}

csa2_status csa2_layer_step(const csa2_layer_args* a, void* stream) {
    if (!a || !a->kv) return CSA2_ERR_INVALID_ARG;
    if (a->mode != CSA2_MODE_FULL && a->mode != CSA2_MODE_REINDEX && a->mode != CSA2_MODE_REUSE)
        return CSA2_ERR_INVALID_ARG;
    const csa2_kv* kv = a->kv;
    csa2_status st;
    if (a->mode == CSA2_MODE_FULL) {
        if (a->n_new > 0) {
            if (!a->new_latent || !a->new_rows || !a->k_proj) return CSA2_ERR_INVALID_ARG;
            st = csa2_append_tokens(a->new_latent, a->n_new, a->k_proj, kv->lat, kv->lat_sc, kv->ik, kv->ik_sc,
                                    a->new_rows, (int64_t)kv->cap * a->B, stream);
            if (st != CSA2_OK) return st;
        }
        bool build = a->pool != nullptr;
        if (build && !a->blockmax) return CSA2_ERR_INVALID_ARG;
        st = csa2_index_topk(a->iq, a->iq_sc, a->w, kv, a->q_pos, a->B, a->Q, a->k, a->idx,
                             build ? a->blockmax : nullptr, a->ws, a->ws_bytes, stream);
        if (st != CSA2_OK) return st;
        if (build) {
            st = csa2_pool_build(a->blockmax, kv, a->q_pos, a->B, a->Q, a->pool_blocks, a->pool, a->ws, a->ws_bytes,
                                 stream);
            if (st != CSA2_OK) return st;
        }
    } else if (a->mode == CSA2_MODE_REINDEX) {
        st = pool_topk(a->iq, a->iq_sc, a->w, kv, a->pool, a->pool_blocks, a->q_pos, a->B, a->Q, a->k, a->idx,
                       a->ws, a->ws_bytes, stream, true);
        if (st != CSA2_OK) return st;
    }
    return csa2_sparse_attn(a->q, kv, a->idx, a->k, a->swa, a->swa_sc, a->swa_pos0, a->T, a->window,
                            a->replay_start, a->q_pos, a->B, a->Q, a->sm_scale, a->out, a->lse, a->ws, a->ws_bytes,
                            stream);
}

}  // extern "C"
