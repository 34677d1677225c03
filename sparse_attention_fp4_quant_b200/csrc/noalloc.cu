// noalloc.cu -- csa2_index_topk_noalloc: the index + Top-K call for callers
// that cannot allocate device memory.  Its scratch (merge counters and the
// per-share candidate lists) lives in one file-scope __device__ array of
// CSA2_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds until
// the process exits.  The array's first 256 bytes hold the call's sticky error
// flag (read by csa2_index_topk_noalloc_status); the index kernels' scratch
// follows it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/csa2.h"
#include "kernels.h"

using namespace csa2;

namespace {

constexpr size_t kScratchBytes = CSA2_NOALLOC_SCRATCH_BYTES;
constexpr size_t kFlagBytes = 256;   // the sticky error flag, then the kernels' scratch
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

csa2_status csa2_index_topk_noalloc(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv,
                                    const int32_t* q_pos, int32_t B, int32_t Q, int32_t k, int32_t* idx_out,
                                    float* blockmax_out, void* stream) {
    if (B < 1 || Q < 1 || (int64_t)B * Q > 65535 || k < 1 || k > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (!q || !q_sc || !w || !q_pos || !idx_out || !kv || !kv->ik || !kv->ik_sc || !kv->n_entries) return CSA2_ERR_INVALID_ARG;
    if (kv->cap < 1 || (kv->m != 1 && kv->m != 2) || kv->cap > (int64_t(1) << 31) / 8) return CSA2_ERR_INVALID_ARG;
    if (((uintptr_t)q & 15u) || ((uintptr_t)kv->ik & 15u) || ((uintptr_t)kv->ik_sc & 15u) || kv->cap % 128 != 0)
        return CSA2_ERR_INVALID_ARG;
    if (((uintptr_t)q_sc & 3u) || ((uintptr_t)w & 3u)) return CSA2_ERR_INVALID_ARG;
    // the fixed scratch serves the per-share and cluster paths (not the many-query one)
    const size_t need = select_ws_bytes(CSA2_OP_INDEX_TOPK, B, Q, kv->cap, k, 0, false);
    if (need > kScratchBytes - kFlagBytes) return CSA2_ERR_WORKSPACE;
    void* base = nullptr;
    cudaError_t e = scratch_on_current_device(&base);
    void* ws = static_cast<char*>(base) + kFlagBytes;
    if (e == cudaSuccess) {
        // the flag and the merge counters must start at zero, and the array keeps
        // the last call's contents: clear both (they are adjacent) in one memset
        e = cudaMemsetAsync(base, 0, kFlagBytes + (size_t)B * Q * sizeof(int32_t), (cudaStream_t)stream);
    }
    if (e == cudaSuccess) {
        SelectParams p{};
        p.q = q;
        p.q_sc = q_sc;
        p.w = w;
        p.ik = kv->ik;
        p.ik_sc = kv->ik_sc;
        p.n_entries = kv->n_entries;
        p.cap = kv->cap;
        p.m = kv->m;
        p.q_pos = q_pos;
        p.B = B;
        p.Q = Q;
        p.k = k;
        p.out = idx_out;
        p.blockmax = blockmax_out;
        p.nb_cap = (kv->cap + CSA2_BLOCK - 1) / CSA2_BLOCK;
        p.test_starve = test_starve_copies();
        const int S = select_splits(CSA2_OP_INDEX_TOPK, B, Q, kv->cap, k, 0);
        select_carve_ws(p, S, ws, B, Q, k, false);
        p.status = static_cast<int32_t*>(base);   // the fixed flag, not the carved one
        e = launch_select(CSA2_OP_INDEX_TOPK, p, S, (cudaStream_t)stream);
    }
    if (e != cudaSuccess) {
        record_cuda_error((int)e);
        return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}

csa2_status csa2_index_topk_noalloc_status(int32_t clear, void* stream) {
    void* base = nullptr;
    cudaError_t e = scratch_on_current_device(&base);
    int32_t flag = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, base, sizeof(flag), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess && flag && clear) e = cudaMemsetAsync(base, 0, sizeof(flag), (cudaStream_t)stream);
    if (e != cudaSuccess) {
        record_cuda_error((int)e);
        return CSA2_ERR_CUDA;
    }
    return flag ? CSA2_ERR_TIMEOUT : CSA2_OK;
}

}  // extern "C"
