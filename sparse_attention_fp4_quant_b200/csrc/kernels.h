// kernels.h -- host-visible parameter blocks and launchers of the CSA2 kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/csa2.h"
#include "host_util.h"

namespace csa2 {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Launch with programmatic stream serialisation (the kernel's pdl_enter waits for
// its predecessor) and, if cluster > 0, a 1-D thread-block cluster of that size.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Record a CUDA error for csa2_last_cuda_error() (this host thread).
void record_cuda_error(int e);

// Index Top-K (Full), pool Top-K (Reindex) and pool build share one kernel.
struct SelectParams {
    const uint8_t* q;
    const uint8_t* q_sc;
    const float* w;
    const uint8_t* ik;
    const uint8_t* ik_sc;
    const int32_t* n_entries;
    int64_t cap;
    int m;
    const int32_t* q_pos;
    int B, Q, k;
    int32_t* out;          // idx_out or pool_out [B*Q][k]
    float* blockmax;       // index: optional output; build: input
    int64_t nb_cap;        // ceil(cap / 8)
    const int32_t* pool;   // pool Top-K input [B*Q][P]
    int P;
    // workspace
    int32_t* counters;     // [B*Q], zero between calls
    int32_t* status;       // sticky: set to 1 if a device-side wait timed out
    int32_t* cand_cnt;     // [B*Q][S]
    uint32_t* cand_key;    // [B*Q][S][k]
    int32_t* cand_pos;     // [B*Q][S][k]
    void* mq_ws;           // index Top-K for many queries: key prefixes and histograms (else null)
    int test_starve;       // test hook (csa2_test_starve_copies): the per-share producer issues no copies
    uint32_t* keys;        // order keys in the workspace, or null: [B Q][cap] for the cluster index when they
                           // outgrow TMEM, [B Q][ceil(P / 16) 128] for the search of an ascending pool
};

// The test hook's current setting (read by the index entry points).
int test_starve_copies();

int select_splits(int op, int B, int Q, int64_t cap, int k, int P);
// mq = false leaves out the many-query index path's part (a fixed scratch that may not hold it)
size_t select_ws_bytes(int op, int B, int Q, int64_t cap, int k, int P, bool mq = true);
void select_carve_ws(SelectParams& p, int S, void* ws, int B, int Q, int k, bool mq = true);
// Index Top-K for many queries per batch row (index_mq.cu).
bool index_mq_eligible(int B, int Q, int64_t cap);
size_t index_mq_ws_bytes(int B, int Q, int64_t cap);
cudaError_t launch_index_mq(SelectParams& p, void* mq_ws, cudaStream_t st);
cudaError_t launch_select(int op, SelectParams& p, int S, cudaStream_t st);
bool index_tc_supported(const SelectParams& p);
cudaError_t launch_index_tc(int op, SelectParams& p, int S, cudaStream_t st);
// Workspace bytes for the order keys of a one-share-per-query search of an ascending pool
// (index_tc mode 2): 4 bytes per slot row, the slots rounded up to whole 128-row tiles.
size_t pool_keys_bytes(int B, int Q, int P);
// One cluster of C CTAs per query (index Top-K, and the pool build over the block
// maxima); 0 = the shape does not fit.
int index_cluster_size(const SelectParams& p, bool* keys_in_ws = nullptr);
cudaError_t launch_index_cluster(SelectParams& p, int C, bool keys_in_ws, cudaStream_t st);
// Workspace bytes for the cluster index's keys (0 when its keys fit TMEM or the shape
// takes another kernel): B Q cap x 4 for decode-sized query counts above 16 x 32,768 entries.
size_t cluster_keys_bytes(int B, int Q, int64_t cap);
int pool_build_cluster_size(const SelectParams& p);
// Pool build for many queries (pool_build.cu): one CTA per query, radix select over
// its block maxima; ok = the shape fits (at most 131,072 blocks, aligned maxima).
bool pool_build_radix_ok(const SelectParams& p);
cudaError_t launch_pool_build_radix(SelectParams& p, cudaStream_t st);
cudaError_t launch_pool_build_cluster(SelectParams& p, int C, cudaStream_t st);
int pool_topk_cluster_size(const SelectParams& p);
cudaError_t launch_pool_topk_cluster(SelectParams& p, int C, cudaStream_t st);

// NVFP4 quantisation and the indexer-K projection.
cudaError_t launch_quant(const void* x, int64_t rows, int ch, uint8_t* codes, uint8_t* scales,
                         const int64_t* dst_rows, int64_t out_rows, cudaStream_t st);
cudaError_t launch_index_k_proj(const void* x, int64_t rows, const float* W, uint8_t* k_codes, uint8_t* k_scales,
                                const int64_t* dst_rows, int64_t out_rows, cudaStream_t st);
cudaError_t launch_append(const void* x, int64_t rows, const float* W, uint8_t* lat_codes, uint8_t* lat_scales,
                          uint8_t* k_codes, uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows,
                          cudaStream_t st);
cudaError_t launch_front_end(const void* x, int64_t rows, const float* rcos, const float* rsin, const float* nw,
                             float eps, const float* W, uint8_t* lat_codes, uint8_t* lat_scales, uint8_t* k_codes,
                             uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows, void* y_out,
                             cudaStream_t st);

// Sparse attention.
struct AttnParams {
    const uint16_t* q;        // bf16 [B*Q][16][512]
    const uint8_t* lat;
    const uint8_t* lat_sc;
    const int32_t* n_entries;
    int64_t cap;
    const int32_t* idx;       // [B*Q][k]
    int k;
    const uint8_t* swa;       // [B][T][512]
    const float* swa_sc;      // [B][T]
    const int32_t* swa_pos0;  // [B]
    int T, window;
    const int32_t* replay_start;
    const int32_t* q_pos;
    int B, Q;
    float sm_scale;
    uint16_t* out;            // bf16 [B*Q][16][512]
    float* lse;               // [B*Q][16] or null
    int slots_total;          // k + window
    int tiles_per_split;      // split-K form: 64-key tiles per split
    int main_per_cta;         // cluster form: main slots per CTA (CTA r: [r n, (r + 1) n) of k)
    int swa_per_cta;          // cluster form: window slots per CTA (likewise of the window)
    // workspace
    int32_t* counters;        // [B*Q]
    int32_t* status;          // sticky: set to 1 if a device-side wait timed out
    float* part_o;            // [B*Q][S][16][512]
    float* part_ml;           // [B*Q][S][16][2]
};

int attn_splits(int B, int Q, int k, int window, int* tiles_per_split);
size_t attn_ws_bytes(int B, int Q, int k, int window);
void attn_carve_ws(AttnParams& p, int S, void* ws);
cudaError_t launch_attn(AttnParams& p, int S, cudaStream_t st);
// One cluster of C CTAs per query; 0 = the shape does not fit.
int attn_cluster_size(int B, int Q, int k, int window, int* main_per_cta, int* swa_per_cta);
cudaError_t launch_attn_cluster(AttnParams& p, int C, cudaStream_t st);

}  // namespace csa2
