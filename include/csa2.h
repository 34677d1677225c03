/*
 * csa2.h -- C ABI of libcsa2.so, the B200 (sm_100a) hot path of CSA2
 * (Compressed Sparse Attention 2) as the public write-ups of the
 * DeepSeek-V4.1-Flash report describe it.
 *
 * Sources cited below:
 *   [Blog]  "一个 token 只花 890 字节：DeepSeek-V4.1-Flash 把 KV 缓存压到了什么程度"
 *           (shibing624.github.io ai-paper-analysis): sections
 *           "CSA2：跨层复用，能借就不自己算" (Fig. 4), "分层稀疏索引器：让深层
 *           indexer 别全文搜索" (Fig. 5), "FP4 与 SWA Bounded Replay：另外两刀".
 *   [Jdon]  "557亿参数只唤醒80亿！…" (jdon.com), section "缓存压缩真的是越大越好吗".
 *   [Lsln]  m.lsln.cn news 211874, section "4.3 消融实验".
 *
 * General rules for every call
 *   - Pointers marked "device" must point to device memory of the current
 *     CUDA device; "host" pointers to host memory.  The library keeps no
 *     pointer after the call returns and never frees caller memory.
 *   - All work is enqueued on `stream` (a cudaStream_t passed as void*, NULL =
 *     the legacy default stream).  No call synchronises the stream.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid argument returns CSA2_ERR_INVALID_ARG and launches nothing.
 *     Device-resident counts and positions (n_entries, q_pos, idx, pool) are
 *     clamped or treated as padding on the device; they never cause an
 *     out-of-bounds access.
 *   - A failed launch returns CSA2_ERR_CUDA; csa2_last_cuda_error() then gives
 *     the cudaError_t value.  No C++ exception crosses this interface.
 *
 * Data layout (row-major, all sizes in bytes unless stated):
 *   main latent row  : 512 channels -> 256 B of E2M1 codes (channel 2j in the
 *                      low nibble of byte j, 2j+1 in the high nibble) plus 32 B
 *                      of E4M3 scales, one per 16 channels (NVFP4 without the
 *                      second-level scale: [Blog] FP4 section, [Lsln] 4.3).
 *   indexer K row    : 64 channels -> 32 B codes + 4 B scales; the codes are
 *                      stored in the tiled order below (not row-major).
 *   indexer K codes  : entries in tiles of 128 (entry e = tile e / 128, row
 *                      e % 128); a tile's codes are 4096 contiguous bytes, and
 *                      half h (channels 32h .. 32h + 31, 16 B) of entry e is at
 *                        4096 (e / 128) + 256 ((e / 8) % 16) + 128 h + 16 (e % 8).
 *                      This is the tensor cores' shared-memory operand image of
 *                      a 128-row tile, so a tile moves with one bulk copy and a
 *                      block of 8 entries is 256 contiguous bytes.
 *   indexer K scales : row-major, 4 bytes per entry (blocks 0..3 in order).
 *   indexer Q        : per query [4 heads][32 B] codes + [4][4] scales.
 *   E2M1 code        : bit 3 sign, bits 2:1 exponent (bias 1), bit 0 mantissa.
 *   E4M3 byte        : "FN" variant, bias 7, no infinities, 0x7F/0xFF NaN
 *                      (NaN scale bytes are not valid input).
 *   SWA KV           : per token 512 E4M3 bytes and one fp32 scale (value =
 *                      e4m3 * scale): the sliding-window KV stays FP8 ([Jdon]).
 *   bf16             : IEEE bfloat16 bit patterns (uint16).
 */
#ifndef CSA2_C_ABI_H
#define CSA2_C_ABI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define CSA2_D 512          /* latent channels = attention head dim (K = V = latent) */
#define CSA2_H 16           /* attention heads per query */
#define CSA2_IH 4           /* indexer heads */
#define CSA2_ID 64          /* indexer head dim */
#define CSA2_BLOCK 8        /* positions per pool block ([Blog] Fig. 5) */
#define CSA2_MAX_K 2048     /* largest Top-K / pool size a call accepts */
#define CSA2_MAX_WINDOW 128 /* largest sliding window ([Blog]: n_win = 128) */

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,
    CSA2_ERR_UNSUPPORTED = 2,
    CSA2_ERR_WORKSPACE = 3,
    CSA2_ERR_CUDA = 4,
    CSA2_ERR_TIMEOUT = 5
} csa2_status;

/* Human-readable name of a status (static storage, never NULL). */
CSA2_API const char* csa2_status_str(csa2_status s);

/* The cudaError_t (as int) recorded by the last call that returned CSA2_ERR_CUDA
 * on this host thread, or 0. */
CSA2_API int csa2_last_cuda_error(void);

/*
 * Test hook for the device-side timeout path (the pages have no counterpart).
 * While enabled (enable != 0; process-wide, off by default), index calls that
 * run the per-share scoring kernel (csa2_index_topk and
 * csa2_index_topk_noalloc for more queries than one wave of clusters holds,
 * with fewer than 8 per batch row) announce their first copy stage on its
 * barrier but issue no copy, so the CTAs' bounded waits (2 s) run out: the call
 * sets its sticky error flag (read by csa2_device_status or
 * csa2_index_topk_noalloc_status) and its results are not valid.  Nothing
 * faults or hangs; the context stays usable.
 */
CSA2_API void csa2_test_starve_copies(int32_t enable);

/*
 * The shared global KV of one CSA2 layer group: the FP4 main latent and the FP4
 * indexer K, both written by the group's Full layer and borrowed by its
 * Reindex and Reuse layers ([Blog] "CSA2" section, Fig. 4).
 *   lat       device [B][cap][256]  E2M1 codes of the main latent
 *   lat_sc    device [B][cap][32]   E4M3 scales of the main latent
 *   ik        device [B][cap][32]   E2M1 codes of the indexer K (tiled order above;
 *                                   entry e of batch row b is cache entry b cap + e)
 *   ik_sc     device [B][cap][4]    E4M3 scales of the indexer K (row-major)
 *   n_entries device [B] int32      valid entries per batch row (clamped to [0, cap])
 *   cap       entries allocated per batch row: a positive multiple of 128
 *             (calls that read ik return CSA2_ERR_INVALID_ARG otherwise)
 *   m         tokens compressed into one entry: 1 (decoder) or 2 (encoder).
 *             Entry e covers tokens [m e, m e + m - 1] and is visible to the
 *             query at token p once complete: m e + m - 1 <= p.
 * All four byte arrays must be 16-byte aligned.
 */
typedef struct csa2_kv {
    uint8_t* lat;
    uint8_t* lat_sc;
    uint8_t* ik;
    uint8_t* ik_sc;
    const int32_t* n_entries;
    int64_t cap;
    int32_t m;
} csa2_kv;

/*
 * Step 1 -- NVFP4 quantisation ([Blog] FP4 section: E2M1 values, one E4M3
 * scale per 16 channels, applied after RoPE; [Lsln] 4.3: no global scale).
 * For each group of 16 channels: scale = E4M3 round-to-nearest-even
 * (saturating at 448) of the fp32 quotient amax / 6; each code is the E2M1
 * value nearest to x / scale (ties to the even code, saturating at 6) with the
 * sign of x; a group whose scale rounds to 0 is written as all-zero codes.
 *   x        device bf16 [rows][ch], 16-byte aligned
 *   rows     >= 0 (0 is a no-op)
 *   ch       multiple of 16, 16..4096
 *   codes    device u8 [out_rows][ch/2], 8-byte aligned; row r goes to row dst_rows[r] (or r)
 *   scales   device u8 [out_rows][ch/16]; same row mapping
 *   dst_rows device int64 [rows] or NULL: destination row of each input row
 *            (used to append one new entry per batch row into a [B][cap] cache);
 *            a destination outside [0, out_rows) is skipped
 *   out_rows rows of codes/scales (>= rows when dst_rows is NULL)
 */
CSA2_API csa2_status csa2_quant_nvfp4(const void* x, int64_t rows, int32_t ch, uint8_t* codes, uint8_t* scales,
                                      const int64_t* dst_rows, int64_t out_rows, void* stream);

/*
 * Indexer-K projection ([Blog] "CSA2" section: the indexer K is projected from
 * the main KV).  k = x W computed per output as an fp32 fused multiply-add
 * chain over the 512 input channels in ascending order (starting from +0),
 * then NVFP4-quantised exactly as csa2_quant_nvfp4 does (64 channels -> 32 B
 * codes + 4 B scales).
 *   x        device bf16 [rows][512] (post-RoPE latent rows), 16-byte aligned
 *   W        device fp32 [512][64], 16-byte aligned
 *   k_codes  device u8 [out_rows][32] (8-byte aligned) in the tiled indexer-K
 *            code order (output row r = cache entry r); k_scales device u8 [out_rows][4];
 *            row mapping as for csa2_quant_nvfp4; out_rows a multiple of 128
 *            (else CSA2_ERR_INVALID_ARG)
 */
CSA2_API csa2_status csa2_index_k_proj(const void* x, int64_t rows, const float* W, uint8_t* k_codes,
                                       uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows, void* stream);

/*
 * Append of new tokens: csa2_quant_nvfp4 of each latent row (ch = 512) into
 * the main-KV codes/scales and csa2_index_k_proj of the same row into the
 * indexer-K codes/scales, in one launch (same bytes as the two calls).
 * Arguments as for those two calls; x, W 16-byte aligned; lat_codes and
 * k_codes 8-byte aligned; both outputs use the same row mapping.
 */
CSA2_API csa2_status csa2_append_tokens(const void* x, int64_t rows, const float* W, uint8_t* lat_codes,
                                        uint8_t* lat_scales, uint8_t* k_codes, uint8_t* k_scales,
                                        const int64_t* dst_rows, int64_t out_rows, void* stream);

/*
 * Front end of new main-KV entries: RMSNorm and RoPE, then the append's
 * quantisation, in one launch ([Jdon] "缓存压缩真的是越大越好吗": the latent is
 * RMSNorm'd, so its L2 norm is at most about sqrt(512), and RoPE keeps that
 * norm; [Blog] FP4 section: the latent is quantised after RoPE; [Blog] "CSA2"
 * section: the indexer K is projected from the main KV).  For each row, in fp32
 * with one IEEE rounding per step:
 *   ss  = fused multiply-add chain of x_c * x_c over c = 0..511, from +0
 *   r   = 1 / sqrt(ss / 512 + eps);   n_c = (x_c * r) * w_c
 *   for k = 0..31, (a, b) = (n_{448+2k}, n_{449+2k}):
 *         a' = a cos_k - b sin_k;   b' = a sin_k + b cos_k   (products rounded first)
 *   y   = n rounded to bf16 (nearest, ties to even)
 * then the bytes csa2_append_tokens(y, ...) writes (NVFP4 latent; projected,
 * quantised indexer K).
 *   x         device bf16 [rows][512] pre-norm latent rows, 16-byte aligned
 *   rope_cos, rope_sin  device fp32 [rows][32]: cos and sin of each row's 32 angles
 *   norm_w    device fp32 [512] RMSNorm weight, or NULL for weight 1
 *   eps       RMSNorm epsilon (1e-6 in the synthetic workloads)
 *   W, lat_codes, lat_scales, k_codes, k_scales, dst_rows, out_rows: as for
 *             csa2_append_tokens (out_rows a multiple of 128)
 *   y_out     device bf16 [rows][512] (16-byte aligned) receiving y, or NULL
 */
CSA2_API csa2_status csa2_front_end(const void* x, int64_t rows, const float* rope_cos, const float* rope_sin,
                                   const float* norm_w, float eps, const float* W, uint8_t* lat_codes,
                                   uint8_t* lat_scales, uint8_t* k_codes, uint8_t* k_scales, const int64_t* dst_rows,
                                   int64_t out_rows, void* y_out, void* stream);

/*
 * Step 2 -- FP4 index scoring + Top-K ([Blog] "CSA2" section: a lightweight
 * indexer scores the causally visible compressed entries and keeps the Top-K,
 * K = 512; [Blog] FP4 section: FP4 indexer Q/K).
 * score(t) = sum_h w_h ReLU(q_h . k_t), evaluated in a fixed order:
 *   I[h][b] = integer dot product of the doubled E2M1 values of block b (16 ch)
 *   T[h][b] = I[h][b] * sq[h][b] * sk[b] / 4            (exact in fp32)
 *   d_h = ((T0 + T1) + T2) + T3 (fp32);  r_h = max(d_h, +0)
 *   score = ((w0 r0 + w1 r1) + w2 r2) + w3 r3 (fp32, each product rounded)
 * The Top-K is the first min(k, n_visible) entries in (score descending,
 * position ascending) order; their positions are written in ascending order
 * and the rest of the row is -1.
 *   q, q_sc       device u8 [B][Q][4][32], [B][Q][4][4]  FP4 indexer queries
 *   w             device fp32 [B][Q][4]                  head weights
 *   kv            host pointer to the group's KV (ik, ik_sc, n_entries, cap, m used)
 *   q_pos         device int32 [B][Q]  token position of each query (visibility)
 *   B, Q          >= 1 with B * Q <= 65535; k in [1, CSA2_MAX_K]
 *   idx_out       device int32 [B][Q][k]
 *   blockmax_out  device fp32 [B][Q][ceil(cap/8)] or NULL: the maximum score of
 *                 each block of 8 positions (visible positions only), -inf for
 *                 blocks with no visible position ([Blog] Fig. 5)
 *   ws, ws_bytes  device workspace of at least csa2_workspace_bytes(CSA2_OP_INDEX_TOPK, ...);
 *                 for more than 148 queries with at least 8 per batch row and
 *                 cap <= 262,144 (a prefill chunk, a replay) it also holds every
 *                 query's 16-bit key prefixes and 2,048-bin histogram (2 B per
 *                 query and entry + 8 KB per query)
 *                 bytes, zero-filled before its first use; every call leaves its
 *                 counters at zero again.  Calls that share a workspace must not
 *                 overlap on the GPU.  The int32 at byte offset
 *                 CSA2_STATUS_OFFSET(B, Q) of the workspace is a sticky error
 *                 flag: a device-side wait that ran out of time (2 s) sets it to 1
 *                 and the kernel winds down; the results of that call are not
 *                 valid.  The caller may read it after the stream completes.
 */
CSA2_API csa2_status csa2_index_topk(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv,
                            const int32_t* q_pos, int32_t B, int32_t Q, int32_t k, int32_t* idx_out,
                            float* blockmax_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 3a -- hierarchical sparse indexer, pool build ([Blog] "分层稀疏索引器",
 * Fig. 5: the first Full layer's scores build a shared candidate pool of at
 * most 2,048 blocks of 8 positions, blocks being chosen by maximum indexer
 * score).  Keeps the first min(max_blocks, visible blocks) blocks in (block
 * max descending, block id ascending) order, written as ascending block ids
 * padded with -1.
 *   blockmax   device fp32 [B][Q][ceil(kv->cap/8)] from csa2_index_topk
 *   kv         host pointer (n_entries, cap, m used)
 *   max_blocks in [1, CSA2_MAX_K]
 *   pool_out   device int32 [B][Q][max_blocks]
 *   ws         as for csa2_index_topk (CSA2_OP_POOL_BUILD)
 */
CSA2_API csa2_status csa2_pool_build(const float* blockmax, const csa2_kv* kv, const int32_t* q_pos, int32_t B, int32_t Q,
                            int32_t max_blocks, int32_t* pool_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 3b -- Reindex layer: Top-K inside the pool ([Blog] "分层稀疏索引器":
 * later Reindex layers select their Top-512 only inside the pool; [Blog] Fig. 4:
 * a Reindex layer re-scores the borrowed global KV with its own indexer Q).
 * Candidates are the visible positions 8b .. 8b+7 of every pool block b >= 0;
 * the score, order and output are those of csa2_index_topk.  Pool block ids
 * must be distinct; out-of-range ids are ignored.
 *   pool   device int32 [B][Q][P]
 *   ws     as above (CSA2_OP_POOL_TOPK)
 */
CSA2_API csa2_status csa2_pool_topk(const uint8_t* q, const uint8_t* q_sc, const float* w, const csa2_kv* kv,
                           const int32_t* pool, int32_t P, const int32_t* q_pos, int32_t B, int32_t Q, int32_t k,
                           int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Step 4 -- sparse attention over the selected FP4 entries and the layer's own
 * FP8 sliding-window KV ([Blog] "CSA2" section: Top-K sparse attention plus the
 * layer's own SWA KV; K = V = the dequantised latent) under the SWA Bounded
 * Replay mask ([Blog] FP4/SWA section: replaying from start s, the query at
 * token i sees SWA keys in [max(s, i - W + 1), i]).  One softmax runs jointly
 * over the main and SWA keys of each head:
 *   z_j = (q_h . k_j) * sm_scale, p = softmax(z), out_h = sum_j p_j v_j.
 *   q            device bf16 [B][Q][16][512], 16-byte aligned
 *   kv           host pointer (lat, lat_sc, n_entries, cap used)
 *   idx, k       device int32 [B][Q][k] main entries; -1 or out-of-range = padding; k in [0, CSA2_MAX_K]
 *   swa, swa_sc  device u8 [B][T][512] (16-byte aligned), fp32 [B][T]; row r holds token swa_pos0[b] + r
 *   swa_pos0     device int32 [B];  T >= 0
 *   window       W in [1, CSA2_MAX_WINDOW]
 *   replay_start device int32 [B] (s) or NULL (no replay bound)
 *   q_pos        device int32 [B][Q] token position i of each query
 *   sm_scale     softmax scale (1/sqrt(512) in the synthetic workloads)
 *   out          device bf16 [B][Q][16][512]; a query with no visible key gets zeros
 *   lse          device fp32 [B][Q][16] (natural-log sum-exp of z) or NULL
 *   ws           as above (CSA2_OP_SPARSE_ATTN)
 */
CSA2_API csa2_status csa2_sparse_attn(const void* q, const csa2_kv* kv, const int32_t* idx, int32_t k, const uint8_t* swa,
                             const float* swa_sc, const int32_t* swa_pos0, int32_t T, int32_t window,
                             const int32_t* replay_start, const int32_t* q_pos, int32_t B, int32_t Q,
                             float sm_scale, void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Workspace sizes.  `op` selects the call; the other arguments are those of the
 * call (k = Top-K or max_blocks; P = pool size for CSA2_OP_POOL_TOPK, else 0).
 * The sizes returned can exceed the minimum a call accepts: the largest decode
 * contexts (the index's order keys) and the Reindex layer of csa2_layer_step at
 * one CTA per query (its pool search's order keys, 4 bytes per pool entry) use
 * the extra space for a faster kernel, and take a slower one without it. */
typedef enum {
    CSA2_OP_INDEX_TOPK = 0,
    CSA2_OP_POOL_BUILD = 1,
    CSA2_OP_POOL_TOPK = 2,
    CSA2_OP_SPARSE_ATTN = 3,
    CSA2_OP_LAYER = 4
} csa2_op;
CSA2_API size_t csa2_workspace_bytes(csa2_op op, int32_t B, int32_t Q, int64_t cap, int32_t k, int32_t P);

/* Byte offset of the sticky device error flag in an index / pool workspace. */
#define CSA2_STATUS_OFFSET(B, Q) ((((size_t)(B) * (size_t)(Q) * 4u) + 255u) & ~(size_t)255u)

/*
 * Reads the sticky device error flag of an index / pool workspace used with
 * batch B and Q queries: waits for `stream` (this call synchronises, unlike the
 * others), returns CSA2_ERR_TIMEOUT if a device-side wait of a call on that
 * workspace ran out of time (its results are not valid), else CSA2_OK.  With
 * clear != 0 the flag is reset to 0 on `stream`.
 */
CSA2_API csa2_status csa2_device_status(void* ws, int32_t B, int32_t Q, int32_t clear, void* stream);

/*
 * Step 5 -- one CSA2 layer dispatched by its static mode ([Blog] "CSA2"
 * section, Fig. 4): FULL computes the group's main KV and indexer K for the new
 * entries and a fresh Top-K (and, if pool != NULL, builds the pool from this
 * layer's block maxima); REINDEX re-scores the borrowed KV inside the pool with
 * its own indexer Q; REUSE borrows the indices as well.  Every mode then runs
 * sparse attention with the layer's own Q and SWA KV.  A REINDEX layer's pool
 * must be one csa2_pool_build wrote (a FULL layer of this call with pool !=
 * NULL): its valid block ids ascending, which lets the search order and break
 * ties by pool slot; csa2_pool_topk takes a pool in any order.
 */
typedef enum { CSA2_MODE_FULL = 0, CSA2_MODE_REINDEX = 1, CSA2_MODE_REUSE = 2 } csa2_mode;

typedef struct csa2_layer_args {
    csa2_mode mode;
    const csa2_kv* kv;            /* host pointer to the group's shared KV */
    int32_t B, Q;
    const int32_t* q_pos;         /* device [B][Q] */
    /* FULL only: append new entries (skipped when n_new == 0) */
    const void* new_latent;       /* device bf16 [n_new][512] post-RoPE latent rows */
    int64_t n_new;
    const int64_t* new_rows;      /* device int64 [n_new]: destination row b*cap + e */
    const float* k_proj;          /* device fp32 [512][64] indexer-K projection */
    /* FULL and REINDEX: the layer's own indexer query */
    const uint8_t* iq;            /* device [B][Q][4][32] */
    const uint8_t* iq_sc;         /* device [B][Q][4][4] */
    const float* w;               /* device [B][Q][4] */
    /* shared selection state of the group */
    int32_t* idx;                 /* device [B][Q][k]: written by FULL/REINDEX, read by all */
    int32_t k;
    int32_t* pool;                /* device [B][Q][pool_blocks]: written by FULL (if not NULL), read by REINDEX */
    int32_t pool_blocks;
    float* blockmax;              /* device [B][Q][ceil(cap/8)] scratch for the FULL layer's pool build */
    /* the layer's own attention inputs */
    const void* q;                /* device bf16 [B][Q][16][512] */
    const uint8_t* swa;           /* device [B][T][512] */
    const float* swa_sc;          /* device [B][T] */
    const int32_t* swa_pos0;      /* device [B] */
    int32_t T, window;
    const int32_t* replay_start;  /* device [B] or NULL */
    float sm_scale;
    void* out;                    /* device bf16 [B][Q][16][512] */
    float* lse;                   /* device [B][Q][16] or NULL */
    void* ws;                     /* workspace of csa2_workspace_bytes(CSA2_OP_LAYER, B, Q, cap, k, pool_blocks) */
    size_t ws_bytes;
} csa2_layer_args;

CSA2_API csa2_status csa2_layer_step(const csa2_layer_args* a, void* stream);

/*
 * csa2_index_topk without a caller-provided workspace.  The pages have no
 * counterpart to this call: it exists for callers that cannot allocate device
 * memory -- hosts whose device memory is owned by their own pool allocator and
 * that hand out no scratch buffers, or latency-critical paths where a
 * cudaMalloc (which can synchronise the device) is not allowed.
 *
 * Arguments and results are those of csa2_index_topk, minus ws and ws_bytes.
 * The scratch the call needs (the merge counters and the candidate lists of
 * the per-query shares) lives in one static device array of
 * CSA2_NOALLOC_SCRATCH_BYTES inside this library; every GPU that loads the
 * library holds that array until the process exits.  The call never takes the
 * many-query path (whose key prefixes would not fit): a prefill-sized request
 * runs the per-share kernels, with the same results.  A call whose scratch
 * would exceed the array (csa2_workspace_bytes(CSA2_OP_INDEX_TOPK, B, Q, cap,
 * k, 0) without the many-query part, plus 256 bytes, > CSA2_NOALLOC_SCRATCH_BYTES)
 * returns CSA2_ERR_WORKSPACE and launches nothing.  The call allocates nothing:
 * no cudaMalloc, cudaFree or allocating library routine; it clears its error
 * flag and counters with cudaMemsetAsync on `stream` and then launches the
 * index kernels.
 *
 * Errors: argument and launch errors are returned at once, as by
 * csa2_index_topk.  A device-side wait that runs out of time (2 s) sets the
 * array's own sticky error flag (there is no workspace for csa2_device_status
 * to read); csa2_index_topk_noalloc_status reads it.  Each call clears the flag
 * before it launches, so the flag reports the last call.
 *
 * The first call on each device looks up the array's device address with that
 * device current (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls share the one array, which keeps the last call's contents:
 * calls that overlap on the GPU (other streams, other host threads) race on it
 * and must be ordered by the caller.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (4u << 20)

CSA2_API csa2_status csa2_index_topk_noalloc(const uint8_t* q, const uint8_t* q_sc, const float* w,
                                             const csa2_kv* kv, const int32_t* q_pos, int32_t B, int32_t Q,
                                             int32_t k, int32_t* idx_out, float* blockmax_out, void* stream);

/*
 * The error flag of the last csa2_index_topk_noalloc call on the current
 * device: waits for `stream` (this call synchronises), returns CSA2_ERR_TIMEOUT
 * if a device-side wait of that call ran out of time (its results are not
 * valid), else CSA2_OK; CSA2_ERR_CUDA if the copy fails.  With clear != 0 a set
 * flag is reset on `stream`.  Allocates nothing.
 */
CSA2_API csa2_status csa2_index_topk_noalloc_status(int32_t clear, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_C_ABI_H */
