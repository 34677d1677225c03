/*
 * csa2_oracle.h -- plain CPU reference of the CSA2 decode/prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  The product (the CUDA
 * library) never links, includes or calls it, and shares no code with it.
 *
 * Sources (three public web pages about the DeepSeek-V4.1-Flash report):
 *   [Blog]  "一个 token 只花 890 字节：DeepSeek-V4.1-Flash 把 KV 缓存压到了什么程度"
 *           (shibing624.github.io ai-paper-analysis), sections
 *           "CSA2：跨层复用，能借就不自己算" (Fig. 4),
 *           "分层稀疏索引器：让深层 indexer 别全文搜索" (Fig. 5),
 *           "FP4 与 SWA Bounded Replay：另外两刀".
 *   [Jdon]  "557亿参数只唤醒80亿！DeepSeek把AI记忆砍掉437倍还拿了第一！" (jdon.com),
 *           sections "三条路线打架" and "缓存压缩真的是越大越好吗".
 *   [Lsln]  m.lsln.cn news 211874, section "4.3 消融实验" and "五、相关工作".
 *
 * Conventions shared with the library only through the documented byte
 * formats (never through code):
 *   - E2M1 code: bit 3 sign, bits 2:1 exponent (bias 1), bit 0 mantissa.
 *     Channel 2j sits in the low nibble of byte j, channel 2j+1 in the high nibble.
 *   - E4M3 scale byte: "FN" variant, bias 7, no infinities, 0x7F/0xFF are NaN.
 *   - Main latent row: 512 channels -> 256 code bytes + 32 scale bytes.
 *   - Indexer K row: 64 channels -> 32 code bytes + 4 scale bytes.
 *   - Indexer Q: 4 heads x 64 channels -> [4][32] code bytes + [4][4] scales.
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* formats */
double orc_e2m1_value(unsigned code);
double orc_e4m3_value(unsigned byte);
unsigned orc_e4m3_encode(double v);
void orc_quant_nvfp4_f32(const float* x, int64_t rows, int ch, uint8_t* packed, uint8_t* scales);
void orc_quant_nvfp4_bf16(const uint16_t* x, int64_t rows, int ch, uint8_t* packed, uint8_t* scales);
void orc_dequant_nvfp4(const uint8_t* packed, const uint8_t* scales, int64_t rows, int ch, double* out);

/* indexer */
void orc_index_k_proj_f32(const uint16_t* x, int64_t rows, const float* W, float* out);
void orc_index_k_proj(const uint16_t* x, int64_t rows, const float* W, uint8_t* k_codes, uint8_t* k_scales);
float orc_index_score(const uint8_t* q, const uint8_t* qs, const float* w, const uint8_t* k, const uint8_t* ks);
int64_t orc_n_visible(int64_t q_pos, int64_t n_entries, int m);
void orc_index_topk(const uint8_t* q, const uint8_t* qs, const float* w,
                    const uint8_t* ik, const uint8_t* iks, const int32_t* n_entries, int64_t cap, int m,
                    const int32_t* q_pos, int B, int Q, int k, int32_t* idx_out,
                    float* blockmax_out, int64_t nb_cap);
void orc_pool_build(const float* blockmax, int64_t nb_cap, const int32_t* n_entries, int m,
                    const int32_t* q_pos, int B, int Q, int max_blocks, int32_t* pool_out);
void orc_pool_topk(const uint8_t* q, const uint8_t* qs, const float* w,
                   const uint8_t* ik, const uint8_t* iks, const int32_t* n_entries, int64_t cap, int m,
                   const int32_t* pool, int P, const int32_t* q_pos, int B, int Q, int k, int32_t* idx_out);

/* front end: RMSNorm + RoPE of a new latent (fp32 values, then bf16) */
void orc_front_end_f32(const uint16_t* x, int64_t rows, const float* cos_t, const float* sin_t, const float* w,
                       float eps, float* out);
void orc_front_end(const uint16_t* x, int64_t rows, const float* cos_t, const float* sin_t, const float* w,
                   float eps, uint16_t* y);

/* attention */
void orc_sparse_attn(const uint16_t* q, const uint8_t* lat, const uint8_t* lat_sc,
                     const int32_t* n_entries, int64_t cap, const int32_t* idx, int k,
                     const uint8_t* swa, const float* swa_sc, const int32_t* swa_pos0, int T,
                     int window, const int32_t* replay_start, const int32_t* q_pos,
                     int B, int Q, double sm_scale, double* out, double* lse);

#ifdef __cplusplus
}
#endif
#endif
