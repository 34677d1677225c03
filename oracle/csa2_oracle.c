/*
 * csa2_oracle.c -- plain, single-threaded CPU reference of the CSA2 hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see csa2_oracle.h).  Written for clarity, not
 * speed: no blocking, no fusion, no reordering beyond what each definition
 * states.  Floating-point rules:
 *   - quantisation decisions are made exactly (comparisons in double of values
 *     that are exact in double);
 *   - the index score follows the fixed fp32 order stated at orc_index_score;
 *   - attention accumulates in double.
 * Build with -ffp-contract=off so that no multiply-add is fused behind our back.
 */
#include "csa2_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 512     /* main-KV latent channels ([Jdon] "缓存压缩真的是越大越好吗": 512-channel latent) */
#define ORC_H 16      /* attention heads of the synthetic workload */
#define ORC_IH 4      /* indexer heads */
#define ORC_ID 64     /* indexer head dim */
#define ORC_BLK 8     /* positions per pool block ([Blog] "分层稀疏索引器", Fig. 5: 2,048 blocks x 8) */

/* ------------------------------------------------------------------------ */
/* Formats.  [Blog] "FP4 与 SWA Bounded Replay": E2M1 values, one E4M3 scale  */
/* per 16 channels; [Lsln] 4.3: no second-level global scale.                */
/* ------------------------------------------------------------------------ */

/* E2M1: sign bit 3, exponent bits 2:1 with bias 1, mantissa bit 0.
 * exponent 0 is subnormal: value = mantissa * 0.5. */
double orc_e2m1_value(unsigned code) {
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* E4M3 "FN": sign bit 7, exponent bits 6:3 with bias 7, mantissa bits 2:0,
 * no infinities, S.1111.111 is NaN, largest finite 448. */
double orc_e4m3_value(unsigned byte) {
    unsigned s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative E4M3 to v >= 0; a tie goes to the code whose mantissa
 * LSB is 0; anything at or above 448 saturates to 448 (code 0x7E).
 * The positive codes 0x00..0x7E have increasing values, so a bisection finds
 * the code just below v and the two neighbours are compared exactly. */
unsigned orc_e4m3_encode(double v) {
    if (!(v > 0.0)) return 0u;
    if (v >= 448.0) return 0x7Eu;
    unsigned lo = 0u, hi = 0x7Eu;
    while (lo < hi) {
        unsigned mid = (lo + hi + 1u) / 2u;
        if (orc_e4m3_value(mid) <= v) lo = mid; else hi = mid - 1u;
    }
    double a = orc_e4m3_value(lo), b = orc_e4m3_value(lo + 1u);
    double da = v - a, db = b - v;          /* exact: v has <= 53 bits near a, b */
    if (da < db) return lo;
    if (db < da) return lo + 1u;
    return (lo & 1u) ? lo + 1u : lo;
}

/* The eight E2M1 magnitudes, in code order. */
static double e2m1_mag(unsigned i) { return orc_e2m1_value(i & 7u); }

/* NVFP4 quantisation of one group of 16 channels.
 * scale = nearest E4M3 of the fp32 quotient amax / 6 (6 = largest E2M1
 * magnitude); each channel takes the E2M1 magnitude nearest to |x| / scale
 * (ties to the even code, above 6 saturates to 6) and the sign of x.
 * A zero scale (all-zero or vanishing group) writes all codes as 0x0. */
static void quant_group16(const float* x, unsigned* codes, unsigned* scale_byte) {
    float amax = 0.0f;
    for (int j = 0; j < 16; ++j) {
        float a = fabsf(x[j]);
        if (a > amax) amax = a;
    }
    float quot = amax / 6.0f;                       /* IEEE fp32 division */
    unsigned sc = orc_e4m3_encode((double)quot);
    double s = orc_e4m3_value(sc);
    *scale_byte = sc;
    for (int j = 0; j < 16; ++j) {
        if (s == 0.0) { codes[j] = 0u; continue; }
        double ax = fabs((double)x[j]);
        unsigned mag = 7u;
        for (unsigned i = 0; i < 7u; ++i) {
            double lo = e2m1_mag(i) * s, hi = e2m1_mag(i + 1u) * s;   /* exact products */
            if (ax < hi) {
                if (ax < lo) { mag = i; break; }      /* only for i == 0, ax < 0 impossible */
                double dlo = ax - lo, dhi = hi - ax;  /* exact */
                if (dlo < dhi) mag = i;
                else if (dhi < dlo) mag = i + 1u;
                else mag = (i & 1u) ? i + 1u : i;     /* tie: even code */
                break;
            }
        }
        unsigned sign = signbit(x[j]) ? 8u : 0u;
        codes[j] = sign | mag;
    }
}

void orc_quant_nvfp4_f32(const float* x, int64_t rows, int ch, uint8_t* packed, uint8_t* scales) {
    int groups = ch / 16;
    for (int64_t r = 0; r < rows; ++r) {
        const float* xr = x + r * ch;
        for (int g = 0; g < groups; ++g) {
            unsigned codes[16], sc;
            quant_group16(xr + 16 * g, codes, &sc);
            scales[r * groups + g] = (uint8_t)sc;
            for (int j = 0; j < 8; ++j)
                packed[r * (ch / 2) + 8 * g + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void orc_quant_nvfp4_bf16(const uint16_t* x, int64_t rows, int ch, uint8_t* packed, uint8_t* scales) {
    float buf[16];
    int groups = ch / 16;
    for (int64_t r = 0; r < rows; ++r) {
        for (int g = 0; g < groups; ++g) {
            for (int j = 0; j < 16; ++j) buf[j] = bf16_to_f32(x[r * ch + 16 * g + j]);
            unsigned codes[16], sc;
            quant_group16(buf, codes, &sc);
            scales[r * groups + g] = (uint8_t)sc;
            for (int j = 0; j < 8; ++j)
                packed[r * (ch / 2) + 8 * g + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

/* value = e2m1(code) * e4m3(scale): [Blog] "FP4 与 SWA Bounded Replay" (the cached
 * value is dequantised before attention). */
void orc_dequant_nvfp4(const uint8_t* packed, const uint8_t* scales, int64_t rows, int ch, double* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int c = 0; c < ch; ++c) {
            uint8_t byte = packed[r * (ch / 2) + c / 2];
            unsigned code = (c & 1) ? (byte >> 4) : (byte & 15u);
            out[r * ch + c] = orc_e2m1_value(code) * orc_e4m3_value(scales[r * (ch / 16) + c / 16]);
        }
}

/* ------------------------------------------------------------------------ */
/* Front end of a new main-KV latent.  [Jdon] "缓存压缩真的是越大越好吗": the   */
/* latent is RMSNorm'd (weight at most about 1, so its L2 norm is at most      */
/* about sqrt(512)) and RoPE preserves that norm; [Blog] "FP4 与 SWA Bounded     */
/* Replay" and [Lsln] 4.3: it is quantised after RoPE.  The fp32 order below is */
/* this implementation's reading (the pages give none):                         */
/*   ss   = fused multiply-add chain of x_c * x_c over c = 0..511 from +0       */
/*   r    = 1 / sqrt(ss / 512 + eps)   (each step one IEEE fp32 rounding)       */
/*   n_c  = (x_c * r) * w_c            (two rounded products)                   */
/*   RoPE on the pairs (448 + 2k, 449 + 2k), k = 0..31, with the caller's       */
/*   cos_k, sin_k:  a' = a cos - b sin,  b' = a sin + b cos  (products rounded, */
/*   then one rounded add / subtract)                                           */
/*   y_c  = n_c rounded to bf16 (nearest, ties to even)                         */
/* ------------------------------------------------------------------------ */

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));  /* inf / nan */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

void orc_front_end_f32(const uint16_t* x, int64_t rows, const float* cos_t, const float* sin_t, const float* w,
                       float eps, float* out) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * ORC_D;
        float ss = 0.0f;
        for (int c = 0; c < ORC_D; ++c) {
            float v = bf16_to_f32(xr[c]);
            ss = fmaf(v, v, ss);
        }
        float mean = ss / 512.0f;
        float t = mean + eps;
        float s = sqrtf(t);
        float inv = 1.0f / s;
        float* o = out + r * ORC_D;
        for (int c = 0; c < ORC_D; ++c) {
            float n = bf16_to_f32(xr[c]) * inv;
            o[c] = n * (w ? w[c] : 1.0f);
        }
        for (int k = 0; k < 32; ++k) {
            float a = o[448 + 2 * k], b = o[449 + 2 * k];
            float cs = cos_t[r * 32 + k], sn = sin_t[r * 32 + k];
            float ac = a * cs, bs = b * sn, as = a * sn, bc = b * cs;   /* separate roundings: no contraction */
            o[448 + 2 * k] = ac - bs;
            o[449 + 2 * k] = as + bc;
        }
    }
}

void orc_front_end(const uint16_t* x, int64_t rows, const float* cos_t, const float* sin_t, const float* w,
                   float eps, uint16_t* y) {
    float buf[ORC_D];
    for (int64_t r = 0; r < rows; ++r) {
        orc_front_end_f32(x + r * ORC_D, 1, cos_t + r * 32, sin_t + r * 32, w, eps, buf);
        for (int c = 0; c < ORC_D; ++c) y[r * ORC_D + c] = f32_to_bf16_rne(buf[c]);
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer.  [Blog] "CSA2" section: a lightweight indexer scores the main KV  */
/* with indexer Q/K and keeps the Top-K (512); the indexer K is projected     */
/* from the main KV.  [Blog] "FP4 与 SWA Bounded Replay": indexer Q/K in FP4.  */
/* ------------------------------------------------------------------------ */

/* k[j] = sum_c x[c] * W[c][j], as an fp32 fused multiply-add chain over c in
 * ascending order starting from +0 (x is the post-RoPE bf16 latent). */
void orc_index_k_proj_f32(const uint16_t* x, int64_t rows, const float* W, float* out) {
    for (int64_t r = 0; r < rows; ++r) {
        float acc[ORC_ID];
        for (int j = 0; j < ORC_ID; ++j) acc[j] = 0.0f;
        for (int c = 0; c < ORC_D; ++c) {
            float xc = bf16_to_f32(x[r * ORC_D + c]);
            for (int j = 0; j < ORC_ID; ++j) acc[j] = fmaf(xc, W[c * ORC_ID + j], acc[j]);
        }
        for (int j = 0; j < ORC_ID; ++j) out[r * ORC_ID + j] = acc[j];
    }
}

void orc_index_k_proj(const uint16_t* x, int64_t rows, const float* W, uint8_t* k_codes, uint8_t* k_scales) {
    float kf[ORC_ID];
    for (int64_t r = 0; r < rows; ++r) {
        orc_index_k_proj_f32(x + r * ORC_D, 1, W, kf);
        orc_quant_nvfp4_f32(kf, 1, ORC_ID, k_codes + r * (ORC_ID / 2), k_scales + r * (ORC_ID / 16));
    }
}

static unsigned nib(const uint8_t* packed, int c) {
    uint8_t byte = packed[c / 2];
    return (c & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
}

/* score = sum_h w_h * ReLU(q_h . k) over the 4 indexer heads, in this fixed order:
 *   I[h][b] = sum over the 16 channels of block b of (2 q)(2 k)   (exact integer)
 *   T[h][b] = I[h][b] * sq[h][b] * sk[b] / 4                      (exact in fp32)
 *   d_h     = ((T0 + T1) + T2) + T3                               (fp32 adds)
 *   r_h     = d_h > 0 ? d_h : +0
 *   score   = ((w0 r0 + w1 r1) + w2 r2) + w3 r3                   (fp32, products rounded)
 * Ties between equal scores are broken toward the lower position by the caller. */
float orc_index_score(const uint8_t* q, const uint8_t* qs, const float* w, const uint8_t* k, const uint8_t* ks) {
    float score = 0.0f;
    for (int h = 0; h < ORC_IH; ++h) {
        float d = 0.0f;
        for (int b = 0; b < 4; ++b) {
            long I = 0;
            for (int j = 0; j < 16; ++j) {
                int c = 16 * b + j;
                long qi = (long)(2.0 * orc_e2m1_value(nib(q + h * 32, c)));
                long ki = (long)(2.0 * orc_e2m1_value(nib(k, c)));
                I += qi * ki;
            }
            double T = (double)I * orc_e4m3_value(qs[h * 4 + b]) * orc_e4m3_value(ks[b]) * 0.25;
            float Tf = (float)T;                          /* exact */
            d = (b == 0) ? Tf : d + Tf;
        }
        float r = d > 0.0f ? d : 0.0f;
        float p = w[h] * r;
        score = (h == 0) ? p : score + p;
    }
    return score;
}

/* Causal visibility.  An entry compresses m consecutive tokens; entry e covers
 * tokens [m e, m e + m - 1] and is visible to the query at token p once it is
 * complete (m e + m - 1 <= p).  [Blog] "CSA2" section: the decoder uses m = 1,
 * the encoder m = 2. */
int64_t orc_n_visible(int64_t q_pos, int64_t n_entries, int m) {
    int64_t v = (q_pos + 1) / (m > 0 ? m : 1);
    if (v > n_entries) v = n_entries;
    if (v < 0) v = 0;
    return v;
}

typedef struct { float s; int32_t p; } scored_t;

/* descending score, ascending position on ties (-0 and +0 compare equal) */
static int cmp_scored(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->p < y->p) ? -1 : (x->p > y->p);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y);
}

/* Keep the first min(k, n) items in (score desc, position asc) order and
 * write their positions in ascending order, padding with -1 up to k. */
static void topk_positions(scored_t* items, int64_t n, int k, int32_t* out) {
    qsort(items, (size_t)n, sizeof(scored_t), cmp_scored);
    int64_t keep = n < k ? n : k;
    for (int64_t i = 0; i < keep; ++i) out[i] = items[i].p;
    qsort(out, (size_t)keep, sizeof(int32_t), cmp_i32);
    for (int64_t i = keep; i < k; ++i) out[i] = -1;
}

void orc_index_topk(const uint8_t* q, const uint8_t* qs, const float* w,
                    const uint8_t* ik, const uint8_t* iks, const int32_t* n_entries, int64_t cap, int m,
                    const int32_t* q_pos, int B, int Q, int k, int32_t* idx_out,
                    float* blockmax_out, int64_t nb_cap) {
    scored_t* items = (scored_t*)malloc(sizeof(scored_t) * (size_t)(cap > 0 ? cap : 1));
    for (int b = 0; b < B; ++b)
        for (int qi = 0; qi < Q; ++qi) {
            int64_t bq = (int64_t)b * Q + qi;
            int64_t nvis = orc_n_visible(q_pos[bq], n_entries[b], m);
            for (int64_t t = 0; t < nvis; ++t) {
                items[t].s = orc_index_score(q + bq * 128, qs + bq * 16, w + bq * 4,
                                             ik + ((int64_t)b * cap + t) * 32, iks + ((int64_t)b * cap + t) * 4);
                items[t].p = (int32_t)t;
            }
            if (blockmax_out) {
                for (int64_t j = 0; j < nb_cap; ++j) {
                    float mx = -INFINITY;
                    for (int64_t t = j * ORC_BLK; t < (j + 1) * ORC_BLK && t < nvis; ++t)
                        if (items[t].s > mx) mx = items[t].s;
                    blockmax_out[bq * nb_cap + j] = mx;
                }
            }
            topk_positions(items, nvis, k, idx_out + bq * k);
        }
    free(items);
}

/* ------------------------------------------------------------------------ */
/* Hierarchical sparse indexer.  [Blog] "分层稀疏索引器", Fig. 5: the first    */
/* Full layer builds a shared candidate pool of at most 2,048 blocks x 8       */
/* positions, the blocks being chosen by maximum indexer score; later Reindex  */
/* layers select their Top-512 only inside the pool.                           */
/* ------------------------------------------------------------------------ */

void orc_pool_build(const float* blockmax, int64_t nb_cap, const int32_t* n_entries, int m,
                    const int32_t* q_pos, int B, int Q, int max_blocks, int32_t* pool_out) {
    scored_t* items = (scored_t*)malloc(sizeof(scored_t) * (size_t)(nb_cap > 0 ? nb_cap : 1));
    for (int b = 0; b < B; ++b)
        for (int qi = 0; qi < Q; ++qi) {
            int64_t bq = (int64_t)b * Q + qi;
            int64_t nvis = orc_n_visible(q_pos[bq], n_entries[b], m);
            int64_t nblk = (nvis + ORC_BLK - 1) / ORC_BLK;
            if (nblk > nb_cap) nblk = nb_cap;
            for (int64_t j = 0; j < nblk; ++j) {
                items[j].s = blockmax[bq * nb_cap + j];
                items[j].p = (int32_t)j;
            }
            topk_positions(items, nblk, max_blocks, pool_out + bq * max_blocks);
        }
    free(items);
}

void orc_pool_topk(const uint8_t* q, const uint8_t* qs, const float* w,
                   const uint8_t* ik, const uint8_t* iks, const int32_t* n_entries, int64_t cap, int m,
                   const int32_t* pool, int P, const int32_t* q_pos, int B, int Q, int k, int32_t* idx_out) {
    scored_t* items = (scored_t*)malloc(sizeof(scored_t) * (size_t)P * ORC_BLK + 1);
    for (int b = 0; b < B; ++b)
        for (int qi = 0; qi < Q; ++qi) {
            int64_t bq = (int64_t)b * Q + qi;
            int64_t nvis = orc_n_visible(q_pos[bq], n_entries[b], m);
            int64_t n = 0;
            for (int i = 0; i < P; ++i) {
                int32_t blk = pool[bq * P + i];
                if (blk < 0) continue;
                for (int64_t t = (int64_t)blk * ORC_BLK; t < (int64_t)blk * ORC_BLK + ORC_BLK; ++t) {
                    if (t >= nvis) break;
                    items[n].s = orc_index_score(q + bq * 128, qs + bq * 16, w + bq * 4,
                                                 ik + ((int64_t)b * cap + t) * 32, iks + ((int64_t)b * cap + t) * 4);
                    items[n].p = (int32_t)t;
                    ++n;
                }
            }
            topk_positions(items, n, k, idx_out + bq * k);
        }
    free(items);
}

/* ------------------------------------------------------------------------ */
/* Sparse attention.  [Blog] "CSA2" section: softmax attention over the        */
/* Top-K main entries plus the layer's own sliding-window KV (K = V = latent). */
/* [Blog] "FP4 与 SWA Bounded Replay": when replaying from start s, the query  */
/* at i sees SWA keys in [max(s, i - W + 1), i].  [Jdon] "缓存压缩真的是越大越好吗": */
/* SWA KV stays in FP8 (here E4M3 with one fp32 scale per token).              */
/* ------------------------------------------------------------------------ */

void orc_sparse_attn(const uint16_t* q, const uint8_t* lat, const uint8_t* lat_sc,
                     const int32_t* n_entries, int64_t cap, const int32_t* idx, int k,
                     const uint8_t* swa, const float* swa_sc, const int32_t* swa_pos0, int T,
                     int window, const int32_t* replay_start, const int32_t* q_pos,
                     int B, int Q, double sm_scale, double* out, double* lse) {
    int maxkeys = k + (T > 0 ? T : 0);
    double* keys = (double*)malloc(sizeof(double) * (size_t)(maxkeys > 0 ? maxkeys : 1) * ORC_D);
    double* z = (double*)malloc(sizeof(double) * (size_t)(maxkeys > 0 ? maxkeys : 1));
    for (int b = 0; b < B; ++b)
        for (int qi = 0; qi < Q; ++qi) {
            int64_t bq = (int64_t)b * Q + qi;
            int nk = 0;
            /* main rows chosen by the indexer; -1 (or any out-of-range value) is padding */
            for (int j = 0; j < k; ++j) {
                int32_t t = idx[bq * k + j];
                if (t < 0 || t >= n_entries[b]) continue;
                orc_dequant_nvfp4(lat + ((int64_t)b * cap + t) * (ORC_D / 2),
                                  lat_sc + ((int64_t)b * cap + t) * (ORC_D / 16), 1, ORC_D, keys + (int64_t)nk * ORC_D);
                ++nk;
            }
            /* own sliding window under the Bounded Replay mask */
            int64_t i = q_pos[bq];
            int64_t lo = i - window + 1;
            if (replay_start && lo < replay_start[b]) lo = replay_start[b];
            for (int64_t tau = lo; tau <= i; ++tau) {
                int64_t r = tau - swa_pos0[b];
                if (r < 0 || r >= T) continue;
                double sc = (double)swa_sc[(int64_t)b * T + r];
                for (int d = 0; d < ORC_D; ++d)
                    keys[(int64_t)nk * ORC_D + d] = orc_e4m3_value(swa[((int64_t)b * T + r) * ORC_D + d]) * sc;
                ++nk;
            }
            for (int h = 0; h < ORC_H; ++h) {
                const uint16_t* qh = q + (bq * ORC_H + h) * ORC_D;
                double* oh = out + (bq * ORC_H + h) * ORC_D;
                for (int d = 0; d < ORC_D; ++d) oh[d] = 0.0;
                if (nk == 0) {
                    if (lse) lse[bq * ORC_H + h] = -INFINITY;
                    continue;
                }
                double zmax = -INFINITY;
                for (int j = 0; j < nk; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < ORC_D; ++d) acc += (double)bf16_to_f32(qh[d]) * keys[(int64_t)j * ORC_D + d];
                    z[j] = acc * sm_scale;
                    if (z[j] > zmax) zmax = z[j];
                }
                double l = 0.0;
                for (int j = 0; j < nk; ++j) {
                    z[j] = exp(z[j] - zmax);
                    l += z[j];
                }
                for (int j = 0; j < nk; ++j) {
                    double p = z[j] / l;
                    for (int d = 0; d < ORC_D; ++d) oh[d] += p * keys[(int64_t)j * ORC_D + d];
                }
                if (lse) lse[bq * ORC_H + h] = zmax + log(l);
            }
        }
    free(keys);
    free(z);
}
