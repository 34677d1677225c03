// score_cc.cuh -- the defined index score on CUDA cores, one entry at a time
// (integer dot products per 16-channel block, then the fixed fp32 order of
// csa2_index_topk).  Used where entries are few or scattered: the fallback
// select kernel and the exact re-scoring of a threshold bin's candidates.
#pragma once
#include "common.cuh"

namespace csa2 {

// The query side of the score, decoded once per CTA.
struct QReg {
    uint32_t q8[kIH][4][4];  // [head][block][word]: doubled E2M1 values as int8x4
    float f[kIH][4];         // sq[h][b] / 4
    float w[kIH];
};

__device__ __forceinline__ void load_query(QReg& R, const uint8_t* q, const uint8_t* qs, const float* w) {
#pragma unroll
    for (int h = 0; h < kIH; ++h) {
        const uint4* src = reinterpret_cast<const uint4*>(q + 32 * h);
        uint4 a = __ldg(src), c = __ldg(src + 1);
        uint32_t cw[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) e2m1x8_to_i8x2(cw[wi], R.q8[h][wi >> 1][2 * (wi & 1)], R.q8[h][wi >> 1][2 * (wi & 1) + 1]);
        uint32_t sw = *reinterpret_cast<const uint32_t*>(qs + 4 * h);
        float sf[4];
        e4m3x4_to_f32(sw, sf);
#pragma unroll
        for (int b = 0; b < 4; ++b) R.f[h][b] = sf[b] * 0.25f;
        R.w[h] = __ldg(w + h);
    }
}

// score = sum_h w_h ReLU(d_h) in the fixed order of csa2_index_topk.
__device__ __forceinline__ float entry_score(const QReg& R, uint4 c0, uint4 c1, uint32_t skw) {
    uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    uint32_t k8[4][4];
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) e2m1x8_to_i8x2(cw[wi], k8[wi >> 1][2 * (wi & 1)], k8[wi >> 1][2 * (wi & 1) + 1]);
    float sk[4];
    e4m3x4_to_f32(skw, sk);
    float score = 0.0f;
#pragma unroll
    for (int h = 0; h < kIH; ++h) {
        float d = 0.0f;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            int I = __dp4a((int)R.q8[h][b][0], (int)k8[b][0], 0);
            I = __dp4a((int)R.q8[h][b][1], (int)k8[b][1], I);
            I = __dp4a((int)R.q8[h][b][2], (int)k8[b][2], I);
            I = __dp4a((int)R.q8[h][b][3], (int)k8[b][3], I);
            float T = __fmul_rn((float)I, __fmul_rn(R.f[h][b], sk[b]));  // exact
            d = (b == 0) ? T : __fadd_rn(d, T);
        }
        float r = d > 0.0f ? d : 0.0f;
        float pr = __fmul_rn(R.w[h], r);
        score = (h == 0) ? pr : __fadd_rn(score, pr);
    }
    return score;
}

__device__ __forceinline__ float entry_score_at(const QReg& R, const uint8_t* ik, const uint8_t* iks, int64_t e) {
    const uint4 c0 = __ldg(reinterpret_cast<const uint4*>(ik + ik_code_off(e, 0)));
    const uint4 c1 = __ldg(reinterpret_cast<const uint4*>(ik + ik_code_off(e, 1)));
    const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(iks + ik_scale_off(e)));
    return entry_score(R, c0, c1, sw);
}

}  // namespace csa2
