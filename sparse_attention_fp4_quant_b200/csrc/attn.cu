// attn.cu -- sparse attention over the Top-K FP4 main rows plus the layer's own
// FP8 sliding-window KV, under the SWA Bounded Replay mask.
//
// Split-K form, for query counts too large for one cluster per query
// (attn_cluster.cu serves the rest).  A CTA (8 warps) takes a split of the
// slot range in tiles of 64 keys.  Each tile is gathered into registers one
// tile ahead (its loads overlap the previous tile's math), dequantised to f16
// in swizzled shared memory (K = V), and S = Q K^T (8 keys per warp) and
// O += P V (64 dims per warp) run on warp-level tensor-core MMAs with the 16
// heads as the M dimension; the softmax is online across tiles.  P enters P V
// rounded to f16 (fp32 accumulation).  Splits of one query are merged by the
// last CTA to finish (atomic ticket).
#include "attn_common.cuh"

namespace csa2 {

constexpr int kAT = 256;      // threads per CTA (8 warps)
constexpr int kKT = 64;       // keys per tile
constexpr int kMaxSplits = (CSA2_MAX_K + CSA2_MAX_WINDOW + kKT - 1) / kKT;
constexpr int kMaxSplitMain = CSA2_MAX_K + kKT;   // main-row ids a split reads (its tiles' slots below k)

struct AttnSmem {
    uint8_t K[kKT * kRowB];   // 64 KB, 16-byte chunks XOR-swizzled by row & 7
    uint8_t Qs[kH * kRowB];   // 16 KB, same swizzle
    uint8_t P[kH * kKT * 2];  // 2 KB, f16 P, 8 chunks per row, same swizzle
    float kf[kKT];            // per-key factor (1 for FP4 rows, token scale for SWA)
    int kvalid[kKT];
    float red_max[8][kH];
    float red_sum[8][kH];
    float m_run[kH], l_run[kH], alpha[kH];
    float cw[kMaxSplits][kH];  // combine weights 2^(m_s - M) / L per split and head
    float qmax[kAT / 32];      // per-warp max |q|
    int last;
    int32_t eidx[kMaxSplitMain];   // this split's main-row ids, read once up front
};

__global__ void __launch_bounds__(kAT, 2) attn_kernel(AttnParams p) {
    pdl_enter();
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, qd = lane & 3;
    const int bq = blockIdx.y;
    const int split = blockIdx.x, S = gridDim.x;
    const int b = bq / p.Q;
    const int64_t i_pos = p.q_pos[bq];
    int64_t lo = i_pos - p.window + 1;
    if (p.replay_start && lo < (int64_t)p.replay_start[b]) lo = p.replay_start[b];
    const int64_t pos0 = p.swa_pos0[b];
    int64_t nmain = p.n_entries[b];
    if (nmain > p.cap) nmain = p.cap;
    float scale_log2 = p.sm_scale * 1.4426950408889634f;

    const uint32_t sK = (uint32_t)__cvta_generic_to_shared(sm.K);
    const uint32_t sQ = (uint32_t)__cvta_generic_to_shared(sm.Qs);
    const uint32_t sP = (uint32_t)__cvta_generic_to_shared(sm.P);

    const int ntiles = (p.slots_total + kKT - 1) / kKT;
    const int t0 = split * p.tiles_per_split;
    const int t1 = min(ntiles, t0 + p.tiles_per_split);
    // gather: key row and quarter of this thread; consecutive lanes take
    // consecutive rows so their swizzled 16-byte stores hit distinct banks.
    // The split's main-row ids go to shared memory first (one round trip for all
    // tiles), so a tile's row loads never wait on an id load.
    const int gr = tid & (kKT - 1), gq = tid >> 6;
    const int sm0 = t0 * kKT, sm1 = min(p.k, t1 * kKT);   // this split's main slots [sm0, sm1)
    {
        constexpr int kPer = (kMaxSplitMain + kAT - 1) / kAT;
        int32_t ev[kPer];   // every id load of the thread in flight before any is stored
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int s = sm0 + tid + kAT * j;
            ev[j] = s < sm1 ? (int32_t)ld_nc_u32(p.idx + (int64_t)bq * p.k + s) : -1;
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (sm0 + tid + kAT * j < sm1) sm.eidx[tid + kAT * j] = ev[j];
    }
    __syncthreads();

    RowQuarter rq;
    if (t0 < t1) fetch_quarter_id(p, b, t0 * kKT + gr, gq, sm.eidx, sm0, i_pos, lo, pos0, nmain, rq);

    // Q [16][512] bf16 -> f16 times a power-of-two prescale -> swizzled smem
    {
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (int64_t)bq * kH * kD);
        uint4 qv[(kH * kD / 8) / kAT];
        float qm = 0.0f;
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kAT; ++it) {
            qv[it] = __ldg(qsrc + it * kAT + tid);
            qm = fmaxf(qm, bf16x8_maxabs(qv[it]));
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xFFFFFFFFu, qm, o2));
        if (lane == 0) sm.qmax[warp] = qm;
        __syncthreads();
        qm = sm.qmax[0];
#pragma unroll
        for (int w = 1; w < kAT / 32; ++w) qm = fmaxf(qm, sm.qmax[w]);
        const int qe = q_prescale_exp(qm);
        const float qmul = __uint_as_float((uint32_t)(127 - qe) << 23);   // 2^-qe
        scale_log2 *= __uint_as_float((uint32_t)(127 + qe) << 23);       // the logits take 2^qe back
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kAT; ++it) {
            const int c = it * kAT + tid;  // 16-byte chunk id
            *reinterpret_cast<uint4*>(sm.Qs + swz(c >> 6, c & 63)) = bf16x8_to_f16(qv[it], qmul);
        }
    }
    if (tid < kH) {
        sm.m_run[tid] = -INFINITY;
        sm.l_run[tid] = 0.0f;
    }

    float o[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[n][j] = 0.0f;

    for (int tile = t0; tile < t1; ++tile) {
        store_quarter(sm.K, sm.kf, sm.kvalid, gr, gq, rq);
        __syncthreads();
        if (tile + 1 < t1)   // in flight meanwhile
            fetch_quarter_id(p, b, (tile + 1) * kKT + gr, gq, sm.eidx, sm0, i_pos, lo, pos0, nmain, rq);

        // ---- S = Q K^T for keys 8*warp .. +7 (two accumulator chains: even and odd k-steps) ----
        float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s4b[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 8
        for (int ks = 0; ks < kD / 16; ks += 2) {
            uint32_t a0, a1, a2, a3, b0, b1, c0, c1, c2, c3, d0, d1;
            const int key = 8 * warp + (lane & 7);
            ldsm_x4(sQ + swz(lane & 15, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
            ldsm_x2(sK + swz(key, 2 * ks + ((lane >> 3) & 1)), b0, b1);
            ldsm_x4(sQ + swz(lane & 15, 2 * ks + 2 + (lane >> 4)), c0, c1, c2, c3);
            ldsm_x2(sK + swz(key, 2 * ks + 2 + ((lane >> 3) & 1)), d0, d1);
            mma_f16(s4, a0, a1, a2, a3, b0, b1);
            mma_f16(s4b, c0, c1, c2, c3, d0, d1);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) s4[j] += s4b[j];
        // logits (log2 units); masked keys -> -inf
        const int key0 = 8 * warp + 2 * qd;
        const float f0 = sm.kf[key0], f1 = sm.kf[key0 + 1];
        const bool v0 = sm.kvalid[key0] != 0, v1 = sm.kvalid[key0 + 1] != 0;
        const float z00 = v0 ? s4[0] * f0 * scale_log2 : -INFINITY, z01 = v1 ? s4[1] * f1 * scale_log2 : -INFINITY;
        const float z10 = v0 ? s4[2] * f0 * scale_log2 : -INFINITY, z11 = v1 ? s4[3] * f1 * scale_log2 : -INFINITY;
        float mx0 = fmaxf(z00, z01), mx1 = fmaxf(z10, z11);
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o2));
        }
        if (qd == 0) {
            sm.red_max[warp][g] = mx0;
            sm.red_max[warp][g + 8] = mx1;
        }
        __syncthreads();
        float mt0 = sm.red_max[0][g], mt1 = sm.red_max[0][g + 8];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            mt0 = fmaxf(mt0, sm.red_max[w][g]);
            mt1 = fmaxf(mt1, sm.red_max[w][g + 8]);
        }
        const float mn0 = fmaxf(sm.m_run[g], mt0), mn1 = fmaxf(sm.m_run[g + 8], mt1);
        const float mu0 = (mn0 == -INFINITY) ? 0.0f : mn0, mu1 = (mn1 == -INFINITY) ? 0.0f : mn1;
        const float p00 = exp2f(z00 - mu0), p01 = exp2f(z01 - mu0), p10 = exp2f(z10 - mu1), p11 = exp2f(z11 - mu1);
        {
            const int chunk = key0 >> 3, within = (key0 & 7) * 2;
            const uint32_t off0 = g * 128 + ((chunk ^ (g & 7)) << 4) + within;
            const uint32_t off1 = (g + 8) * 128 + ((chunk ^ ((g + 8) & 7)) << 4) + within;
            const float u00 = p00 * f0, u01 = p01 * f1, u10 = p10 * f0, u11 = p11 * f1;
            *reinterpret_cast<__half2*>(sm.P + off0) = __floats2half2_rn(u00, u01);
            *reinterpret_cast<__half2*>(sm.P + off1) = __floats2half2_rn(u10, u11);
        }
        float sum0 = p00 + p01, sum1 = p10 + p11;
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
            sum0 += __shfl_xor_sync(0xFFFFFFFFu, sum0, o2);
            sum1 += __shfl_xor_sync(0xFFFFFFFFu, sum1, o2);
        }
        if (qd == 0) {
            sm.red_sum[warp][g] = sum0;
            sm.red_sum[warp][g + 8] = sum1;
        }
        __syncthreads();
        if (tid < kH) {
            float mt = sm.red_max[0][tid], ssum = 0.0f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                mt = fmaxf(mt, sm.red_max[w][tid]);
                ssum += sm.red_sum[w][tid];
            }
            const float mo = sm.m_run[tid];
            const float mn = fmaxf(mo, mt);
            const float al = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
            sm.alpha[tid] = al;
            sm.l_run[tid] = sm.l_run[tid] * al + ssum;
            sm.m_run[tid] = mn;
        }
        __syncthreads();

        // ---- O[:, 64 warp .. +63] = alpha O + P V ----
        {
            const float al0 = sm.alpha[g], al1 = sm.alpha[g + 8];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                o[n][0] *= al0;
                o[n][1] *= al0;
                o[n][2] *= al1;
                o[n][3] *= al1;
            }
#pragma unroll
            for (int kk = 0; kk < kKT / 16; ++kk) {
                uint32_t a0, a1, a2, a3;
                {
                    const int row = lane & 15, chunk = 2 * kk + (lane >> 4);
                    ldsm_x4(sP + (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)), a0, a1, a2, a3);
                }
                const int mi = lane >> 3;
                const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(sK + swz(key, 8 * warp + 2 * np + (mi >> 1)), b0, b1, b2, b3);
                    mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
                    mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        __syncthreads();
    }

    // ---- write the split's partial, or the final output ----
    const float LN2 = 0.6931471805599453f;
    if (S == 1) {
        const float l0 = sm.l_run[g], l1 = sm.l_run[g + 8];
        const float inv0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, inv1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
        uint16_t* out = p.out + (int64_t)bq * kH * kD;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int d = 64 * warp + 8 * n + 2 * qd;
            *reinterpret_cast<uint32_t*>(out + g * kD + d) = pack_bf16(o[n][0] * inv0, o[n][1] * inv0);
            *reinterpret_cast<uint32_t*>(out + (g + 8) * kD + d) = pack_bf16(o[n][2] * inv1, o[n][3] * inv1);
        }
        if (p.lse && tid < kH) {
            const float l = sm.l_run[tid];
            p.lse[(int64_t)bq * kH + tid] = l > 0.0f ? (sm.m_run[tid] + log2f(l)) * LN2 : -INFINITY;
        }
        return;
    }
    {
        float* po = p.part_o + ((int64_t)bq * S + split) * kH * kD;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int d = 64 * warp + 8 * n + 2 * qd;
            *reinterpret_cast<float2*>(po + g * kD + d) = make_float2(o[n][0], o[n][1]);
            *reinterpret_cast<float2*>(po + (g + 8) * kD + d) = make_float2(o[n][2], o[n][3]);
        }
        if (tid < kH) {
            float* pml = p.part_ml + (((int64_t)bq * S + split) * kH + tid) * 2;
            pml[0] = sm.m_run[tid];
            pml[1] = sm.l_run[tid];
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = (atomicAdd(&p.counters[bq], 1) == S - 1);
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    // combine the S partials: weight 2^(m_s - M) / L with L = sum_s l_s 2^(m_s - M)
    if (tid < kH) {
        float M = -INFINITY;
        for (int c = 0; c < S; ++c) M = fmaxf(M, __ldcg(p.part_ml + (((int64_t)bq * S + c) * kH + tid) * 2));
        const float Mu = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f;
        for (int c = 0; c < S; ++c) {
            const float* pml = p.part_ml + (((int64_t)bq * S + c) * kH + tid) * 2;
            const float wgt = exp2f(__ldcg(pml) - Mu);
            sm.cw[c][tid] = wgt;
            L += __ldcg(pml + 1) * wgt;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (int c = 0; c < S; ++c) sm.cw[c][tid] *= inv;
        if (p.lse) p.lse[(int64_t)bq * kH + tid] = L > 0.0f ? (Mu + log2f(L)) * LN2 : -INFINITY;
    }
    __syncthreads();
    {
        // thread owns 8 float4 of the [16][512] output: element 4 (tid + 256 j)
        constexpr int kV = kH * kD / 4 / kAT;   // 8
        float4 acc[kV];
#pragma unroll
        for (int j = 0; j < kV; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < S; ++c) {
            const float4* src = reinterpret_cast<const float4*>(p.part_o + ((int64_t)bq * S + c) * kH * kD);
#pragma unroll
            for (int j = 0; j < kV; ++j) {
                const int e4 = tid + kAT * j;
                const float wgt = sm.cw[c][(4 * e4) / kD];
                const float4 v = __ldcg(src + e4);
                acc[j].x += v.x * wgt;
                acc[j].y += v.y * wgt;
                acc[j].z += v.z * wgt;
                acc[j].w += v.w * wgt;
            }
        }
        uint16_t* out = p.out + (int64_t)bq * kH * kD;
#pragma unroll
        for (int j = 0; j < kV; ++j) {
            const int e4 = tid + kAT * j;
            *reinterpret_cast<uint2*>(out + 4 * e4) = make_uint2(pack_bf16(acc[j].x, acc[j].y), pack_bf16(acc[j].z, acc[j].w));
        }
    }
    if (tid == 0) p.counters[bq] = 0;
}

int attn_splits(int B, int Q, int k, int window, int* tiles_per_split) {
    int ntiles = (k + window + kKT - 1) / kKT;
    if (ntiles < 1) ntiles = 1;
    int64_t bq = (int64_t)B * Q;
    int64_t want = (2 * kSplitSMs) / (bq > 0 ? bq : 1);
    if (want < 1) want = 1;
    if (want > ntiles) want = ntiles;
    int tps = (int)((ntiles + want - 1) / want);
    int S = (ntiles + tps - 1) / tps;
    if (tiles_per_split) *tiles_per_split = tps;
    return S;
}

size_t attn_ws_bytes(int B, int Q, int k, int window) {
    // bound the split count over every window <= CSA2_MAX_WINDOW: S <= min(tiles, CTA budget)
    (void)window;
    int64_t bq = (int64_t)B * Q;
    int64_t want = (2 * kSplitSMs) / (bq > 0 ? bq : 1);
    if (want < 1) want = 1;
    int64_t ntiles_max = (k + CSA2_MAX_WINDOW + kKT - 1) / kKT;
    int64_t S = want < ntiles_max ? want : ntiles_max;
    size_t ubq = (size_t)bq;
    size_t bytes = align256(ubq * 4) + 256;   // counters, status word
    if (S > 1) bytes += align256(ubq * S * kH * kD * 4) + align256(ubq * S * kH * 2 * 4);
    return bytes;
}

void attn_carve_ws(AttnParams& p, int S, void* ws) {
    int64_t bq = (int64_t)p.B * p.Q;
    int64_t want = (2 * kSplitSMs) / (bq > 0 ? bq : 1);
    if (want < 1) want = 1;
    int64_t ntiles_max = (p.k + CSA2_MAX_WINDOW + kKT - 1) / kKT;
    int64_t Sb = want < ntiles_max ? want : ntiles_max;
    char* c = (char*)ws;
    p.counters = (int32_t*)c;
    c += align256((size_t)bq * 4);
    p.status = (int32_t*)c;
    c += 256;
    if (S > 1) {
        p.part_o = (float*)c;
        c += align256((size_t)bq * Sb * kH * kD * 4);
        p.part_ml = (float*)c;
    }
}

cudaError_t launch_attn(AttnParams& p, int S, cudaStream_t st) {
    static DeviceOnce attr;
    const int smem = (int)sizeof(AttnSmem);
    cudaError_t e = attr.run([&] { return cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
    if (e != cudaSuccess) return e;
    dim3 grid(S, p.B * p.Q);
    return launch_ex(attn_kernel, grid, dim3(kAT), smem, st, 0, p);
}

}  // namespace csa2
