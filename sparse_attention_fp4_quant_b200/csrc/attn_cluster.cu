// attn_cluster.cu -- csa2_sparse_attn for decode-sized query counts: one
// thread-block cluster of C CTAs per query.
//
// CTA r of the cluster takes the key slots [r * n, (r + 1) * n) of its query
// (n <= 160, a multiple of 16; slots as in attn_common.cuh) and gathers them
// all at once, so a CTA waits on global memory once instead of once per tile.
// The rows are dequantised to bf16 in swizzled shared memory (K = V); with the
// 16 heads as the M dimension, S = Q K^T runs on warp-level tensor-core MMAs
// (8 keys per warp and tile), then the CTA's own softmax (max and sum over its
// keys), then O_r = P V (32 dims per warp; P as a rounded bf16 term plus its
// bf16 remainder).  The partial results meet in distributed shared memory:
// each CTA publishes O_r (fp32) and its per-head (max, sum); CTA r then forms
// dims [r * 512 / C, (r + 1) * 512 / C) of the output as
//   sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c,   M = max_c m_c,
// and writes them as bf16.  No partials go to global memory and no CTA waits
// for a ticket.
#include "attn_common.cuh"
#include "cluster.cuh"

namespace csa2 {
namespace {

constexpr int kCT = 512;                      // threads per CTA (16 warps)
constexpr int kCW = kCT / 32;
constexpr int kMaxKeys = 160;                 // key slots per CTA
constexpr int kPStride = kMaxKeys * 2 + 16;   // bytes per head row of P (conflict-free ldmatrix)
constexpr int kOStride = kD + 4;              // floats per head row of the partial O (conflict-free stores)
static_assert(kMaxKeys % 16 == 0, "keys per CTA");
static_assert(kH * kOStride * 4 <= kMaxKeys * kRowB, "partial O fits the key buffer");

struct ClAttnSmem {
    uint8_t K[kMaxKeys * kRowB];   // bf16 keys (= values), swizzled; afterwards the fp32 partial O [16][kOStride]
    uint8_t Qs[kH * kRowB];        // bf16 query, swizzled
    uint8_t P[kH * kPStride];      // bf16 P (rounded), [head][key]
    uint8_t Pl[kH * kPStride];     // bf16 remainder P - rounded(P)
    float kf[kMaxKeys];            // per-key factor (1 for FP4 rows, token scale for SWA)
    int kvalid[kMaxKeys];
    float red[kCW][kH];
    float m_loc[kH];
    alignas(16) float ml[kH][2];   // this CTA's (max, sum) per head (log2 units), read by the cluster
    float cw[16][kH];              // combine weight of rank c for head h (for this CTA's output slice)
};

__global__ void __launch_bounds__(kCT, 1) attn_cluster_kernel(AttnParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ClAttnSmem& sm = *reinterpret_cast<ClAttnSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, qd = lane & 3;
    const uint32_t rank = cl::rank(), C = cl::ctas();
    const int bq = blockIdx.y;
    const int b = bq / p.Q;
    const int64_t i_pos = p.q_pos[bq];
    int64_t lo = i_pos - p.window + 1;
    if (p.replay_start && lo < (int64_t)p.replay_start[b]) lo = p.replay_start[b];
    const int64_t pos0 = p.swa_pos0[b];
    int64_t nmain = p.n_entries[b];
    if (nmain > p.cap) nmain = p.cap;
    const float scale_log2 = p.sm_scale * 1.4426950408889634f;

    // this CTA's slots [s0, s0 + nk), padded to n16 (dead slots past nk)
    const int s0 = min(p.slots_total, (int)rank * p.keys_per_cta);
    const int nk = min(p.slots_total, s0 + p.keys_per_cta) - s0;
    const int n16 = (nk + 15) & ~15;

    const uint32_t sK = (uint32_t)__cvta_generic_to_shared(sm.K);
    const uint32_t sQ = (uint32_t)__cvta_generic_to_shared(sm.Qs);
    const uint32_t sP = (uint32_t)__cvta_generic_to_shared(sm.P);
    const uint32_t sPl = (uint32_t)__cvta_generic_to_shared(sm.Pl);

    // ---- gather: row quarter u = r + n16 * qq (consecutive lanes, consecutive rows)
    {
        constexpr int kPer = (kMaxKeys * 4 + kCT - 1) / kCT;   // 2
        RowQuarter rq[kPer];
        int rr[kPer], qs[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = tid + kCT * j;
            rq[j].kind = 0;
            rr[j] = -1;
            if (u < 4 * n16) {
                rr[j] = u % n16;
                qs[j] = u / n16;
                const int slot = rr[j] < nk ? s0 + rr[j] : p.slots_total;   // past nk: dead
                fetch_quarter(p, bq, b, slot, qs[j], i_pos, lo, pos0, nmain, rq[j]);
            }
        }
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (int64_t)bq * kH * kD);
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) {
            const int c = it * kCT + tid;   // 16-byte chunk id
            const int row = c >> 6, ch = c & 63;
            *reinterpret_cast<uint4*>(sm.Qs + swz(row, ch)) = __ldg(qsrc + c);
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (rr[j] >= 0) store_quarter(sm.K, sm.kf, sm.kvalid, rr[j], qs[j], rq[j]);
    }
    __syncthreads();

    // ---- S = Q K^T: warp w takes key tiles w and w + 16 (8 keys each)
    const int nt = n16 >> 3;
    const bool has0 = warp < nt, has1 = warp + kCW < nt;
    float s4[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (has0) {
        const int key = 8 * warp + (lane & 7);
#pragma unroll 4
        for (int ks = 0; ks < kD / 16; ++ks) {
            uint32_t a0, a1, a2, a3, b0, b1;
            ldsm_x4(sQ + swz(lane & 15, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
            ldsm_x2(sK + swz(key, 2 * ks + ((lane >> 3) & 1)), b0, b1);
            mma_bf16(s4[0], a0, a1, a2, a3, b0, b1);
            if (has1) {
                ldsm_x2(sK + swz(key + 8 * kCW, 2 * ks + ((lane >> 3) & 1)), b0, b1);
                mma_bf16(s4[1], a0, a1, a2, a3, b0, b1);
            }
        }
    }
    // logits (log2 units), masked keys -> -inf; z[t][0..3] = (g, key0), (g, key0+1), (g+8, key0), (g+8, key0+1)
    float z[2][4], f[2][2];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const bool has = t == 0 ? has0 : has1;
        const int key0 = 8 * (warp + kCW * t) + 2 * qd;
        f[t][0] = has ? sm.kf[key0] : 0.0f;
        f[t][1] = has ? sm.kf[key0 + 1] : 0.0f;
        const bool v0 = has && sm.kvalid[key0] != 0, v1 = has && sm.kvalid[key0 + 1] != 0;
        z[t][0] = v0 ? s4[t][0] * f[t][0] * scale_log2 : -INFINITY;
        z[t][1] = v1 ? s4[t][1] * f[t][1] * scale_log2 : -INFINITY;
        z[t][2] = v0 ? s4[t][2] * f[t][0] * scale_log2 : -INFINITY;
        z[t][3] = v1 ? s4[t][3] * f[t][1] * scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(z[t][0], z[t][1]));
        mx1 = fmaxf(mx1, fmaxf(z[t][2], z[t][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o2));
    }
    if (qd == 0) {
        sm.red[warp][g] = mx0;
        sm.red[warp][g + 8] = mx1;
    }
    __syncthreads();
    if (tid < kH) {
        float m = sm.red[0][tid];
#pragma unroll
        for (int w = 1; w < kCW; ++w) m = fmaxf(m, sm.red[w][tid]);
        sm.m_loc[tid] = m;
    }
    __syncthreads();
    {
        const float m0 = sm.m_loc[g], m1 = sm.m_loc[g + 8];
        const float mu0 = (m0 == -INFINITY) ? 0.0f : m0, mu1 = (m1 == -INFINITY) ? 0.0f : m1;
        float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const bool has = t == 0 ? has0 : has1;
            if (!has) continue;
            const int key0 = 8 * (warp + kCW * t) + 2 * qd;
            const float p00 = exp2f(z[t][0] - mu0), p01 = exp2f(z[t][1] - mu0);
            const float p10 = exp2f(z[t][2] - mu1), p11 = exp2f(z[t][3] - mu1);
            sum0 += p00 + p01;
            sum1 += p10 + p11;
            const float u00 = p00 * f[t][0], u01 = p01 * f[t][1], u10 = p10 * f[t][0], u11 = p11 * f[t][1];
            const __nv_bfloat162 h0 = __floats2bfloat162_rn(u00, u01), h1 = __floats2bfloat162_rn(u10, u11);
            const uint32_t off0 = g * kPStride + key0 * 2, off1 = (g + 8) * kPStride + key0 * 2;
            *reinterpret_cast<__nv_bfloat162*>(sm.P + off0) = h0;
            *reinterpret_cast<__nv_bfloat162*>(sm.P + off1) = h1;
            *reinterpret_cast<uint32_t*>(sm.Pl + off0) = pack_bf16(u00 - __low2float(h0), u01 - __high2float(h0));
            *reinterpret_cast<uint32_t*>(sm.Pl + off1) = pack_bf16(u10 - __low2float(h1), u11 - __high2float(h1));
        }
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
            sum0 += __shfl_xor_sync(0xFFFFFFFFu, sum0, o2);
            sum1 += __shfl_xor_sync(0xFFFFFFFFu, sum1, o2);
        }
        if (qd == 0) {   // red's maxima were consumed before the last barrier
            sm.red[warp][g] = sum0;
            sm.red[warp][g + 8] = sum1;
        }
    }
    __syncthreads();
    if (tid < kH) {
        float l = 0.0f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) l += sm.red[w][tid];
        sm.ml[tid][0] = sm.m_loc[tid];
        sm.ml[tid][1] = l;
    }

    // ---- O_r[:, 32 warp .. +31] = P V over the CTA's keys
    float o[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[n][j] = 0.0f;
    for (int kk = 0; kk < (n16 >> 4); ++kk) {
        uint32_t a0, a1, a2, a3, l0, l1, l2, l3;
        const uint32_t poff = (uint32_t)((lane & 15) * kPStride + (16 * kk + 8 * (lane >> 4)) * 2);
        ldsm_x4(sP + poff, a0, a1, a2, a3);
        ldsm_x4(sPl + poff, l0, l1, l2, l3);
        const int mi = lane >> 3;
        const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sK + swz(key, 4 * warp + 2 * np + (mi >> 1)), b0, b1, b2, b3);
            mma_bf16(o[2 * np], a0, a1, a2, a3, b0, b1);
            mma_bf16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
            mma_bf16(o[2 * np], l0, l1, l2, l3, b0, b1);
            mma_bf16(o[2 * np + 1], l0, l1, l2, l3, b2, b3);
        }
    }
    __syncthreads();   // every warp is done with K: its buffer now takes the partial O
    float* Of = reinterpret_cast<float*>(sm.K);
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int d = 32 * warp + 8 * n + 2 * qd;
        *reinterpret_cast<float2*>(Of + g * kOStride + d) = make_float2(o[n][0], o[n][1]);
        *reinterpret_cast<float2*>(Of + (g + 8) * kOStride + d) = make_float2(o[n][2], o[n][3]);
    }
    cl::sync();   // every CTA's partial O and (max, sum) are published

    // ---- combine: this CTA's slice of the output dims
    const int DS = kD / (int)C;
    if (tid < kH) {
        float mc[16], lc[16];
        float M = -INFINITY;
        for (uint32_t c = 0; c < C; ++c) {
            const uint2 x = cl::ld_v2(cl::map_rank((uint32_t)__cvta_generic_to_shared(&sm.ml[tid][0]), c));
            mc[c] = __uint_as_float(x.x);
            lc[c] = __uint_as_float(x.y);
            M = fmaxf(M, mc[c]);
        }
        const float Mu = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f;
        for (uint32_t c = 0; c < C; ++c) {
            const float wgt = exp2f(mc[c] - Mu);
            sm.cw[c][tid] = wgt;
            L += lc[c] * wgt;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (uint32_t c = 0; c < C; ++c) sm.cw[c][tid] *= inv;
        if (p.lse && rank == 0) p.lse[(int64_t)bq * kH + tid] = L > 0.0f ? (Mu + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
    {
        const int per_head = DS / 4;   // float4 per head in the slice
        const uint32_t sOf = (uint32_t)__cvta_generic_to_shared(Of);
        uint16_t* out = p.out + (int64_t)bq * kH * kD;
        for (int e4 = tid; e4 < kH * per_head; e4 += kCT) {
            const int h = e4 / per_head;
            const int d = (int)rank * DS + 4 * (e4 - h * per_head);
            const uint32_t la = sOf + (uint32_t)(h * kOStride + d) * 4u;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t c = 0; c < C; ++c) {
                const uint4 x = cl::ld_v4(cl::map_rank(la, c));
                const float wgt = sm.cw[c][h];
                acc.x += __uint_as_float(x.x) * wgt;
                acc.y += __uint_as_float(x.y) * wgt;
                acc.z += __uint_as_float(x.z) * wgt;
                acc.w += __uint_as_float(x.w) * wgt;
            }
            *reinterpret_cast<uint2*>(out + h * kD + d) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
        }
    }
    cl::sync();   // no CTA leaves while the cluster may read it
}

int g_max_active[17];
bool g_max_active_known[17];
bool g_attr_done = false, g_attr_ok = false, g_nonportable = false;

int smem_bytes() { return (int)sizeof(ClAttnSmem); }

bool set_attributes() {
    if (g_attr_done) return g_attr_ok;
    g_attr_done = true;
    if (cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes()) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    g_nonportable = cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                    cudaSuccess;
    if (!g_nonportable) (void)cudaGetLastError();
    g_attr_ok = true;
    return true;
}

cudaLaunchConfig_t make_config(int C, int bq, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, bq);
    cfg.blockDim = dim3(kCT);
    cfg.dynamicSmemBytes = smem_bytes();
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

int max_active_clusters(int C, int bq) {
    if (g_max_active_known[C]) return g_max_active[C];
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = make_config(C, bq, 0, attr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_cluster_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    g_max_active[C] = n;
    g_max_active_known[C] = true;
    return n;
}

}  // namespace

int attn_cluster_size(int B, int Q, int slots_total, int* keys_per_cta) {
    const int bq = B * Q;
    if (bq <= 0 || slots_total <= 0 || !set_attributes()) return 0;
    for (int C = g_nonportable ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > kNumSMs) continue;
        const int n = ((slots_total + C - 1) / C + 15) / 16 * 16;
        if (n > kMaxKeys) return 0;   // a smaller cluster only lengthens the chunk
        if (max_active_clusters(C, bq) >= bq) {
            if (keys_per_cta) *keys_per_cta = n;
            return C;
        }
    }
    return 0;
}

cudaError_t launch_attn_cluster(AttnParams& p, int C, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = make_config(C, p.B * p.Q, st, attr);
    return cudaLaunchKernelEx(&cfg, attn_cluster_kernel, p);
}

}  // namespace csa2
