// attn_cluster.cu -- csa2_sparse_attn for decode-sized query counts: one
// thread-block cluster of C CTAs per query.
//
// CTA r of the cluster takes the key slots [r * n, (r + 1) * n) of its query
// (n <= 160, a multiple of 16; slots as in attn_common.cuh) and gathers them
// all at once, so a CTA waits on global memory once instead of once per tile.
// The rows are dequantised to f16 in swizzled shared memory (K = V); with the
// 16 heads as the M dimension, S = Q K^T runs on warp-level tensor-core MMAs
// (each warp a quarter of the channels of a fifth of the keys), then the CTA's
// own softmax (one warp per head: max and sum over its keys), then O_r = P V
// (32 dims per warp; P as a rounded f16 term plus its f16 remainder).  The partial results meet in distributed shared memory:
// each CTA stores, into CTA c's (by then idle) key buffer, its slice
// [c * 512 / C, (c + 1) * 512 / C) of O_r (fp32) and its per-head (max, sum);
// CTA c then forms its slice of the output as
//   sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r,   M = max_r m_r,
// from its own shared memory and writes it as bf16.  No partials go to global
// memory and no CTA waits for a ticket.
#include "attn_common.cuh"
#include "cluster.cuh"

namespace csa2 {
namespace {

constexpr int kCT = 512;                      // threads per CTA (16 warps)
constexpr int kMaxKeys = 160;                 // key slots per CTA
constexpr int kPStride = kMaxKeys * 2 + 16;   // bytes per head row of P (conflict-free ldmatrix)
constexpr int kQG = 4;                        // key-tile groups of the S warps (x 4 channel groups)
constexpr int kQT = kMaxKeys / 8 / kQG;       // key tiles per S warp
constexpr int kSStride = kMaxKeys + 4;        // floats per head row of a partial S
static_assert(kMaxKeys % 32 == 0 && kMaxKeys % (8 * kQG) == 0, "keys per CTA");
static_assert(kCT / 32 == kH, "one warp per head in the softmax");
static_assert(2 * kH * kSStride * 4 <= kH * kRowB + 2 * kH * kPStride, "partial S fit the Q and P buffers");
static_assert((16 * kH * (kD / 16 + 4) + 16 * kH * 2) * 4 <= kMaxKeys * kRowB, "received slices fit the key buffer");

struct ClAttnSmem {
    uint8_t K[kMaxKeys * kRowB];   // f16 keys (= values), swizzled; afterwards the received output slices
    uint8_t Qs[kH * kRowB];        // f16 query (prescaled), swizzled; then (with P) the two partial S arrays
    uint8_t P[kH * kPStride];      // f16 P (rounded), [head][key]
    uint8_t Pl[kH * kPStride];     // f16 remainder P - rounded(P)
    float kf[kMaxKeys];            // per-key factor (1 for FP4 rows, token scale for SWA)
    int kvalid[kMaxKeys];
    alignas(16) float ml[kH][2];   // this CTA's (max, sum) per head (log2 units), read by the cluster
    float cw[16][kH];              // combine weight of rank c for head h (for this CTA's output slice)
    float qmax[kCT / 32];          // per-warp max |q|
};

__global__ void __launch_bounds__(kCT, 1) attn_cluster_kernel(AttnParams p) {
    pdl_enter();
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
    float scale_log2 = p.sm_scale * 1.4426950408889634f;

    // this CTA's slots [s0, s0 + nk), padded to n16 (dead slots past nk)
    const int s0 = min(p.slots_total, (int)rank * p.keys_per_cta);
    const int nk = min(p.slots_total, s0 + p.keys_per_cta) - s0;
    const int n16 = (nk + 15) & ~15;

    const uint32_t sK = (uint32_t)__cvta_generic_to_shared(sm.K);
    const uint32_t sQ = (uint32_t)__cvta_generic_to_shared(sm.Qs);
    const uint32_t sP = (uint32_t)__cvta_generic_to_shared(sm.P);
    const uint32_t sPl = (uint32_t)__cvta_generic_to_shared(sm.Pl);

    // ---- gather: row quarter u = r + n16 * qq (consecutive lanes, consecutive rows).
    // Every load of the thread is in flight before any is used: the main-row
    // ids first, then the rows, then the query.
    {
        constexpr int kPer = (kMaxKeys * 4 + kCT - 1) / kCT;   // 2
        RowQuarter rq[kPer];
        int rr[kPer], qs[kPer], slot[kPer];
        int32_t e[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int u = tid + kCT * j;
            rr[j] = -1;
            e[j] = -1;
            slot[j] = p.slots_total;
            if (u < 4 * n16) {
                rr[j] = u % n16;
                qs[j] = u / n16;
                if (rr[j] < nk) slot[j] = s0 + rr[j];   // past nk: dead
                if (slot[j] < p.k) e[j] = (int32_t)ld_nc_u32(p.idx + (int64_t)bq * p.k + slot[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            rq[j].kind = 0;
            if (rr[j] >= 0) {
                int64_t row = 0;
                const int kind = slot_row(p, b, slot[j], e[j], i_pos, lo, pos0, nmain, row);
                issue_quarter(p, kind, row, qs[j], rq[j]);
            }
        }
        const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + (int64_t)bq * kH * kD);
        uint4 qv[(kH * kD / 8) / kCT];
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) qv[it] = ld_nc_v4(qsrc + 16 * (it * kCT + tid));
        float qm = 0.0f;   // max |q| of the query, for its power-of-two prescale into f16
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) qm = fmaxf(qm, bf16x8_maxabs(qv[it]));
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xFFFFFFFFu, qm, o2));
        if (lane == 0) sm.qmax[warp] = qm;
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (rr[j] >= 0) store_quarter(sm.K, sm.kf, sm.kvalid, rr[j], qs[j], rq[j]);
        __syncthreads();
        qm = sm.qmax[0];
#pragma unroll
        for (int w = 1; w < kCT / 32; ++w) qm = fmaxf(qm, sm.qmax[w]);
        const int qe = q_prescale_exp(qm);
        const float qmul = __uint_as_float((uint32_t)(127 - qe) << 23);   // 2^-qe
        scale_log2 *= __uint_as_float((uint32_t)(127 + qe) << 23);       // the logits take 2^qe back
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) {
            const int c = it * kCT + tid;   // 16-byte chunk id
            *reinterpret_cast<uint4*>(sm.Qs + swz(c >> 6, c & 63)) = bf16x8_to_f16(qv[it], qmul);
        }
    }
    __syncthreads();

    // ---- S = Q K^T.  Warp (kg, ng) = (warp % 4, warp / 4) takes channels
    // [128 kg, 128 kg + 128) (its Q fragments stay in registers) of key tiles
    // ng, ng + 4, ..., ng + 16 (8 keys each); the four channel partials are
    // added in the fixed order (p0 + p2) + (p1 + p3) in shared memory.
    const int nt = n16 >> 3;
    const int kg = warp & 3, ng = warp >> 2;
    float s4[kQT][4];
    {
        uint32_t qa[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            ldsm_x4(sQ + swz(lane & 15, 2 * (8 * kg + j) + (lane >> 4)), qa[j][0], qa[j][1], qa[j][2], qa[j][3]);
#pragma unroll
        for (int i = 0; i < kQT; ++i) {
            s4[i][0] = s4[i][1] = s4[i][2] = s4[i][3] = 0.0f;
            const int tile = ng + kQG * i;
            if (tile < nt) {   // warp-uniform
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t b0, b1;
                    ldsm_x2(sK + swz(8 * tile + (lane & 7), 2 * (8 * kg + j) + ((lane >> 3) & 1)), b0, b1);
                    mma_f16(s4[i], qa[j][0], qa[j][1], qa[j][2], qa[j][3], b0, b1);
                }
            }
        }
    }
    __syncthreads();   // every warp holds its Q fragments: the Q and P buffers take the partial sums
    float* S0 = reinterpret_cast<float*>(sm.Qs);   // [16][kSStride], then S1 right after
    float* S1 = S0 + kH * kSStride;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        if ((kg >> 1) == pass) {
            float* S = (kg & 1) ? S1 : S0;
#pragma unroll
            for (int i = 0; i < kQT; ++i) {
                const int tile = ng + kQG * i;
                if (tile >= nt) continue;
                const int key0 = 8 * tile + 2 * qd;
                float2* r0 = reinterpret_cast<float2*>(S + g * kSStride + key0);
                float2* r1 = reinterpret_cast<float2*>(S + (g + 8) * kSStride + key0);
                if (pass == 0) {
                    *r0 = make_float2(s4[i][0], s4[i][1]);
                    *r1 = make_float2(s4[i][2], s4[i][3]);
                } else {
                    const float2 x0 = *r0, x1 = *r1;
                    *r0 = make_float2(x0.x + s4[i][0], x0.y + s4[i][1]);
                    *r1 = make_float2(x1.x + s4[i][2], x1.y + s4[i][3]);
                }
            }
        }
        __syncthreads();
    }
    // ---- softmax over the CTA's keys: warp h owns head h (keys lane + 32 j)
    {
        const int h = warp;
        float z[kMaxKeys / 32], fk[kMaxKeys / 32];
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < kMaxKeys / 32; ++j) {
            const int t = lane + 32 * j;
            const bool v = t < n16 && sm.kvalid[t] != 0;
            fk[j] = t < n16 ? sm.kf[t] : 0.0f;
            z[j] = v ? (S0[h * kSStride + t] + S1[h * kSStride + t]) * fk[j] * scale_log2 : -INFINITY;
            m = fmaxf(m, z[j]);
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o2));
        const float mu = (m == -INFINITY) ? 0.0f : m;
        float l = 0.0f;
#pragma unroll
        for (int j = 0; j < kMaxKeys / 32; ++j) {
            z[j] = exp2f(z[j] - mu);
            l += z[j];
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o2);
        __syncthreads();   // every partial sum is read: P may overwrite them
#pragma unroll
        for (int j = 0; j < kMaxKeys / 32; ++j) {
            const int t = lane + 32 * j;
            if (t < n16) {
                const float u = z[j] * fk[j];
                const __half hi = __float2half_rn(u);
                *reinterpret_cast<__half*>(sm.P + h * kPStride + 2 * t) = hi;
                *reinterpret_cast<__half*>(sm.Pl + h * kPStride + 2 * t) = __float2half_rn(u - __half2float(hi));
            }
        }
        if (lane == 0) {
            sm.ml[h][0] = m;
            sm.ml[h][1] = l;
        }
    }
    __syncthreads();

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
            mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
            mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
            mma_f16(o[2 * np], l0, l1, l2, l3, b0, b1);
            mma_f16(o[2 * np + 1], l0, l1, l2, l3, b2, b3);
        }
    }

    // ---- combine: every CTA pushes the slice of O_r and its (max, sum) that CTA c
    // owns (dims [c DS, (c + 1) DS)) into c's key buffer, which is free once every
    // CTA has finished P V
    const int DS = kD / (int)C;
    const int rstride = DS + 4;   // floats per head row of a received slice
    float* Rf = reinterpret_cast<float*>(sm.K);                 // [C][16][rstride]
    float* MLf = Rf + (int)C * kH * rstride;                    // [C][16][2]
    cl::sync();   // #1: every CTA is done with its key buffer
    {
        const uint32_t sR = (uint32_t)__cvta_generic_to_shared(Rf);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int d = 32 * warp + 8 * n + 2 * qd;
            const uint32_t owner = (uint32_t)(d / DS);
            const int dd = d - (int)owner * DS;
            const uint32_t a0 = sR + (uint32_t)(((int)rank * kH + g) * rstride + dd) * 4u;
            const uint32_t a1 = sR + (uint32_t)(((int)rank * kH + g + 8) * rstride + dd) * 4u;
            cl::st_v2f(cl::map_rank(a0, owner), o[n][0], o[n][1]);
            cl::st_v2f(cl::map_rank(a1, owner), o[n][2], o[n][3]);
        }
        if (tid < kH * (int)C) {
            const uint32_t owner = (uint32_t)(tid / kH);
            const int h = tid % kH;
            const uint32_t a = (uint32_t)__cvta_generic_to_shared(MLf + ((int)rank * kH + h) * 2);
            cl::st_v2f(cl::map_rank(a, owner), sm.ml[h][0], sm.ml[h][1]);
        }
    }
    cl::sync();   // #2: every slice has arrived; nothing reads another CTA's memory after this
    if (tid < kH) {
        float M = -INFINITY;
        for (uint32_t c = 0; c < C; ++c) M = fmaxf(M, MLf[((int)c * kH + tid) * 2]);
        const float Mu = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f;
        for (uint32_t c = 0; c < C; ++c) {
            const float wgt = exp2f(MLf[((int)c * kH + tid) * 2] - Mu);
            sm.cw[c][tid] = wgt;
            L += MLf[((int)c * kH + tid) * 2 + 1] * wgt;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (uint32_t c = 0; c < C; ++c) sm.cw[c][tid] *= inv;
        if (p.lse && rank == 0) p.lse[(int64_t)bq * kH + tid] = L > 0.0f ? (Mu + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
    {
        const int per_head = DS / 4;   // float4 per head in the slice
        uint16_t* out = p.out + (int64_t)bq * kH * kD;
        for (int e4 = tid; e4 < kH * per_head; e4 += kCT) {
            const int h = e4 / per_head;
            const int dd = 4 * (e4 - h * per_head);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t c = 0; c < C; ++c) {
                const float4 x = *reinterpret_cast<const float4*>(Rf + ((int)c * kH + h) * rstride + dd);
                const float wgt = sm.cw[c][h];
                acc.x += x.x * wgt;
                acc.y += x.y * wgt;
                acc.z += x.z * wgt;
                acc.w += x.w * wgt;
            }
            *reinterpret_cast<uint2*>(out + h * kD + (int)rank * DS + dd) =
                make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
        }
    }
}

DeviceOnce g_attr;
bool g_nonportable[kMaxDevices];

int smem_bytes() { return (int)sizeof(ClAttnSmem); }

// Shared-memory size and (where allowed) 16-CTA clusters, once per device.
bool set_attributes() {
    return g_attr.run([] {
        cudaError_t e =
            cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return e;
        }
        const int d = current_device();
        g_nonportable[d] =
            cudaFuncSetAttribute(attn_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
        if (!g_nonportable[d]) (void)cudaGetLastError();
        return cudaSuccess;
    }) == cudaSuccess;
}

bool nonportable() {
    const int d = current_device();
    return d >= 0 && d < kMaxDevices && g_nonportable[d];
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

struct ClusterOcc {
    int n[17];
};
DeviceValue<ClusterOcc> g_occ;

// Clusters of C CTAs that can be resident at once on the current device (0 if refused).
int max_active_clusters(int C) {
    const ClusterOcc occ = g_occ.get(
        [] {
            ClusterOcc o{};
            for (int c = 1; c <= (nonportable() ? 16 : 8); c <<= 1) {
                cudaLaunchAttribute attr[1];
                const cudaLaunchConfig_t cfg = make_config(c, 1, 0, attr);
                if (cudaOccupancyMaxActiveClusters(&o.n[c], attn_cluster_kernel, &cfg) != cudaSuccess) {
                    (void)cudaGetLastError();
                    o.n[c] = 0;
                }
            }
            return o;
        },
        ClusterOcc{});
    return occ.n[C];
}

}  // namespace

int attn_cluster_size(int B, int Q, int slots_total, int* keys_per_cta) {
    const int bq = B * Q;
    if (bq <= 0 || slots_total <= 0 || !set_attributes()) return 0;
    const int sms = device_sm_count();
    for (int C = nonportable() ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > sms) continue;
        const int n = ((slots_total + C - 1) / C + 15) / 16 * 16;
        if (n > kMaxKeys) return 0;   // a smaller cluster only lengthens the chunk
        if (max_active_clusters(C) >= bq) {
            if (keys_per_cta) *keys_per_cta = n;
            return C;
        }
    }
    return 0;
}

cudaError_t launch_attn_cluster(AttnParams& p, int C, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    return launch_ex(attn_cluster_kernel, dim3(C, p.B * p.Q), dim3(kCT), smem_bytes(), st, C, p);
}

}  // namespace csa2
