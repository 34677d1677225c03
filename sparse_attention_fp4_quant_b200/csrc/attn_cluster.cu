// attn_cluster.cu -- csa2_sparse_attn for decode-sized query counts: one
// thread-block cluster of C CTAs per query.
//
// CTA r of the cluster takes the main slots [r nm, (r + 1) nm) of its query's
// k selected entries and the window slots [r nw, (r + 1) nw) of its W window
// positions (nm = ceil(k / C), nw = ceil(W / C), nm + nw <= 160), so every CTA
// moves about the same bytes, and gathers them all at once: a CTA waits on
// global memory once instead of once per tile, and each warp reads whole rows.
// The rows are dequantised to f16 in swizzled shared memory (K = V); with the
// 16 heads as the M dimension, S = Q K^T runs on warp-level tensor-core MMAs
// (each warp a quarter of the channels of a fifth of the keys), then the CTA's
// own softmax (one warp per head: max and sum over its keys), then O_r = P V
// (32 dims per warp; P rounded to f16, fp32 accumulation).  The partial results
// meet in distributed shared memory: each CTA keeps its O_r (fp32) and per-head
// (max, sum) in its own shared memory, and after one cluster barrier CTA c
// loads the slice [c * 512 / C, (c + 1) * 512 / C) of every rank's O_r and
// forms its slice of the output as
//   sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r,   M = max_r m_r,
// written as bf16.  (Stores into the owners' memory drained at ~12 bytes per
// clock and needed a second full barrier.)  No partials go to global memory and
// no CTA waits for a ticket.
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
static_assert(2 * kH * kSStride * 4 <= kH * kRowB + kH * kPStride, "partial S fit the Q and P buffers");
static_assert(kH * (kD + 4) * 4 <= kMaxKeys * kRowB, "O_r fits the key buffer");

// 188 KB: the rest of the SM's 256 KB stays L1, which holds the gather's loads in flight
struct ClAttnSmem {
    uint8_t K[kMaxKeys * kRowB];   // f16 keys (= values), swizzled; afterwards this CTA's O_r
    uint8_t Qs[kH * kRowB];        // f16 query (prescaled), swizzled; then (with P) the two partial S arrays
    uint8_t P[kH * kPStride];      // f16 P, [head][key]
    float kf[kMaxKeys];            // per-key factor (1 for FP4 rows, token scale for SWA)
    int kvalid[kMaxKeys];
    alignas(16) float ml[kH][2];   // this CTA's (max, sum) per head (log2 units), read by the cluster
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

    // this CTA's rows: main slots [m0, m0 + nm) then window slots [w0, w0 + nw) (an interleaved
    // share, so every CTA of the cluster moves about the same bytes), padded to n16 dead rows
    const int m0 = min(p.k, (int)rank * p.main_per_cta);
    const int nm = min(p.k, m0 + p.main_per_cta) - m0;
    const int w0 = min(p.window, (int)rank * p.swa_per_cta);
    const int nw = min(p.window, w0 + p.swa_per_cta) - w0;
    const int nk = nm + nw;
    const int n16 = (nk + 15) & ~15;

    const uint32_t sK = (uint32_t)__cvta_generic_to_shared(sm.K);
    const uint32_t sQ = (uint32_t)__cvta_generic_to_shared(sm.Qs);
    const uint32_t sP = (uint32_t)__cvta_generic_to_shared(sm.P);

    // ---- gather.  Item u = 32 r + x: 16 dims (16 x .. 16 x + 15) of row r, so a warp
    // reads one row's 256 B of codes (or 512 B of a window row) in whole lines.  Every
    // load of the thread is in flight before any is used: the query and the row ids
    // first (one id per row, shared by the warp), then the rows.
    {
        const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + (int64_t)bq * kH * kD);
        uint4 qv[(kH * kD / 8) / kCT];
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) qv[it] = ld_nc_v4(qsrc + 16 * (it * kCT + tid));
        constexpr int kPer = kMaxKeys * 32 / kCT;   // 10 items per thread
        int32_t e[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = (tid >> 5) + (kCT / 32) * j;
            e[j] = r < nm ? (int32_t)ld_nc_u32(p.idx + (int64_t)bq * p.k + m0 + r) : -1;
        }
        uint4 raw[kPer];
        uint32_t sc[kPer];
        int kind[kPer];   // 0 dead or padding, 1 FP4 main row, 2 FP8 window row
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = (tid >> 5) + (kCT / 32) * j, x = lane;
            kind[j] = 0;
            raw[j] = make_uint4(0, 0, 0, 0);
            sc[j] = 0;
            if (r < nm) {
                if (e[j] >= 0 && e[j] < nmain) {
                    const int64_t row = (int64_t)b * p.cap + e[j];
                    const uint2 c2 = ld_nc_v2(p.lat + row * (kD / 2) + 8 * x);
                    raw[j].x = c2.x;
                    raw[j].y = c2.y;
                    sc[j] = (uint32_t)__ldg(p.lat_sc + row * (kD / 16) + x);
                    kind[j] = 1;
                }
            } else if (r < nk) {
                const int64_t tau = i_pos - p.window + 1 + (w0 + (r - nm));
                const int64_t rr = tau - pos0;
                if (tau >= lo && tau <= i_pos && rr >= 0 && rr < p.T) {
                    const int64_t row = (int64_t)b * p.T + rr;
                    raw[j] = ld_nc_v4(p.swa + row * kD + 16 * x);
                    if (x == 0) sc[j] = ld_nc_u32(p.swa_sc + row);
                    kind[j] = 2;
                }
            }
        }
        float qm = 0.0f;   // max |q| of the query, for its power-of-two prescale into f16
#pragma unroll
        for (int it = 0; it < (kH * kD / 8) / kCT; ++it) qm = fmaxf(qm, bf16x8_maxabs(qv[it]));
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xFFFFFFFFu, qm, o2));
        if (lane == 0) sm.qmax[warp] = qm;
        // rows -> f16 in the swizzled key buffer: chunks 2x and 2x + 1 of row r (exact: every
        // E2M1 x E4M3 product and every E4M3 value is an f16); dead and padding rows are zero
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int r = (tid >> 5) + (kCT / 32) * j, x = lane;
            if (r >= n16) continue;
            uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
            if (kind[j] == 1) {
                uint32_t s16;
                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s16) : "h"((uint16_t)sc[j]));
                const uint32_t s2 = __byte_perm(s16, 0u, 0x1010);
                lo4 = fp4x8_to_f16(raw[j].x, s2);
                hi4 = fp4x8_to_f16(raw[j].y, s2);
            } else if (kind[j] == 2) {
                const uint2 a = fp8x4_to_f16(raw[j].x), bb = fp8x4_to_f16(raw[j].y);
                const uint2 c = fp8x4_to_f16(raw[j].z), d = fp8x4_to_f16(raw[j].w);
                lo4 = make_uint4(a.x, a.y, bb.x, bb.y);
                hi4 = make_uint4(c.x, c.y, d.x, d.y);
            }
            *reinterpret_cast<uint4*>(sm.K + swz(r, 2 * x)) = lo4;
            *reinterpret_cast<uint4*>(sm.K + swz(r, 2 * x + 1)) = hi4;
            if (x == 0) {
                sm.kvalid[r] = kind[j] != 0;
                sm.kf[r] = kind[j] == 2 ? __uint_as_float(sc[j]) : 1.0f;
            }
        }
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
            if (t < n16) *reinterpret_cast<__half*>(sm.P + h * kPStride + 2 * t) = __float2half_rn(z[j] * fk[j]);
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
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sP + (uint32_t)((lane & 15) * kPStride + (16 * kk + 8 * (lane >> 4)) * 2), a0, a1, a2, a3);
        const int mi = lane >> 3;
        const int key = 16 * kk + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sK + swz(key, 4 * warp + 2 * np + (mi >> 1)), b0, b1, b2, b3);
            mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
            mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
    }

    // ---- combine: every CTA keeps its O_r (fp32 [16][512]) in its own key buffer (free once
    // its warps are done with P V) beside its (max, sum) per head; after one cluster barrier,
    // CTA c loads dims [c DS, (c + 1) DS) of every rank's O_r and the ranks' (max, sum) of the
    // same head, four ranks' loads in flight together, and forms its output slice
    //   sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r,   M = max_r m_r
    // (over the ranks in order, four at a time with a running maximum).  The loads are the last
    // use of another CTA's memory: an arrive after them and a wait at the very end keep every
    // CTA resident until all have read.
    constexpr int kOS = kD + 4;   // floats per head row of O_r (conflict-free float2 stores)
    float* Ow = reinterpret_cast<float*>(sm.K);
    __syncthreads();   // every warp is done reading the key buffer
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        const int d = 32 * warp + 8 * n + 2 * qd;
        *reinterpret_cast<float2*>(Ow + g * kOS + d) = make_float2(o[n][0], o[n][1]);
        *reinterpret_cast<float2*>(Ow + (g + 8) * kOS + d) = make_float2(o[n][2], o[n][3]);
    }
    cl::sync();   // every CTA's O_r and (max, sum) are in place
    {
        const int DS = kD / (int)C;       // output dims owned by each rank
        const int per_head = DS / 4;      // float4 of one head's slice
        const uint32_t sO = (uint32_t)__cvta_generic_to_shared(Ow);
        const uint32_t sML = (uint32_t)__cvta_generic_to_shared(&sm.ml[0][0]);
        uint16_t* out = p.out + (int64_t)bq * kH * kD;
        for (int e4 = tid; e4 < kH * per_head; e4 += kCT) {
            const int h = e4 / per_head;
            const int d = (int)rank * DS + 4 * (e4 - h * per_head);
            const uint32_t oa = sO + 4u * (uint32_t)(h * kOS + d), ma = sML + 8u * (uint32_t)h;
            float M = -INFINITY, L = 0.0f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t r0 = 0; r0 < C; r0 += 4) {
                uint4 x[4];
                uint2 ml[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (r0 + j < C) {
                        x[j] = cl::ld_v4(cl::map_rank(oa, r0 + j));
                        ml[j] = cl::ld_v2(cl::map_rank(ma, r0 + j));
                    }
                }
                float Mn = M;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (r0 + j < C) Mn = fmaxf(Mn, __uint_as_float(ml[j].x));
                const float Mu = (Mn == -INFINITY) ? 0.0f : Mn;
                const float sc = (M == -INFINITY) ? 0.0f : exp2f(M - Mu);   // rescale what came before
                L *= sc;
                acc.x *= sc;
                acc.y *= sc;
                acc.z *= sc;
                acc.w *= sc;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (r0 + j < C) {
                        const float w = exp2f(__uint_as_float(ml[j].x) - Mu);
                        L += __uint_as_float(ml[j].y) * w;
                        acc.x += __uint_as_float(x[j].x) * w;
                        acc.y += __uint_as_float(x[j].y) * w;
                        acc.z += __uint_as_float(x[j].z) * w;
                        acc.w += __uint_as_float(x[j].w) * w;
                    }
                }
                M = Mn;
            }
            const float inv = L > 0.0f ? 1.0f / L : 0.0f;
            *reinterpret_cast<uint2*>(out + h * kD + d) =
                make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
            if (p.lse && rank == 0 && d == 0)
                p.lse[(int64_t)bq * kH + h] = L > 0.0f ? (((M == -INFINITY) ? 0.0f : M) + log2f(L)) * 0.6931471805599453f
                                                       : -INFINITY;
        }
    }
    cl::arrive_relaxed();   // this CTA has read every rank's memory it needs
    cl::wait_acquire();     // ... and so has every other: no CTA leaves while it could be read
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

int attn_cluster_size(int B, int Q, int k, int window, int* main_per_cta, int* swa_per_cta) {
    const int bq = B * Q;
    if (bq <= 0 || k < 0 || window < 0 || k + window <= 0 || !set_attributes()) return 0;
    const int sms = device_sm_count();
    for (int C = nonportable() ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > sms) continue;
        const int nm = (k + C - 1) / C, nw = (window + C - 1) / C;
        if (nm + nw > kMaxKeys) return 0;   // a smaller cluster only lengthens the share
        if (max_active_clusters(C) >= bq) {
            if (main_per_cta) *main_per_cta = nm;
            if (swa_per_cta) *swa_per_cta = nw;
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
