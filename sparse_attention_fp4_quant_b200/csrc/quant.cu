// quant.cu -- NVFP4 quantisation of latent rows and the indexer-K projection.
//
// NVFP4 here: E2M1 codes, one E4M3 scale per 16 channels, no second-level
// scale.  scale = E4M3_rne_satfinite(fp32(amax / 6)); each code rounds
// |x| / scale to the nearest E2M1 magnitude, ties to the even code, by
// comparing |x| with the exact fp32 midpoints m * scale.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

__device__ __forceinline__ void quant16(const float v[16], uint32_t& scale_byte, uint32_t& lo, uint32_t& hi) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const uint32_t sc = f32_to_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_f32(sc);
    // midpoints between consecutive E2M1 magnitudes, times the scale (exact)
    const float t0 = 0.25f * s, t1 = 0.75f * s, t2 = 1.25f * s, t3 = 1.75f * s;
    const float t4 = 2.5f * s, t5 = 3.5f * s, t6 = 5.0f * s;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float a = fabsf(v[j]);
        // a tie at a midpoint goes to the even code: strict for 0.25/1.25/2.5/5, inclusive for 0.75/1.75/3.5
        uint32_t mag = (uint32_t)(a > t0) + (uint32_t)(a >= t1) + (uint32_t)(a > t2) + (uint32_t)(a >= t3) +
                       (uint32_t)(a > t4) + (uint32_t)(a >= t5) + (uint32_t)(a > t6);
        uint32_t code = mag | ((__float_as_uint(v[j]) >> 31) << 3);
        w[j >> 3] |= code << (4 * (j & 7));
    }
    if (s == 0.0f) w[0] = w[1] = 0u;
    scale_byte = sc;
    lo = w[0];
    hi = w[1];
}

__global__ void __launch_bounds__(256) quant_kernel(const uint16_t* __restrict__ x, int64_t rows, int ch,
                                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                    const int64_t* __restrict__ dst_rows, int64_t out_rows) {
    pdl_enter();
    const int G = ch / 16;
    int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= rows * G) return;
    int64_t r = t / G;
    int g = (int)(t - r * G);
    const uint4* src = reinterpret_cast<const uint4*>(x + r * ch + 16 * g);
    uint4 a = __ldg(src), b = __ldg(src + 1);
    uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        v[2 * j] = __uint_as_float(u[j] << 16);
        v[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
    uint32_t sc, lo, hi;
    quant16(v, sc, lo, hi);
    int64_t orow = dst_rows ? __ldg(dst_rows + r) : r;
    if (orow < 0 || orow >= out_rows) return;
    *reinterpret_cast<uint2*>(codes + orow * (ch / 2) + 8 * g) = make_uint2(lo, hi);
    scales[orow * G + g] = (uint8_t)sc;
}

cudaError_t launch_quant(const void* x, int64_t rows, int ch, uint8_t* codes, uint8_t* scales,
                         const int64_t* dst_rows, int64_t out_rows, cudaStream_t st) {
    int64_t n = rows * (ch / 16);
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    return launch_ex(quant_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 0, static_cast<const uint16_t*>(x), rows, ch,
                     codes, scales, dst_rows, out_rows);
}

// k = x W as fp32 fused multiply-add chains over the 512 channels in ascending
// order; a 64-row x 64-output tile per CTA, 4 x 4 outputs per thread.
constexpr int kPR = 64;   // rows per CTA
constexpr int kPC = 32;   // channels per smem chunk

__global__ void __launch_bounds__(256) index_k_proj_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                           const float* __restrict__ W, uint8_t* __restrict__ kc,
                                                           uint8_t* __restrict__ ks,
                                                           const int64_t* __restrict__ dst_rows, int64_t out_rows) {
    pdl_enter();
    __shared__ float xs[kPC][kPR + 4];
    __shared__ float wsm[kPC][kID + 4];
    __shared__ float outs[kPR][kID + 4];
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    const int64_t r0 = (int64_t)blockIdx.x * kPR;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

    for (int c0 = 0; c0 < kD; c0 += kPC) {
        // x chunk [64 rows][32 ch] -> transposed fp32
#pragma unroll
        for (int it = 0; it < (kPR * kPC) / 256; ++it) {
            int e = it * 256 + tid;
            int rr = e / kPC, cc = e % kPC;
            int64_t row = r0 + rr;
            float v = 0.0f;
            if (row < rows) v = __uint_as_float(((uint32_t)__ldg(x + row * kD + c0 + cc)) << 16);
            xs[cc][rr] = v;
        }
#pragma unroll
        for (int it = 0; it < (kPC * kID) / 256; ++it) {
            int e = it * 256 + tid;
            int cc = e / kID, jj = e % kID;
            wsm[cc][jj] = __ldg(W + (int64_t)(c0 + cc) * kID + jj);
        }
        __syncthreads();
#pragma unroll 8
        for (int cc = 0; cc < kPC; ++cc) {
            float a[4], bw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[cc][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bw[j] = wsm[cc][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], bw[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) outs[ty * 4 + i][tx * 4 + j] = acc[i][j];
    __syncthreads();
    // one thread per (row, group of 16 outputs)
    const int rr = tid >> 2, g = tid & 3;
    const int64_t row = r0 + rr;
    if (row < rows) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = outs[rr][16 * g + j];
        uint32_t sc, lo, hi;
        quant16(v, sc, lo, hi);
        int64_t orow = dst_rows ? __ldg(dst_rows + row) : row;
        if (orow >= 0 && orow < out_rows) {
            *reinterpret_cast<uint2*>(kc + ik_code_off(orow, g >> 1) + 8 * (g & 1)) = make_uint2(lo, hi);
            ks[ik_scale_off(orow) + g] = (uint8_t)sc;
        }
    }
}

// Few rows (a decode append): one thread per (row, output) runs its 512-long
// FMA chain, 4 rows per CTA.  All of W (128 KB) is copied into shared memory
// with cp.async up front, so the copy costs one memory latency and the chain
// then waits only on its own FMAs.  The 64 outputs of a row are quantised from
// shared memory by 4 threads.
constexpr int kProjRowsPerCTA = 4;
constexpr int kProjSmem = (kD * kID + kProjRowsPerCTA * kD) * 4;

__global__ void __launch_bounds__(256) index_k_proj_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                const float* __restrict__ W, uint8_t* __restrict__ kc,
                                                                uint8_t* __restrict__ ks,
                                                                const int64_t* __restrict__ dst_rows, int64_t out_rows) {
    pdl_enter();
    extern __shared__ __align__(16) float wsm[];   // W [512][64], then the rows [4][512]
    float* xs = wsm + kD * kID;
    __shared__ float outs[kProjRowsPerCTA][kID];
    const int tid = threadIdx.x;
    const int rr = tid >> 6, j = tid & 63;
    const int64_t r0 = (int64_t)blockIdx.x * kProjRowsPerCTA;
    const uint32_t wbase = (uint32_t)__cvta_generic_to_shared(wsm);
    for (int i = tid; i < kD * kID / 4; i += 256)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(wbase + 16u * i), "l"(W + 4 * i) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int e = tid; e < kProjRowsPerCTA * kD; e += 256) {
        const int64_t row = r0 + e / kD;
        xs[e] = row < rows ? __uint_as_float(((uint32_t)__ldg(x + row * kD + e % kD)) << 16) : 0.0f;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    const float* xr = xs + rr * kD;
    float acc = 0.0f;
#pragma unroll 16
    for (int c = 0; c < kD; ++c) acc = __fmaf_rn(xr[c], wsm[c * kID + j], acc);
    outs[rr][j] = acc;
    __syncthreads();
    if (tid < 4 * kProjRowsPerCTA) {
        const int r2 = tid >> 2, g = tid & 3;
        const int64_t row2 = r0 + r2;
        if (row2 < rows) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = outs[r2][16 * g + q];
            uint32_t sc, lo, hi;
            quant16(v, sc, lo, hi);
            const int64_t orow = dst_rows ? __ldg(dst_rows + row2) : row2;
            if (orow >= 0 && orow < out_rows) {
                *reinterpret_cast<uint2*>(kc + ik_code_off(orow, g >> 1) + 8 * (g & 1)) = make_uint2(lo, hi);
                ks[ik_scale_off(orow) + g] = (uint8_t)sc;
            }
        }
    }
}

// Append of a few new rows (a decode step): one launch quantises each latent
// row into the main KV and projects + quantises its indexer K.  A projection
// CTA takes 32 rows and one 16-output block of W (32 KB, staged with cp.async
// next to the 32 bf16 rows): thread (row, output) runs the 512-long FMA chain
// in ascending channel order, and since the 16 outputs of a row are exactly
// one NVFP4 block, the CTA quantises its block alone.  The remaining CTAs
// quantise the latent rows, one thread per 16 channels.
constexpr int kAppRows = 32;
constexpr int kAppThreads = kAppRows * 4;   // projection: one row x four outputs per thread
constexpr int kAppXStride = kD + 8;   // bf16 per staged row (16 bytes of padding: no bank conflicts)
constexpr int kAppSmem = kD * 16 * 4 + kAppRows * kAppXStride * 2 + kAppRows * 16 * 4;

__global__ void __launch_bounds__(kAppThreads) append_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                             const float* __restrict__ W, uint8_t* __restrict__ lc,
                                                             uint8_t* __restrict__ ls, uint8_t* __restrict__ kc,
                                                             uint8_t* __restrict__ ks,
                                                             const int64_t* __restrict__ dst_rows, int64_t out_rows,
                                                             int nproj) {
    pdl_enter();
    const int tid = threadIdx.x;
    if ((int)blockIdx.x >= nproj) {
        // latent rows -> NVFP4, one thread per 16 channels
        const int64_t t = (int64_t)(blockIdx.x - nproj) * kAppThreads + tid;
        if (t >= rows * (kD / 16)) return;
        const int64_t r = t / (kD / 16);
        const int g = (int)(t - r * (kD / 16));
        const uint4* src = reinterpret_cast<const uint4*>(x + r * kD + 16 * g);
        const uint4 a = __ldg(src), b = __ldg(src + 1);
        const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = __uint_as_float(u[j] << 16);
            v[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
        uint32_t sc, lo, hi;
        quant16(v, sc, lo, hi);
        const int64_t orow = dst_rows ? __ldg(dst_rows + r) : r;
        if (orow < 0 || orow >= out_rows) return;
        *reinterpret_cast<uint2*>(lc + orow * (kD / 2) + 8 * g) = make_uint2(lo, hi);
        ls[orow * (kD / 16) + g] = (uint8_t)sc;
        return;
    }
    extern __shared__ __align__(16) uint8_t app_smem[];
    float* Wb = reinterpret_cast<float*>(app_smem);                                 // [512][16]
    uint16_t* xs = reinterpret_cast<uint16_t*>(app_smem + kD * 16 * 4);             // [32][kAppXStride]
    float* outs = reinterpret_cast<float*>(app_smem + kD * 16 * 4 + kAppRows * kAppXStride * 2);   // [32][16]
    const int cb = blockIdx.x & 3;                  // output block: outputs 16 cb .. 16 cb + 15
    const int64_t r0 = (int64_t)(blockIdx.x >> 2) * kAppRows;
    const uint32_t sW = (uint32_t)__cvta_generic_to_shared(Wb), sX = (uint32_t)__cvta_generic_to_shared(xs);
    for (int i = tid; i < kD * 4; i += kAppThreads) {   // row c of the block: 4 x 16 B
        const int c = i >> 2, q = i & 3;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sW + 16u * i), "l"(W + c * kID + 16 * cb + 4 * q)
                     : "memory");
    }
    for (int i = tid; i < kAppRows * (kD / 8); i += kAppThreads) {   // 32 rows x 64 x 16 B
        const int rr = i / (kD / 8), q = i % (kD / 8);
        if (r0 + rr < rows)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sX + (uint32_t)(rr * kAppXStride * 2 + 16 * q)),
                         "l"(x + (r0 + rr) * kD + 8 * q)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
    __syncthreads();
    // four chains per thread (outputs 4 og .. 4 og + 3 of row rr), each in channel order: one
    // load of x and one 16-byte load of W feed four fused multiply-adds
    const int rr = tid >> 2, og = tid & 3;
    const uint16_t* xr = xs + rr * kAppXStride;
    float acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
#pragma unroll 8
    for (int c = 0; c < kD; ++c) {
        const float xv = __uint_as_float((uint32_t)xr[c] << 16);
        const float4 w = *reinterpret_cast<const float4*>(Wb + c * 16 + 4 * og);
        acc0 = __fmaf_rn(xv, w.x, acc0);
        acc1 = __fmaf_rn(xv, w.y, acc1);
        acc2 = __fmaf_rn(xv, w.z, acc2);
        acc3 = __fmaf_rn(xv, w.w, acc3);
    }
    *reinterpret_cast<float4*>(outs + rr * 16 + 4 * og) = make_float4(acc0, acc1, acc2, acc3);
    __syncthreads();
    if (tid < kAppRows && r0 + tid < rows) {
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = outs[tid * 16 + q];
        uint32_t sc, lo, hi;
        quant16(v, sc, lo, hi);
        const int64_t orow = dst_rows ? __ldg(dst_rows + r0 + tid) : r0 + tid;
        if (orow >= 0 && orow < out_rows) {
            *reinterpret_cast<uint2*>(kc + ik_code_off(orow, cb >> 1) + 8 * (cb & 1)) = make_uint2(lo, hi);
            ks[ik_scale_off(orow) + cb] = (uint8_t)sc;
        }
    }
}

cudaError_t launch_append(const void* x, int64_t rows, const float* W, uint8_t* lat_codes, uint8_t* lat_scales,
                          uint8_t* k_codes, uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows,
                          cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (rows > 2048) {
        cudaError_t e = launch_quant(x, rows, kD, lat_codes, lat_scales, dst_rows, out_rows, st);
        if (e != cudaSuccess) return e;
        return launch_index_k_proj(x, rows, W, k_codes, k_scales, dst_rows, out_rows, st);
    }
    static DeviceOnce attr;
    cudaError_t e = attr.run(
        [] { return cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAppSmem); });
    if (e != cudaSuccess) return e;
    const int nproj = (int)((rows + kAppRows - 1) / kAppRows) * 4;
    const int nquant = (int)((rows * (kD / 16) + kAppThreads - 1) / kAppThreads);
    return launch_ex(append_kernel, dim3(nproj + nquant), dim3(kAppThreads), kAppSmem, st, 0,
                     static_cast<const uint16_t*>(x), rows, W, lat_codes, lat_scales, k_codes, k_scales, dst_rows,
                     out_rows, nproj);
}

cudaError_t launch_index_k_proj(const void* x, int64_t rows, const float* W, uint8_t* k_codes, uint8_t* k_scales,
                                const int64_t* dst_rows, int64_t out_rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (rows <= 2048) {
        static DeviceOnce attr;
        cudaError_t e = attr.run([] {
            return cudaFuncSetAttribute(index_k_proj_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kProjSmem);
        });
        if (e != cudaSuccess) return e;
        return launch_ex(index_k_proj_rows_kernel, dim3((unsigned)((rows + kProjRowsPerCTA - 1) / kProjRowsPerCTA)),
                         dim3(256), kProjSmem, st, 0, static_cast<const uint16_t*>(x), rows, W, k_codes, k_scales,
                         dst_rows, out_rows);
    }
    int64_t blocks = (rows + kPR - 1) / kPR;
    return launch_ex(index_k_proj_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 0, static_cast<const uint16_t*>(x),
                     rows, W, k_codes, k_scales, dst_rows, out_rows);
}

}  // namespace csa2

namespace csa2 {

// ---- fused front end --------------------------------------------------------
// RMSNorm + RoPE of new pre-norm latent rows, bf16 rounding, NVFP4 quantisation
// of the result and its indexer-K projection + quantisation, in one launch
// ([Jdon] "缓存压缩真的是越大越好吗": the latent is RMSNorm'd and RoPE keeps its
// norm; [Blog] "FP4 与 SWA Bounded Replay": quantised after RoPE; [Blog] "CSA2"
// section: the indexer K is projected from the main KV).  fp32 order, each step
// one IEEE rounding: ss = fused multiply-add chain of x_c^2 over c ascending;
// r = 1 / sqrt(ss / 512 + eps); n_c = (x_c r) w_c; pairs (448 + 2k, 449 + 2k):
// a' = a cos - b sin, b' = a sin + b cos with rounded products; y = bf16(n).
// Then the bytes of csa2_quant_nvfp4(y) and csa2_index_k_proj(y).
//
// A CTA takes 64 rows (256 threads): the bf16 rows are staged in shared memory
// (row stride 1040 B), 64 threads run the rows' sum-of-squares chains, every
// thread normalises and rotates 16-byte chunks in place, quantises 16-channel
// groups, and the projection runs as 4 x 4 register tiles of chains over 32-
// channel chunks of W, as index_k_proj_kernel does.
constexpr int kFR = 64;                 // rows per CTA
constexpr int kFXS = kD + 8;            // bf16 per staged row (16 B pad)
constexpr int kFrontSmem = kFR * kFXS * 2 + kPC * (kID + 4) * 4 + kFR * (kID + 4) * 4 + kFR * 4;

__global__ void __launch_bounds__(256) front_end_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                        const float* __restrict__ rcos, const float* __restrict__ rsin,
                                                        const float* __restrict__ nw, float eps,
                                                        const float* __restrict__ W, uint8_t* __restrict__ lc,
                                                        uint8_t* __restrict__ ls, uint8_t* __restrict__ kc,
                                                        uint8_t* __restrict__ ks, const int64_t* __restrict__ dst_rows,
                                                        int64_t out_rows, uint16_t* __restrict__ y_out) {
    pdl_enter();
    extern __shared__ __align__(16) uint8_t fe_smem[];
    uint16_t* xs = reinterpret_cast<uint16_t*>(fe_smem);                                  // [64][kFXS] bf16
    float* wsm = reinterpret_cast<float*>(fe_smem + kFR * kFXS * 2);                      // [32][68]
    float* outs = wsm + kPC * (kID + 4);                                                  // [64][68]
    float* inv = outs + kFR * (kID + 4);                                                  // [64]
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)blockIdx.x * kFR;
    const int nr = (int)min((int64_t)kFR, rows - r0);

    // stage the rows (16 B per thread and step; rows past the end are zero)
    for (int i = tid; i < kFR * (kD / 8); i += 256) {
        const int rr = i / (kD / 8), q = i % (kD / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (rr < nr) v = __ldg(reinterpret_cast<const uint4*>(x + (r0 + rr) * kD) + q);
        *reinterpret_cast<uint4*>(xs + rr * kFXS + 8 * q) = v;
    }
    __syncthreads();
    // sum of squares: one chain per row, channels ascending
    if (tid < kFR) {
        const uint16_t* xr = xs + tid * kFXS;
        float ss = 0.0f;
#pragma unroll 8
        for (int c = 0; c < kD; ++c) {
            const float v = __uint_as_float((uint32_t)xr[c] << 16);
            ss = __fmaf_rn(v, v, ss);
        }
        const float t = __fadd_rn(__fdiv_rn(ss, 512.0f), eps);
        inv[tid] = __fdiv_rn(1.0f, __fsqrt_rn(t));
    }
    __syncthreads();
    // normalise, rotate, round to bf16 in place: 16-byte chunk q (channels 8q .. 8q + 7) of row rr
    for (int i = tid; i < kFR * (kD / 8); i += 256) {
        const int rr = i / (kD / 8), q = i % (kD / 8);
        uint4* p = reinterpret_cast<uint4*>(xs + rr * kFXS + 8 * q);
        const uint4 v = *p;
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        const float r = inv[rr];
        float n[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            n[2 * j] = __fmul_rn(__uint_as_float(u[j] << 16), r);
            n[2 * j + 1] = __fmul_rn(__uint_as_float(u[j] & 0xFFFF0000u), r);
        }
        if (nw) {
#pragma unroll
            for (int j = 0; j < 8; ++j) n[j] = __fmul_rn(n[j], __ldg(nw + 8 * q + j));
        }
        if (q >= 56 && rr < nr) {   // channels 448 .. 511: pairs k = 4 (q - 56) .. + 3
            const float* cs = rcos + (r0 + rr) * 32 + 4 * (q - 56);
            const float* sn = rsin + (r0 + rr) * 32 + 4 * (q - 56);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a = n[2 * j], b = n[2 * j + 1], c = __ldg(cs + j), s = __ldg(sn + j);
                n[2 * j] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
                n[2 * j + 1] = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(n[2 * j]));
            const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(n[2 * j + 1]));
            o[j] = lo | (hi << 16);
        }
        const uint4 ov = make_uint4(o[0], o[1], o[2], o[3]);
        *p = ov;
        if (y_out && rr < nr) *reinterpret_cast<uint4*>(y_out + (r0 + rr) * kD + 8 * q) = ov;
    }
    __syncthreads();
    // main latent -> NVFP4: one thread per (row, 16-channel group)
    for (int i = tid; i < kFR * (kD / 16); i += 256) {
        const int rr = i / (kD / 16), g = i % (kD / 16);
        if (rr >= nr) continue;
        const uint4* src = reinterpret_cast<const uint4*>(xs + rr * kFXS + 16 * g);
        const uint4 a = src[0], b = src[1];
        const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = __uint_as_float(u[j] << 16);
            v[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
        uint32_t sc, lo, hi;
        quant16(v, sc, lo, hi);
        const int64_t orow = dst_rows ? __ldg(dst_rows + r0 + rr) : r0 + rr;
        if (orow < 0 || orow >= out_rows) continue;
        *reinterpret_cast<uint2*>(lc + orow * (kD / 2) + 8 * g) = make_uint2(lo, hi);
        ls[orow * (kD / 16) + g] = (uint8_t)sc;
    }
    // indexer-K projection of the bf16 rows: 4 x 4 chains per thread, channels ascending
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    for (int c0 = 0; c0 < kD; c0 += kPC) {
        __syncthreads();   // the previous chunk of W is consumed (and, first time, the bf16 rows are final)
#pragma unroll
        for (int it = 0; it < (kPC * kID) / 256; ++it) {
            const int e = it * 256 + tid;
            const int cc = e / kID, jj = e % kID;
            wsm[cc * (kID + 4) + jj] = __ldg(W + (int64_t)(c0 + cc) * kID + jj);
        }
        __syncthreads();
#pragma unroll 8
        for (int cc = 0; cc < kPC; ++cc) {
            float a[4], bw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = __uint_as_float((uint32_t)xs[(ty * 4 + i) * kFXS + c0 + cc] << 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) bw[j] = wsm[cc * (kID + 4) + tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], bw[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) outs[(ty * 4 + i) * (kID + 4) + tx * 4 + j] = acc[i][j];
    __syncthreads();
    {
        const int rr = tid >> 2, g = tid & 3;
        if (rr < nr) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = outs[rr * (kID + 4) + 16 * g + j];
            uint32_t sc, lo, hi;
            quant16(v, sc, lo, hi);
            const int64_t orow = dst_rows ? __ldg(dst_rows + r0 + rr) : r0 + rr;
            if (orow >= 0 && orow < out_rows) {
                *reinterpret_cast<uint2*>(kc + ik_code_off(orow, g >> 1) + 8 * (g & 1)) = make_uint2(lo, hi);
                ks[ik_scale_off(orow) + g] = (uint8_t)sc;
            }
        }
    }
}

cudaError_t launch_front_end(const void* x, int64_t rows, const float* rcos, const float* rsin, const float* nw,
                             float eps, const float* W, uint8_t* lat_codes, uint8_t* lat_scales, uint8_t* k_codes,
                             uint8_t* k_scales, const int64_t* dst_rows, int64_t out_rows, void* y_out,
                             cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    static DeviceOnce attr;
    cudaError_t e = attr.run(
        [] { return cudaFuncSetAttribute(front_end_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFrontSmem); });
    if (e != cudaSuccess) return e;
    const int64_t blocks = (rows + kFR - 1) / kFR;
    return launch_ex(front_end_kernel, dim3((unsigned)blocks), dim3(256), kFrontSmem, st, 0,
                     static_cast<const uint16_t*>(x), rows, rcos, rsin, nw, eps, W, lat_codes, lat_scales, k_codes,
                     k_scales, dst_rows, out_rows, static_cast<uint16_t*>(y_out));
}

}  // namespace csa2
