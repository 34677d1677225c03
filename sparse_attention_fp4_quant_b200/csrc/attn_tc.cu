// attn_tc.cu -- csa2_sparse_attn for decode-sized query counts on the
// 5th-generation tensor cores: one thread-block cluster of C CTAs per query.
//
// Sparse attention ([Blog] "CSA2" section: softmax attention over the Top-K
// main entries plus the layer's own sliding-window KV, K = V = the dequantised
// latent; [Blog] "FP4 与 SWA Bounded Replay": dequantise before attention, and
// the replay mask [max(s, i - W + 1), i]).
//
// Work split.  CTA r of a query's cluster takes the main slots
// [r km, (r + 1) km) and the window slots [r kw, (r + 1) kw), km = ceil(k / C),
// kw = ceil(W / C), so every CTA moves the same bytes (at C = 4: 128 FP4 rows
// of 288 B and 32 FP8 rows of 516 B).  Its rows are key rows 0 .. nm - 1
// (main) and nm .. nk - 1 (window) of one f16 tile.
//
// Data path.
//   1. Every thread reads the ids of the main rows it copies, then copies them
//      (256 B of E2M1 codes and 32 B of E4M3 scales per row) into a staging
//      area with cp.async, laid out so that one warp instruction moves whole
//      128-byte lines; then it issues the loads that need nothing else (the
//      query, its share of the window rows), all in flight at once.  (Per-row
//      bulk copies issued by one warp took about 7 us longer, and 16-byte copies
//      spread over different rows about 2 us: the number of requests, not the
//      bytes, set the pace.)
//   2. Rows become f16 in the tensor cores' no-swizzle core-matrix layout
//      (8 rows x 16 B blocks): FP4 through the hardware E2M1 -> f16
//      conversion and an exact f16 multiply by the block scale (every
//      E2M1 x E4M3 product has at most 5 significant bits); window rows as
//      their E4M3 values (exact in f16), their fp32 token scale applied to the
//      logit and to the probability.  The bf16 query is brought into f16 range
//      by a power of two that the logits take back.
//   3. S^T = K Q^T on tcgen05 (kind::f16, fp32 accumulators in TMEM): keys as
//      M = 128, the 16 heads as N.  More than 128 rows take a second tile that
//      ends at the last row (its first rows repeat the first tile's); the two
//      tiles are issued by two threads in different warps, in parallel.
//   4. Softmax over the CTA's keys: TMEM lane = key, one thread per key; per
//      head max and sum by warp butterflies and a cross-warp step.  P goes to
//      shared memory as f16 plus its f16 remainder (K-major B operand).
//   5. O^T = V^T P^T on tcgen05: the same f16 tile read as an MN-major A
//      operand (dims as M, four tiles of 128; keys as K), N = 16 heads; one
//      issuing thread per dim tile (warps 0-3), so the four tiles go in parallel.
//   6. Combine in distributed shared memory: CTA c owns dims
//      [c 512 / C, (c + 1) 512 / C); every CTA pushes its slices of O^T and its
//      per-head (max, sum) into the owners' staging areas (free by then: a
//      split cluster barrier orders the pushes after every CTA's step 2),
//      one cluster barrier, then each owner forms
//        sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r,   M = max_r m_r,
//      and writes its slice of the output as bf16.
//
// Every mbarrier wait is bounded (2 s); a timeout sets the workspace's sticky
// flag and the CTA carries on without the data, reaching both cluster barriers
// like every other thread, waits (bounded) for its MMAs, and frees its TMEM.
#include "attn_common.cuh"
#include "cluster.cuh"
#include "tc.cuh"

namespace csa2 {
namespace {

constexpr int kTT = 256;                     // threads per CTA (8 warps)
constexpr int kMaxRows = 160;                // key rows per CTA
constexpr int kMaxMain = 128;                // main rows per CTA (the staging area)
constexpr int kRawStride = 304;              // staged row: 256 B codes, 32 B scales, 16 B pad (bank spread)
constexpr int kGrpBytes = 64 * 128;          // one 8-row group of a 512-wide f16 tile: 64 core matrices
constexpr int kPGrp = (kMaxRows / 8) * 128;  // one 8-head group of P^T (keys along K)
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColS0 = 0, kColS1 = 16, kColO = 32;
constexpr int kRecvOff = 0;                  // received O slices: float [C][512 / C][16]
constexpr int kRecvMlOff = 32768;            // received (max, sum): float [C][16][2]
constexpr int kCwOff = kRecvMlOff + 16 * kH * 8;   // combine weights: float [C][16]
static_assert(kCwOff + 16 * kH * 4 <= kMaxMain * kRawStride, "the combine buffers fit the staging area");

struct TcAttnSmem {
    uint8_t kv[kMaxRows / 8 * kGrpBytes];   // f16 keys (= values): [row group][chunk][8 rows x 16 B]
    uint8_t qs[2 * kGrpBytes];              // f16 query: [head group][chunk][8 heads x 16 B]
    uint8_t raw[kMaxMain * kRawStride];     // staged FP4 main rows; then the combine buffers
    uint8_t phi[2 * kPGrp];                 // f16 P^T: [head group][key chunk][8 heads x 16 B]
    uint8_t plo[2 * kPGrp];                 // f16 remainders P - rounded(P)
    float kf[kMaxRows];                     // per-key factor: 1 (main row) or the window row's token scale
    uint8_t kvalid[kMaxRows];
    float red[2][4][8];                     // softmax: [head half][warp of the half][head]
    float ml[kH][2];                        // this CTA's (max, sum) per head, log2 units
    float qmax[kTT / 32];
    uint64_t mma_s, mma_o;
    uint32_t tmem;
    int timed_out;
};

__device__ __forceinline__ uint32_t idesc_f16(int M, int N, bool a_mn) {
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16_tc(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

// Byte offset of 16-byte chunk c (dims 8c .. 8c + 7) of row j in a core-matrix tile.
__device__ __forceinline__ uint32_t tile_off(int j, int c) {
    return (uint32_t)((j >> 3) * kGrpBytes + c * 128 + (j & 7) * 16);
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }

// Reduce eight per-head values over the 32 lanes of a warp: afterwards lane l
// holds head (l >> 2) & 7 (max if IS_MAX, else sum).
template <bool IS_MAX>
__device__ __forceinline__ float warp_reduce8(float (&v)[8], int lane) {
    auto op = [](float a, float b) { return IS_MAX ? fmaxf(a, b) : a + b; };
    {
        const bool hi = (lane >> 4) & 1;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = hi ? v[i] : v[i + 4];
            const float keep = hi ? v[i + 4] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 16));
        }
    }
    {
        const bool hi = (lane >> 3) & 1;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = hi ? v[i] : v[i + 2];
            const float keep = hi ? v[i + 2] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 8));
        }
    }
    float r;
    {
        const bool hi = (lane >> 2) & 1;
        const float send = hi ? v[0] : v[1];
        const float keep = hi ? v[1] : v[0];
        r = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
    }
    r = op(r, __shfl_xor_sync(0xFFFFFFFFu, r, 2));
    r = op(r, __shfl_xor_sync(0xFFFFFFFFu, r, 1));
    return r;
}

__global__ void __launch_bounds__(kTT, 1) attn_tc_kernel(AttnParams p) {
    pdl_enter();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    TcAttnSmem& sm = *reinterpret_cast<TcAttnSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cl::rank(), C = cl::ctas();
    const int bq = blockIdx.y;
    const int b = bq / p.Q;
    const int64_t i_pos = p.q_pos[bq];
    int64_t lo = i_pos - p.window + 1;
    if (p.replay_start && lo < (int64_t)p.replay_start[b]) lo = p.replay_start[b];
    const int64_t pos0 = p.swa_pos0[b];
    int64_t nmain = p.n_entries[b];
    if (nmain > p.cap) nmain = p.cap;

    // this CTA's rows: main slots [m0, m0 + nm), window slots [w0, w0 + nw)
    const int m0 = min(p.k, (int)rank * p.main_per_cta);
    const int nm = min(p.k, m0 + p.main_per_cta) - m0;
    const int w0 = min(p.window, (int)rank * p.swa_per_cta);
    const int nw = min(p.window, w0 + p.swa_per_cta) - w0;
    const int nk = nm + nw;
    const int npad = (nk + 15) & ~15;

    // the critical chain starts first: the ids of the main rows this thread copies.  Codes:
    // chunk c (16 B) of row r is item 16 r + c, so a warp moves two rows' 256 B each (whole
    // 128-byte lines); thread tid takes items tid + 256 j, j < 8 (rows (tid >> 4) + 16 j).
    // Scales: 32 B per row in two 16-byte halves, thread tid takes row tid >> 1, half tid & 1.
    int32_t ce[kMaxMain / 16];
#pragma unroll
    for (int j = 0; j < kMaxMain / 16; ++j) {
        const int r = (tid >> 4) + 16 * j;
        ce[j] = r < nm ? (int32_t)ld_nc_u32(p.idx + (int64_t)bq * p.k + m0 + r) : -1;
    }
    const int my_row = tid >> 1, my_half = tid & 1;
    const int32_t my_e = my_row < nm ? (int32_t)ld_nc_u32(p.idx + (int64_t)bq * p.k + m0 + my_row) : -1;

    const int s_tiles = npad > 128 ? 2 : 1;   // S tiles: one issuing thread each
    if (tid == 0) {
        tc::mbar_init(&sm.mma_s, s_tiles);
        tc::mbar_init(&sm.mma_o, kD / 128);      // P V: one issuing thread per dim tile
        sm.timed_out = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(&sm.tmem, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = sm.tmem;

    // ---- 1. the main rows into the staging area with cp.async (codes at 0, scales at 256
    // of each 304-byte row); then the loads that need nothing else (the query, this CTA's
    // window rows, their token scales), all in flight while the rows land
    {
        const uint32_t rb = tc::smem_u32(sm.raw);
#pragma unroll
        for (int j = 0; j < kMaxMain / 16; ++j) {
            const int r = (tid >> 4) + 16 * j, c = tid & 15;
            if (r < nm && ce[j] >= 0 && ce[j] < nmain) {
                const uint8_t* src = p.lat + ((int64_t)b * p.cap + ce[j]) * (kD / 2) + 16 * c;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(rb + (uint32_t)(r * kRawStride + 16 * c)),
                             "l"(src)
                             : "memory");
            }
        }
        const bool live = my_row < nm && my_e >= 0 && my_e < nmain;
        if (my_row < nm && my_half == 0) {
            sm.kvalid[my_row] = live ? 1 : 0;
            sm.kf[my_row] = 1.0f;
        }
        if (live) {
            const uint8_t* src = p.lat_sc + ((int64_t)b * p.cap + my_e) * (kD / 16) + 16 * my_half;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(rb + (uint32_t)(my_row * kRawStride + 256 +
                                                                                         16 * my_half)),
                         "l"(src)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + (int64_t)bq * kH * kD);
    uint4 qv[4];
    int qoff[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int u = tid + kTT * it;   // u = [head group][chunk][head in group]
        const int h = (u >> 9) * 8 + (u & 7), c = (u >> 3) & 63;
        qv[it] = ld_nc_v4(qsrc + (h * kD + 8 * c) * 2);
        qoff[it] = (u >> 9) * kGrpBytes + c * 128 + (u & 7) * 16;
    }
    // window rows: 32 chunks of 16 B per row, chunk x of row t at u = 32 t + x
    constexpr int kWPer = (kMaxRows - kMaxMain) * 32 / kTT;   // 4 chunks per thread (<= 32 rows)
    uint4 wv[kWPer];
    int wrow[kWPer];
#pragma unroll
    for (int it = 0; it < kWPer; ++it) {
        const int u = tid + kTT * it;
        const int t = u >> 5, x = u & 31;
        wrow[it] = -1;
        wv[it] = make_uint4(0, 0, 0, 0);
        if (t < nw) {
            const int64_t tau = i_pos - p.window + 1 + (w0 + t);
            const int64_t rr = tau - pos0;
            if (tau >= lo && tau <= i_pos && rr >= 0 && rr < p.T) {
                wrow[it] = (int)rr;
                wv[it] = ld_nc_v4(p.swa + ((int64_t)b * p.T + rr) * kD + 16 * x);
            }
        }
    }
    bool wlive = false;   // thread t < nw: window row t's validity and token scale
    float wsc = 0.0f;
    if (tid < nw) {
        const int64_t tau = i_pos - p.window + 1 + (w0 + tid);
        const int64_t rr = tau - pos0;
        wlive = tau >= lo && tau <= i_pos && rr >= 0 && rr < p.T;
        if (wlive) wsc = __uint_as_float(ld_nc_u32(p.swa_sc + (int64_t)b * p.T + rr));
    }
    float qm = 0.0f;
#pragma unroll
    for (int it = 0; it < 4; ++it) qm = fmaxf(qm, bf16x8_maxabs(qv[it]));
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xFFFFFFFFu, qm, o2));
    if (lane == 0) sm.qmax[warp] = qm;
    // window rows -> f16 (row nm + t, chunks 2x and 2x + 1); dead slots become zero rows
#pragma unroll
    for (int it = 0; it < kWPer; ++it) {
        const int u = tid + kTT * it;
        const int t = u >> 5, x = u & 31;
        if (t < nw) {
            uint4 a = make_uint4(0, 0, 0, 0), c2 = make_uint4(0, 0, 0, 0);
            if (wrow[it] >= 0) {
                const uint2 p0 = fp8x4_to_f16(wv[it].x), p1 = fp8x4_to_f16(wv[it].y);
                const uint2 p2 = fp8x4_to_f16(wv[it].z), p3 = fp8x4_to_f16(wv[it].w);
                a = make_uint4(p0.x, p0.y, p1.x, p1.y);
                c2 = make_uint4(p2.x, p2.y, p3.x, p3.y);
            }
            *reinterpret_cast<uint4*>(sm.kv + tile_off(nm + t, 2 * x)) = a;
            *reinterpret_cast<uint4*>(sm.kv + tile_off(nm + t, 2 * x + 1)) = c2;
        }
    }
    if (tid < nw) {
        sm.kvalid[nm + tid] = wlive ? 1 : 0;
        sm.kf[nm + tid] = wsc;
    }
    // padding rows nk .. npad - 1 (fewer than 16): zero, so that P V reads finite values
    for (int u = tid; u < (npad - nk) * 64; u += kTT)
        *reinterpret_cast<uint4*>(sm.kv + tile_off(nk + (u >> 6), u & 63)) = make_uint4(0, 0, 0, 0);
    if (tid < npad - nk) {
        sm.kvalid[nk + tid] = 0;
        sm.kf[nk + tid] = 0.0f;
    }
    __syncthreads();   // the per-warp query maxima
    qm = sm.qmax[0];
#pragma unroll
    for (int w = 1; w < kTT / 32; ++w) qm = fmaxf(qm, sm.qmax[w]);
    const int qe = q_prescale_exp(qm);
    const float qmul = __uint_as_float((uint32_t)(127 - qe) << 23);   // 2^-qe
    const float scale_log2 = p.sm_scale * 1.4426950408889634f * __uint_as_float((uint32_t)(127 + qe) << 23);
#pragma unroll
    for (int it = 0; it < 4; ++it) *reinterpret_cast<uint4*>(sm.qs + qoff[it]) = bf16x8_to_f16(qv[it], qmul);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();   // every thread's row copies have landed

    // ---- 2. main rows -> f16: item u = [row group of 8][chunk][row in group]
    for (int u = tid; u < ((nm + 7) >> 3) * 512; u += kTT) {
        const int jl = u & 7, c = (u >> 3) & 63, r = 8 * (u >> 9) + jl;
        if (r >= nm) continue;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (sm.kvalid[r]) {
            const uint8_t* src = sm.raw + r * kRawStride;
            const uint32_t w = *reinterpret_cast<const uint32_t*>(src + 4 * c);
            const uint32_t sb = src[256 + (c >> 1)];
            uint32_t s16;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s16) : "h"((uint16_t)sb));
            val = fp4x8_to_f16(w, __byte_perm(s16, 0u, 0x1010));
        }
        *reinterpret_cast<uint4*>(sm.kv + tile_off(r, c)) = val;
    }
    tc::fence_proxy_async_smem();   // generic-proxy tile writes -> the tensor cores' reads
    __syncthreads();
    cluster_arrive();   // the staging area is free: peers may push into it after their wait

    // ---- 3. S^T = K Q^T (one thread issues)
    const int s1 = npad - 128;   // first row of the second tile (used when npad > 128)
    if (lane == 0 && warp >= 1 && warp <= s_tiles) {   // warp 1: tile 0, warp 2: tile 1 (in parallel)
        tc::tc_fence_after();
        const int tile = warp - 1;
        const uint32_t id = idesc_f16(128, 16, false);
        const uint32_t kv0 = tc::smem_u32(sm.kv), q0 = tc::smem_u32(sm.qs);
        const int row0 = tile == 0 ? 0 : s1;
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = tc::smem_desc(kv0 + (uint32_t)((row0 >> 3) * kGrpBytes + kk * 256), 128, kGrpBytes,
                                              tc::kLayoutNone);
            const uint64_t bd = tc::smem_desc(q0 + (uint32_t)(kk * 256), 128, kGrpBytes, tc::kLayoutNone);
            mma_f16_tc(tmem + (tile == 0 ? kColS0 : kColS1), ad, bd, id, kk > 0 ? 1u : 0u);
        }
        tc::tc_commit(&sm.mma_s);
    }

    // ---- 4. softmax: warps 0-3 heads 0-7, warps 4-7 heads 8-15; thread = key t (tile 0)
    // and, past row 127, key s1 + t (tile 1)
    {
        const int half = warp >> 2, qtr = warp & 3;
        const int t = 32 * qtr + lane;
        if (!tc::mbar_wait(&sm.mma_s, 0) && lane == 0) {
            sm.timed_out = 1;
            if (p.status) atomicExch(p.status, 1);
        }
        __syncwarp();
        tc::tc_fence_after();
        uint32_t r0[8], r1[8];
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * qtr) << 16);
        tmem_ld_x8(lane_addr + kColS0 + 8 * half, r0);
        const bool two = npad > 128;
        if (two) tmem_ld_x8(lane_addr + kColS1 + 8 * half, r1);
        tc::tmem_ld_wait();
        const int j0 = t, j1 = s1 + t;
        const bool v0 = j0 < nk && sm.kvalid[j0];
        const bool v1 = two && j1 >= 128 && j1 < nk && sm.kvalid[j1];
        const float f0 = v0 ? sm.kf[j0] : 0.0f;   // masked keys: p = 0 and a zero factor
        const float f1 = v1 ? sm.kf[j1] : 0.0f;
        float z0[8], z1[8], v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            z0[i] = v0 ? __uint_as_float(r0[i]) * f0 * scale_log2 : -INFINITY;
            z1[i] = v1 ? __uint_as_float(r1[i]) * f1 * scale_log2 : -INFINITY;
            v[i] = fmaxf(z0[i], z1[i]);
        }
        float mx = warp_reduce8<true>(v, lane);
        if ((lane & 3) == 0) sm.red[half][qtr][(lane >> 2) & 7] = mx;
        __syncthreads();
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[i] = fmaxf(fmaxf(sm.red[half][0][i], sm.red[half][1][i]), fmaxf(sm.red[half][2][i], sm.red[half][3][i]));
        __syncthreads();   // red is reused for the sums
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float mu = m[i] == -INFINITY ? 0.0f : m[i];
            z0[i] = exp2f(z0[i] - mu);
            z1[i] = exp2f(z1[i] - mu);
            v[i] = z0[i] + z1[i];
        }
        const float sum = warp_reduce8<false>(v, lane);
        if ((lane & 3) == 0) sm.red[half][qtr][(lane >> 2) & 7] = sum;
        // P (times the token scale) as f16 + f16 remainder, at [head][key] of the K-major B operand
#pragma unroll
        for (int rep = 0; rep < 2; ++rep) {
            const int j = rep == 0 ? j0 : j1;
            if (rep == 1 && !(two && j1 >= 128)) continue;
            if (j >= npad) continue;
            const float fk = rep == 0 ? f0 : f1;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float u = (rep == 0 ? z0[i] : z1[i]) * fk;
                const __half hi = __float2half_rn(u);
                const uint32_t off = (uint32_t)(half * kPGrp + (j >> 3) * 128 + i * 16 + (j & 7) * 2);
                *reinterpret_cast<__half*>(sm.phi + off) = hi;
                *reinterpret_cast<__half*>(sm.plo + off) = __float2half_rn(u - __half2float(hi));
            }
        }
        __syncthreads();
        if (qtr == 0 && (lane & 3) == 0) {   // lane 4 i of warps 0 and 4: head 8 half + i
            const int i = (lane >> 2) & 7;
            sm.ml[8 * half + i][0] = m[i];
            sm.ml[8 * half + i][1] =
                (sm.red[half][0][i] + sm.red[half][1][i]) + (sm.red[half][2][i] + sm.red[half][3][i]);
        }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();

    // ---- 5. O^T = V^T P^T: four dim tiles of 128 (M), keys as K in steps of 16
    if (lane == 0 && warp < kD / 128) {   // warp t issues dim tile t (the four run in parallel)
        tc::tc_fence_after();
        const uint32_t id = idesc_f16(128, 16, true);
        const uint32_t kv0 = tc::smem_u32(sm.kv), ph = tc::smem_u32(sm.phi), pl = tc::smem_u32(sm.plo);
        const int nsteps = npad >> 4;
        const int t = warp;
        {
            for (int s = 0; s < nsteps; ++s) {
                // A: rows (keys) 16 s .. 16 s + 15 = row groups 2 s, 2 s + 1 (LBO apart);
                // dims 128 t .. = chunks 16 t .. (SBO = 128 apart)
                const uint64_t ad = tc::smem_desc(kv0 + (uint32_t)(2 * s * kGrpBytes + 16 * t * 128), kGrpBytes, 128,
                                                  tc::kLayoutNone);
                const uint64_t bh = tc::smem_desc(ph + (uint32_t)(2 * s * 128), 128, kPGrp, tc::kLayoutNone);
                const uint64_t bl = tc::smem_desc(pl + (uint32_t)(2 * s * 128), 128, kPGrp, tc::kLayoutNone);
                mma_f16_tc(tmem + kColO + 16 * t, ad, bh, id, s > 0 ? 1u : 0u);
                mma_f16_tc(tmem + kColO + 16 * t, ad, bl, id, 1u);
            }
        }
        tc::tc_commit(&sm.mma_o);
    }

    // ---- 6. combine in distributed shared memory
    const int DS = kD / (int)C;
    cluster_wait();   // every CTA of the cluster is past step 2: its staging area takes pushes
    {
        if (!tc::mbar_wait(&sm.mma_o, 0) && lane == 0) {
            sm.timed_out = 1;
            if (p.status) atomicExch(p.status, 1);
        }
        __syncwarp();
        tc::tc_fence_after();
        const int qtr = warp & 3, t0 = 2 * (warp >> 2);
        const uint32_t recv = tc::smem_u32(sm.raw + kRecvOff);
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const int t = t0 + tt;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * qtr) << 16) + kColO + 16 * t, r);
            tc::tmem_ld_wait();
            const int d = 128 * t + 32 * qtr + lane;
            const uint32_t owner = (uint32_t)(d / DS);
            const int dd = d - (int)owner * DS;
            const uint32_t a = cl::map_rank(recv + (uint32_t)(((int)rank * DS + dd) * kH * 4), owner);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
                st_cluster_v4(a + 16 * v4, __uint_as_float(r[4 * v4]), __uint_as_float(r[4 * v4 + 1]),
                              __uint_as_float(r[4 * v4 + 2]), __uint_as_float(r[4 * v4 + 3]));
        }
        if (tid < kH * (int)C) {
            const uint32_t owner = (uint32_t)(tid / kH);
            const int h = tid % kH;
            const uint32_t a = tc::smem_u32(sm.raw + kRecvMlOff + ((int)rank * kH + h) * 8);
            cl::st_v2f(cl::map_rank(a, owner), sm.ml[h][0], sm.ml[h][1]);
        }
    }
    tc::tc_fence_before();
    cluster_arrive();
    cluster_wait();   // every slice has arrived; no CTA touches another's memory after this
    const float* Rv = reinterpret_cast<const float*>(sm.raw + kRecvOff);
    const float* Rml = reinterpret_cast<const float*>(sm.raw + kRecvMlOff);
    float* cw = reinterpret_cast<float*>(sm.raw + kCwOff);
    if (tid < kH) {
        float M = -INFINITY;
        for (uint32_t c = 0; c < C; ++c) M = fmaxf(M, Rml[((int)c * kH + tid) * 2]);
        const float Mu = M == -INFINITY ? 0.0f : M;
        float L = 0.0f;
        for (uint32_t c = 0; c < C; ++c) {
            const float wgt = exp2f(Rml[((int)c * kH + tid) * 2] - Mu);
            cw[c * kH + tid] = wgt;
            L += Rml[((int)c * kH + tid) * 2 + 1] * wgt;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (uint32_t c = 0; c < C; ++c) cw[c * kH + tid] *= inv;
        if (p.lse && rank == 0)
            p.lse[(int64_t)bq * kH + tid] = L > 0.0f ? (Mu + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
    {
        // item = (dim d of the slice, heads 4 hq .. 4 hq + 3); lanes 4 apart hold dims d, d + 1
        uint16_t* out = p.out + (int64_t)bq * kH * kD + (int)rank * DS;
        for (int base = 0; base < DS * 4; base += kTT) {
            const int it = base + tid;
            const int d = it >> 2, hq = it & 3;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (d < DS) {
                for (uint32_t c = 0; c < C; ++c) {
                    const float4 x = *reinterpret_cast<const float4*>(Rv + (((int)c * DS + d) * kH + 4 * hq));
                    acc[0] += x.x * cw[c * kH + 4 * hq];
                    acc[1] += x.y * cw[c * kH + 4 * hq + 1];
                    acc[2] += x.z * cw[c * kH + 4 * hq + 2];
                    acc[3] += x.w * cw[c * kH + 4 * hq + 3];
                }
            }
            float nb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) nb[i] = __shfl_xor_sync(0xFFFFFFFFu, acc[i], 4);
            if (d < DS && (d & 1) == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<uint32_t*>(out + (4 * hq + i) * kD + d) = pack_bf16(acc[i], nb[i]);
            }
        }
    }

    // ---- teardown: copies and MMAs have landed (bounded waits again after a timeout), free TMEM
    __syncthreads();
    if (sm.timed_out && tid == 0) {
        (void)tc::mbar_wait(&sm.mma_s, 0);
        (void)tc::mbar_wait(&sm.mma_o, 0);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

DeviceOnce g_attr;
bool g_nonportable[kMaxDevices];

int smem_bytes() { return (int)sizeof(TcAttnSmem); }

bool set_attributes() {
    return g_attr.run([] {
        cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return e;
        }
        const int d = current_device();
        g_nonportable[d] =
            cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
        if (!g_nonportable[d]) (void)cudaGetLastError();
        return cudaSuccess;
    }) == cudaSuccess;
}

bool nonportable() {
    const int d = current_device();
    return d >= 0 && d < kMaxDevices && g_nonportable[d];
}

struct ClusterOcc {
    int n[17];
};
DeviceValue<ClusterOcc> g_occ;

int max_active_clusters(int C) {
    const ClusterOcc occ = g_occ.get(
        [] {
            ClusterOcc o{};
            for (int c = 1; c <= (nonportable() ? 16 : 8); c <<= 1) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3(c, 1);
                cfg.blockDim = dim3(kTT);
                cfg.dynamicSmemBytes = smem_bytes();
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = c;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                if (cudaOccupancyMaxActiveClusters(&o.n[c], attn_tc_kernel, &cfg) != cudaSuccess) {
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

int attn_tc_cluster_size(int B, int Q, int k, int window, int* main_per_cta, int* swa_per_cta) {
    const int bq = B * Q;
    if (bq <= 0 || !set_attributes()) return 0;
    const int sms = device_sm_count();
    for (int C = nonportable() ? 16 : 8; C >= 1; C >>= 1) {
        if ((int64_t)bq * C > sms) continue;
        const int km = (k + C - 1) / C, kw = (window + C - 1) / C;
        if (km > kMaxMain || kw > kMaxRows - kMaxMain || km + kw > kMaxRows) return 0;   // smaller C: more rows
        if (max_active_clusters(C) >= bq) {
            *main_per_cta = km;
            *swa_per_cta = kw;
            return C;
        }
    }
    return 0;
}

cudaError_t launch_attn_tc(AttnParams& p, int C, cudaStream_t st) {
    if (!set_attributes()) return cudaErrorInvalidValue;
    return launch_ex(attn_tc_kernel, dim3(C, p.B * p.Q), dim3(kTT), smem_bytes(), st, C, p);
}

}  // namespace csa2
