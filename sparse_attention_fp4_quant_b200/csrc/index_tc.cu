// index_tc.cu -- FP4 index scoring on the tcgen05 tensor cores, fused with the
// exact Top-K (Full layers: csa2_index_topk; Reindex layers: csa2_pool_topk).
//
// Scoring as a block-scaled FP4 MMA.  A = 128 indexer-K rows (E2M1, K = 64
// channels) with their E4M3 block scales; B = the query as a block-diagonal
// 16 x 64 operand: column n = 4 h + b holds head h's codes in block b only, so
// accumulator column n of row t is exactly one block's
//   T[h][b] = (sum over 16 channels of q k) * sq[h][b] * sk[b]
// (at most 20 significant bits: exact in fp32 whatever the MMA's summation
// order).  The epilogue then sums the blocks and heads in the fixed order
// ((T0 + T1) + T2) + T3 and ((w0 r0 + w1 r1) + w2 r2) + w3 r3 on CUDA cores,
// which reproduces the defined score bit for bit.
//
// One CTA = one share of one query's candidates.  Warp 0 streams 128-row
// tiles with TMA (32-byte swizzle) and copies the scale bytes with 4-byte
// cp.async straight into the TMEM-copy layout; warp 1 owns TMEM, copies the
// scales to TMEM and issues the MMAs; warps 2-5 read the accumulators,
// finish the scores and run the Top-K filter (named barrier 1).  The last CTA
// of a query merges the shares.  Every mbarrier wait is bounded; a timeout
// sets the workspace status word and the CTA winds down.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "topk.cuh"

namespace csa2 {
namespace {

constexpr int kTile = 128;       // rows per MMA (M)
constexpr int kTPS = 4;          // tiles per pipeline stage
constexpr int kStages = 4;       // smem stages
constexpr int kAcc = 2;          // accumulator stages
constexpr int kEpiT0 = 64, kEpiN = 256;   // 8 epilogue warps: two per TMEM lane quarter
constexpr int kThreads = kEpiT0 + kEpiN;
constexpr int kTPG = kTPS / 2;   // tiles of a stage per epilogue warp group
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColAcc = 0, kColSfa = kAcc * kTPS * 16, kColSfb = kColSfa + kStages * kTPS * 4;
static_assert(kColSfb + 4 <= kTmemCols, "TMEM columns");
constexpr uint32_t kIdesc = tc::idesc_mxf4nvf4(128, 16);
constexpr int kPoolPerTile = kTile / kBlk;   // 16 pool blocks of 8 rows per tile

template <int CAP>
struct TcSmem {
    uint8_t A[kStages][kTPS][kTile * 32];   // K-major, 32-byte swizzle (written by TMA)
    uint8_t SF[kStages][kTPS][512];         // scale bytes in the 32 x (4 x 4 B) TMEM-copy layout
    uint8_t Bq[16 * 32];                    // block-diagonal query, no swizzle, K-major
    uint8_t SFB[512];                       // its scales, TMEM-copy layout
    uint64_t full[kStages], empty[kStages], accfull[kAcc], accempty[kAcc], done;
    uint32_t tmem_base;
    int abort_flag;
    int last;
    typename TopK<kEpiN, CAP, 1, kEpiT0>::Smem topk;
};

template <class SM>
__device__ __forceinline__ void raise_abort(SM& s, int32_t* status) {
    *reinterpret_cast<volatile int*>(&s.abort_flag) = 1;
    if (status) atomicExch(status, 1);
}

template <class SM>
__device__ __forceinline__ bool aborted(SM& s) { return *reinterpret_cast<volatile int*>(&s.abort_flag) != 0; }

// OR of `v` over the epilogue warps, through named barrier 1 (every epilogue
// thread gets the same answer, so they all leave or all stay).
__device__ __forceinline__ bool epilogue_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kEpiN)
        : "memory");
    return r != 0;
}

template <int MODE, int CAP>  // MODE 0 = dense range (index Top-K), 1 = pool blocks (pool Top-K)
__global__ void __launch_bounds__(kThreads, 2)
    index_tc_kernel(SelectParams p, const __grid_constant__ CUtensorMap tmap) {
    using TKE = TopK<kEpiN, CAP, 1, kEpiT0>;
    using TcSmem = csa2::TcSmem<CAP>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align by pointer arithmetic on the shared array (an integer round trip would
    // hide the address space and turn every shared access into a generic one)
    TcSmem& s = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bq = blockIdx.y, share = blockIdx.x, S = gridDim.x;
    const int b = bq / p.Q;
    const int k = p.k;
    const int nvis = n_visible(p.q_pos[bq], p.n_entries[b], p.m, p.cap);
    const int64_t row_base = (int64_t)b * p.cap;

    // this share's candidates: dense = entries [lo, hi); pool = pool slots [lo, hi)
    int lo, hi, ntiles;
    if (MODE == 0) {
        int chunk = (((nvis + S - 1) / S) + (kTPS * kTile - 1)) / (kTPS * kTile) * (kTPS * kTile);
        lo = min(nvis, share * chunk);
        hi = min(nvis, lo + chunk);
        ntiles = (hi - lo + kTile - 1) / kTile;
    } else {
        int chunk = (((p.P + S - 1) / S) + (kTPS * kPoolPerTile - 1)) / (kTPS * kPoolPerTile) * (kTPS * kPoolPerTile);
        lo = min(p.P, share * chunk);
        hi = min(p.P, lo + chunk);
        ntiles = (hi - lo + kPoolPerTile - 1) / kPoolPerTile;
    }
    const int nstages = (ntiles + kTPS - 1) / kTPS;
    const int32_t* pool = (MODE == 1) ? p.pool + (int64_t)bq * p.P : nullptr;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            tc::mbar_init(&s.full[i], 1 + 32);   // expect_tx arrive + 32 cp.async arrivals
            tc::mbar_init(&s.empty[i], 1);       // MMA commit
        }
        for (int i = 0; i < kAcc; ++i) {
            tc::mbar_init(&s.accfull[i], 1);     // MMA commit
            tc::mbar_init(&s.accempty[i], kEpiN);
        }
        tc::mbar_init(&s.done, 1);
        s.abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&s.tmem_base, kTmemCols);
        // block-diagonal query: row n = 4h + b keeps head h's 8 code bytes of block b
        const uint8_t* q = p.q + (int64_t)bq * 128;
        const uint8_t* qs = p.q_sc + (int64_t)bq * 16;
        for (int i = lane; i < 16 * 32; i += 32) s.Bq[i] = 0;
        for (int i = lane; i < 512; i += 32) s.SFB[i] = 0;
        __syncwarp();
        if (lane < 16) {
            const int n = lane, h = n >> 2, blk = n & 3;
            const int kc = blk >> 1, off = 8 * (blk & 1);
            uint8_t* row = s.Bq + (n >> 3) * 256 + kc * 128 + (n & 7) * 16 + off;
            const uint8_t* src = q + 32 * h + 8 * blk;
#pragma unroll
            for (int j = 0; j < 8; ++j) row[j] = src[j];
#pragma unroll
            for (int j = 0; j < 4; ++j) s.SFB[16 * n + j] = qs[4 * h + j];
        }
        tc::fence_proxy_async_smem();
    }
    __syncthreads();
    const uint32_t tbase = s.tmem_base;
    int32_t* status = p.status;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint8_t* iks = p.ik_sc;
        int issued = 0;
        for (int t = 0; t < nstages; ++t) {
            const int slot = t % kStages;
            const uint32_t ph = (uint32_t)(t / kStages) & 1u;
            int ok = 1;
            if (lane == 0) ok = tc::mbar_wait(&s.empty[slot], ph ^ 1u);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (lane == 0 && !ok) raise_abort(s, status);
            if (__any_sync(0xFFFFFFFFu, !ok || aborted(s))) break;   // warp-uniform
            uint32_t bytes = 0;
            if (MODE == 0) {
                for (int i = 0; i < kTPS; ++i)
                    if (t * kTPS + i < ntiles) bytes += kTile * 32;
            } else {
                for (int i = 0; i < kTPS; ++i) {
                    const int g = t * kTPS + i;
                    if (g >= ntiles) break;
                    for (int j = 0; j < kPoolPerTile; ++j) {
                        const int sl = lo + g * kPoolPerTile + j;
                        if (sl < hi) {
                            const int blk = __ldg(pool + sl);
                            if (blk >= 0 && (int64_t)blk * kBlk < nvis) bytes += kBlk * 32;
                        }
                    }
                }
            }
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(&s.full[slot], bytes);
                for (int i = 0; i < kTPS; ++i) {
                    const int g = t * kTPS + i;
                    if (g >= ntiles) break;
                    if (MODE == 0) {
                        tc::tma_load_2d(s.A[slot][i], &tmap, 0, (int)(row_base + lo + g * kTile), &s.full[slot]);
                    } else {
                        for (int j = 0; j < kPoolPerTile; ++j) {
                            const int sl = lo + g * kPoolPerTile + j;
                            if (sl >= hi) break;
                            const int blk = __ldg(pool + sl);
                            if (blk >= 0 && (int64_t)blk * kBlk < nvis)
                                tc::tma_load_2d(s.A[slot][i] + 256 * j, &tmap, 0, (int)(row_base + (int64_t)blk * kBlk),
                                                &s.full[slot]);
                        }
                    }
                }
            }
            // scale bytes: row m = lane + 32 j goes to byte 16 * lane + 4 * j
            for (int i = 0; i < kTPS; ++i) {
                const int g = t * kTPS + i;
                if (g >= ntiles) break;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
                    int64_t e = -1;
                    if (MODE == 0) {
                        const int ee = lo + g * kTile + m;
                        if (ee < hi) e = ee;
                    } else {
                        const int sl = lo + g * kPoolPerTile + (m >> 3);
                        if (sl < hi) {
                            const int blk = __ldg(pool + sl);
                            const int64_t ee = (int64_t)blk * kBlk + (m & 7);
                            if (blk >= 0 && ee < nvis) e = ee;
                        }
                    }
                    if (e >= 0) tc::cp_async_4(&s.SF[slot][i][16 * lane + 4 * j], iks + (row_base + e) * 4);
                }
            }
            tc::cp_async_arrive_noinc(&s.full[slot]);
            ++issued;
        }
        // never leave copies in flight: wait (bounded) for the stages still pending
        if (lane == 0) {
            for (int t = max(0, issued - kStages); t < issued; ++t)
                if (!tc::mbar_wait(&s.full[t % kStages], (uint32_t)(t / kStages) & 1u)) raise_abort(s, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            tc::tc_fence_after();
            const uint32_t sa_sfb = tc::smem_u32(s.SFB);
            tc::tmem_cp_32x128_x4(tbase + kColSfb, tc::smem_desc(sa_sfb, 16, 128, tc::kLayoutNone));
            const uint64_t bdesc = tc::smem_desc(tc::smem_u32(s.Bq), 128, 256, tc::kLayoutNone);
            for (int t = 0; t < nstages; ++t) {
                const int slot = t % kStages;
                const uint32_t ph = (uint32_t)(t / kStages) & 1u;
                const int a = t % kAcc;
                const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
                if (!tc::mbar_wait(&s.full[slot], ph) || !tc::mbar_wait(&s.accempty[a], aph ^ 1u)) {
                    raise_abort(s, status);
                    break;
                }
                if (aborted(s)) break;
                tc::tc_fence_after();
                tc::fence_proxy_async_smem();   // scale bytes came through cp.async (generic proxy)
                for (int i = 0; i < kTPS; ++i) {
                    if (t * kTPS + i >= ntiles) break;
                    const uint32_t sfa = tbase + kColSfa + (uint32_t)(slot * kTPS + i) * 4;
                    tc::tmem_cp_32x128_x4(sfa, tc::smem_desc(tc::smem_u32(s.SF[slot][i]), 16, 128, tc::kLayoutNone));
                    const uint64_t adesc = tc::smem_desc(tc::smem_u32(s.A[slot][i]), 16, 256, tc::kLayoutSw32);
                    tc::mma_mxf4nvf4(tbase + kColAcc + (uint32_t)(a * kTPS + i) * 16, adesc, bdesc, kIdesc, 0u, sfa,
                                     tbase + kColSfb);
                }
                tc::tc_commit(&s.empty[slot]);
                tc::tc_commit(&s.accfull[a]);
            }
            tc::tc_commit(&s.done);
            if (!tc::mbar_wait(&s.done, 0)) raise_abort(s, status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        TKE tk(s.topk);
        tk.init();
        const int quarter = warp & 3;             // TMEM lanes this warp may read
        const int group = (warp - 2) >> 2;        // tiles 2*group, 2*group+1 of each stage
        const int row = quarter * 32 + lane;
        const float w0 = __ldg(p.w + (int64_t)bq * 4 + 0), w1 = __ldg(p.w + (int64_t)bq * 4 + 1);
        const float w2 = __ldg(p.w + (int64_t)bq * 4 + 2), w3 = __ldg(p.w + (int64_t)bq * 4 + 3);
        float* bm = (MODE == 0 && p.blockmax) ? p.blockmax + (int64_t)bq * p.nb_cap : nullptr;
        bool stop = false;
        for (int t = 0; t < nstages && !stop; ++t) {
            const int a = t % kAcc;
            const uint32_t aph = (uint32_t)(t / kAcc) & 1u;
            const bool ok = __all_sync(0xFFFFFFFFu, tc::mbar_wait(&s.accfull[a], aph));  // warp-uniform
            if (!ok && lane == 0) raise_abort(s, status);
            tc::tc_fence_after();
            uint32_t v[kTPG][16];
#pragma unroll
            for (int j = 0; j < kTPG; ++j) {
                const int i = kTPG * group + j;
                if (ok) {
                    tc::tmem_ld_32x32b_x16(tbase + ((uint32_t)(quarter * 32) << 16) + kColAcc + (uint32_t)(a * kTPS + i) * 16,
                                           v[j]);
                }
            }
            if (ok) tc::tmem_ld_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(&s.accempty[a]);
            if (epilogue_any(aborted(s))) {   // also the barrier that orders the previous offers
                stop = true;
                break;
            }
            if (tk.count() > CAP - kTPS * kTile) tk.compact(k);
            const auto th = tk.threshold();
#pragma unroll
            for (int j = 0; j < kTPG; ++j) {
                const int g = t * kTPS + kTPG * group + j;
                int64_t e = -1;
                if (g < ntiles) {
                    if (MODE == 0) {
                        const int ee = lo + g * kTile + row;
                        if (ee < hi) e = ee;
                    } else {
                        const int sl = lo + g * kPoolPerTile + (row >> 3);
                        if (sl < hi) {
                            const int blk = __ldg(pool + sl);
                            const int64_t ee = (int64_t)blk * kBlk + (row & 7);
                            if (blk >= 0 && ee < nvis) e = ee;
                        }
                    }
                }
                const bool valid = e >= 0;
                float score = -INFINITY;
                if (valid) {
                    const float* T = reinterpret_cast<const float*>(v[j]);
                    float r[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float d = __fadd_rn(__fadd_rn(__fadd_rn(T[4 * h], T[4 * h + 1]), T[4 * h + 2]), T[4 * h + 3]);
                        r[h] = d > 0.0f ? d : 0.0f;
                    }
                    score = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(w0, r[0]), __fmul_rn(w1, r[1])), __fmul_rn(w2, r[2])),
                                      __fmul_rn(w3, r[3]));
                }
                if (MODE == 0 && bm && g < ntiles) {
                    float m8 = score;
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) m8 = fmaxf(m8, __shfl_xor_sync(0xFFFFFFFFu, m8, o));
                    if ((lane & 7) == 0 && valid) bm[e >> 3] = m8;
                }
                tk.offer(th, valid, score_key(valid ? score : 0.0f), (int32_t)(valid ? e : 0));
            }
        }
        if (!stop && MODE == 0 && bm) {  // blocks with no visible position
            const int64_t jb = (nvis + kBlk - 1) / kBlk;
            const int64_t rest = p.nb_cap - jb;
            if (rest > 0) {
                const int64_t cs = (rest + S - 1) / S;
                const int64_t j0 = jb + (int64_t)share * cs, j1 = min(p.nb_cap, j0 + cs);
                for (int64_t j = j0 + (tid - kEpiT0); j < j1; j += kEpiN) bm[j] = -INFINITY;
            }
        }
        if (!stop) tk.finish(k);
    }
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tbase, kTmemCols);
    if (warp < 2 || aborted(s)) return;

    // ---------------------------------------------------------------- output
    TKE tk(s.topk);
    const int et = tid - kEpiT0;
    if (S > 1) {
        const int cnt = tk.count();
        const int64_t off = ((int64_t)bq * S + share) * k;
        for (int i = et; i < cnt; i += kEpiN) {
            p.cand_key[off + i] = tk.key_at(i);
            p.cand_pos[off + i] = tk.pos_at(i);
        }
        if (et == 0) p.cand_cnt[(int64_t)bq * S + share] = cnt;
        __threadfence();
        TKE::sync();
        if (et == 0) s.last = (atomicAdd(&p.counters[bq], 1) == S - 1);
        TKE::sync();
        if (!s.last) return;
        __threadfence();
        tk.init();
        for (int c = 0; c < S; ++c) {
            const int n = __ldcg(&p.cand_cnt[(int64_t)bq * S + c]);
            const int64_t coff = ((int64_t)bq * S + c) * k;
            for (int base = 0; base < n; base += kEpiN) {
                tk.make_room(k, kEpiN);
                const int i = base + et;
                const bool valid = i < n;
                const uint32_t key = valid ? __ldcg(&p.cand_key[coff + i]) : 0u;
                const int32_t pos = valid ? __ldcg(&p.cand_pos[coff + i]) : 0;
                tk.offer(valid, key, pos);
            }
        }
        tk.finish(k);
        if (et == 0) p.counters[bq] = 0;
    }
    const int cnt = tk.count();
    tk.sort_positions(cnt);
    for (int i = et; i < k; i += kEpiN) p.out[(int64_t)bq * k + i] = i < cnt ? tk.pos_at(i) : -1;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

}  // namespace

bool index_tc_supported(const SelectParams& p) {
    return (((uintptr_t)p.ik) & 15u) == 0 && (int64_t)p.B * p.cap < (int64_t(1) << 31);
}

template <int MODE, int CAP>
cudaError_t launch_tc(SelectParams& p, int S, cudaStream_t st, const CUtensorMap& map) {
    const int smem = (int)sizeof(TcSmem<CAP>) + 1024;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<MODE, CAP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    dim3 grid(S, p.B * p.Q);
    index_tc_kernel<MODE, CAP><<<grid, kThreads, smem, st>>>(p, map);
    return cudaGetLastError();
}

cudaError_t launch_index_tc(int op, SelectParams& p, int S, cudaStream_t st) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    const int mode = (op == CSA2_OP_POOL_TOPK) ? 1 : 0;
    CUtensorMap map;
    cuuint64_t dims[2] = {32, (cuuint64_t)p.B * (cuuint64_t)p.cap};
    cuuint64_t strides[1] = {32};
    cuuint32_t box[2] = {32, (cuuint32_t)(mode == 0 ? kTile : kBlk)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)p.ik, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // the buffer must hold k survivors plus one stage of offers
    if (p.k <= 2048 - kTPS * kTile) return mode == 0 ? launch_tc<0, 2048>(p, S, st, map) : launch_tc<1, 2048>(p, S, st, map);
    return mode == 0 ? launch_tc<0, 4096>(p, S, st, map) : launch_tc<1, 4096>(p, S, st, map);
}

}  // namespace csa2
