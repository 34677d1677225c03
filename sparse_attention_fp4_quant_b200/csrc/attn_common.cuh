// attn_common.cuh -- device pieces shared by the sparse-attention kernels:
// exact FP4 / FP8 -> f16 decoding, the row-quarter gather of one key slot,
// ldmatrix / mma.sync wrappers, and the swizzled 16-bit row layout.
//
// Key slots of a query: [0, k) are the main rows idx[0..k), [k, k + W) are the
// window tokens i - W + 1 .. i.  A slot is live if its row exists and (for the
// window) the token lies in [max(s, i - W + 1), i] and in the stored SWA rows.
// Keys and values are f16 in shared memory: FP4 rows dequantise exactly (the
// hardware E2M1 -> f16 conversion, then an exact f16 multiply by the block
// scale); an SWA row is kept as its E4M3 values (exact in f16) and its fp32
// token scale multiplies the logit and the probability.  The bf16 query is
// brought into f16 range by a power of two that the logits take back.
#pragma once
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

constexpr int kRowB = kD * 2;   // bytes per 16-bit row of 512

// 16-byte chunk `chunk` of 16-bit row `row`, XOR-swizzled by row & 7.
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return (uint32_t)(row * kRowB + ((chunk ^ (row & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// 8 E2M1 codes (nibble n = dim n) times the block scale (f16x2 s2) -> 8 f16,
// by the hardware E2M1 -> f16 conversion.  Every E2M1 x E4M3 product (at most
// 5 significant bits, 2^-10 .. 2688) is exact in f16, so the multiply is exact.
__device__ __forceinline__ uint4 fp4x8_to_f16(uint32_t w, uint32_t s2) {
    uint32_t r0, r1, r2, r3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\tcvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\tcvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
        : "r"(w));
    return make_uint4(f16x2_mul(r0, s2), f16x2_mul(r1, s2), f16x2_mul(r2, s2), f16x2_mul(r3, s2));
}

// 4 E4M3 bytes -> 4 f16 (exact).
__device__ __forceinline__ uint2 fp8x4_to_f16(uint32_t w) {
    uint32_t lo, hi;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"((uint16_t)(w & 0xFFFFu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"((uint16_t)(w >> 16)));
    return make_uint2(lo, hi);
}

// Power-of-two exponent e >= 0 that brings max |q| below 2^15, so q 2^-e fits f16
// exactly (bf16 has 8 significant bits) except for values under 2^-14.
__device__ __forceinline__ int q_prescale_exp(float maxabs) {
    const int ex = (int)((__float_as_uint(maxabs) >> 23) & 0xFFu) - 127;
    return max(0, ex - 14);
}

// 8 bf16 (a 16-byte chunk) times 2^-e -> 8 f16.
__device__ __forceinline__ uint4 bf16x8_to_f16(uint4 v, float mul) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack_f16(__uint_as_float(w[i] << 16) * mul, __uint_as_float(w[i] & 0xFFFF0000u) * mul);
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ float bf16x8_maxabs(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
    return m;
}

__device__ __forceinline__ void mma_f16(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// One quarter (128 dims) of one key row, held in registers between its load
// and its dequantisation.
struct RowQuarter {
    uint4 raw[8];   // FP4: raw[0..3] = 64 code bytes; FP8: raw[0..7] = 128 bytes
    uint2 sc;       // FP4: the 8 block scales of the quarter
    float fac;      // FP8: the token scale
    int kind;       // 0 = dead slot, 1 = FP4 main row, 2 = FP8 window row
};

// Issue the loads of quarter qq (128 dims) of key slot `slot`: a main row's id comes
// from shared memory (ids[slot - id0]), so its row loads never wait on an id load.
__device__ __forceinline__ void fetch_quarter_id(const AttnParams& p, int b, int slot, int qq, const int32_t* ids,
                                                 int id0, int64_t i_pos, int64_t lo, int64_t pos0, int64_t nmain,
                                                 RowQuarter& q) {
    q.kind = 0;
    if (slot < p.k) {
        const int32_t e = ids[slot - id0];
        if (e >= 0 && e < nmain) {
            q.kind = 1;
            const int64_t row = (int64_t)b * p.cap + e;
            const uint4* cs = reinterpret_cast<const uint4*>(p.lat + row * (kD / 2) + 64 * qq);
#pragma unroll
            for (int v = 0; v < 4; ++v) q.raw[v] = __ldg(cs + v);
            q.sc = __ldg(reinterpret_cast<const uint2*>(p.lat_sc + row * (kD / 16) + 8 * qq));
        }
    } else if (slot < p.slots_total) {
        const int64_t tau = i_pos - p.window + 1 + (slot - p.k);
        const int64_t rr = tau - pos0;
        if (tau >= lo && tau <= i_pos && rr >= 0 && rr < p.T) {
            q.kind = 2;
            const int64_t row = (int64_t)b * p.T + rr;
            q.fac = __ldg(p.swa_sc + row);
            const uint4* cs = reinterpret_cast<const uint4*>(p.swa + row * kD + 128 * qq);
#pragma unroll
            for (int v = 0; v < 8; ++v) q.raw[v] = __ldg(cs + v);
        }
    }
}

// Loads of read-only data as volatile asm: they issue in program order, so a
// thread can put all of its loads in flight before it consumes any of them.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Which row a key slot reads (the main row id e of slot < k is given):
// 1 = FP4 main row, 2 = FP8 window row, 0 = dead; `row` = its row in the cache.
__device__ __forceinline__ int slot_row(const AttnParams& p, int b, int slot, int32_t e, int64_t i_pos, int64_t lo,
                                        int64_t pos0, int64_t nmain, int64_t& row) {
    if (slot < p.k) {
        if (e >= 0 && e < nmain) {
            row = (int64_t)b * p.cap + e;
            return 1;
        }
    } else if (slot < p.slots_total) {
        const int64_t tau = i_pos - p.window + 1 + (slot - p.k);
        const int64_t rr = tau - pos0;
        if (tau >= lo && tau <= i_pos && rr >= 0 && rr < p.T) {
            row = (int64_t)b * p.T + rr;
            return 2;
        }
    }
    return 0;
}

// Issue the loads of quarter qq of a row chosen by slot_row.
__device__ __forceinline__ void issue_quarter(const AttnParams& p, int kind, int64_t row, int qq, RowQuarter& q) {
    q.kind = kind;
    if (kind == 1) {
        const uint8_t* cs = p.lat + row * (kD / 2) + 64 * qq;
#pragma unroll
        for (int v = 0; v < 4; ++v) q.raw[v] = ld_nc_v4(cs + 16 * v);
        q.sc = ld_nc_v2(p.lat_sc + row * (kD / 16) + 8 * qq);
    } else if (kind == 2) {
        q.fac = __uint_as_float(ld_nc_u32(p.swa_sc + row));
        const uint8_t* cs = p.swa + row * kD + 128 * qq;
#pragma unroll
        for (int v = 0; v < 8; ++v) q.raw[v] = ld_nc_v4(cs + 16 * v);
    }
}

__device__ __forceinline__ void store_quarter(uint8_t* K, float* kf, int* kvalid, int r, int qq, const RowQuarter& q) {
    if (q.kind == 1) {
        uint32_t s2[8];   // the 8 block scales as f16 pairs (exact: E4M3 fits f16)
        {
            const uint2 sp = fp8x4_to_f16(q.sc.x), sq = fp8x4_to_f16(q.sc.y);
            const uint32_t pr[4] = {sp.x, sp.y, sq.x, sq.y};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                s2[2 * i] = __byte_perm(pr[i], 0u, 0x1010);       // (low, low)
                s2[2 * i + 1] = __byte_perm(pr[i], 0u, 0x3232);   // (high, high)
            }
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint32_t ws[4] = {q.raw[v].x, q.raw[v].y, q.raw[v].z, q.raw[v].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int word = 4 * v + j;   // 8 dims per word, one scale per 16 dims
                *reinterpret_cast<uint4*>(K + swz(r, 16 * qq + word)) = fp4x8_to_f16(ws[j], s2[word >> 1]);
            }
        }
    } else if (q.kind == 2) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const uint2 a = fp8x4_to_f16(q.raw[v].x), bb = fp8x4_to_f16(q.raw[v].y);
            const uint2 c = fp8x4_to_f16(q.raw[v].z), d = fp8x4_to_f16(q.raw[v].w);
            *reinterpret_cast<uint4*>(K + swz(r, 16 * qq + 2 * v)) = make_uint4(a.x, a.y, bb.x, bb.y);
            *reinterpret_cast<uint4*>(K + swz(r, 16 * qq + 2 * v + 1)) = make_uint4(c.x, c.y, d.x, d.y);
        }
    } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(K + swz(r, 16 * qq + c)) = make_uint4(0, 0, 0, 0);
    }
    if (qq == 0) {
        kvalid[r] = q.kind != 0;
        kf[r] = q.kind == 2 ? q.fac : 1.0f;
    }
}

}  // namespace csa2
