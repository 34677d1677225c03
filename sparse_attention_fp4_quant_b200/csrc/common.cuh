// common.cuh -- device helpers shared by the CSA2 kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int kD = CSA2_D;
constexpr int kH = CSA2_H;
constexpr int kIH = CSA2_IH;
constexpr int kID = CSA2_ID;
constexpr int kBlk = CSA2_BLOCK;
// The CTA budget that split counts are derived from (B200's 148 SMs).  Split
// counts fix workspace sizes, which callers compute on the host without a
// device, so this stays a constant; the choice of kernel and cluster size uses
// the device's own SM count (device_sm_count).
constexpr int kSplitSMs = 148;

// ---- formats -------------------------------------------------------------

// E4M3 (FN) byte -> float, via the hardware fp8x2 -> f16x2 conversion.
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    uint32_t h2;
    uint16_t in = (uint16_t)(byte & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Four E4M3 bytes of a word -> four floats.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float out[4]) {
    uint32_t lo, hi;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(lo) : "h"((uint16_t)(w & 0xFFFFu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hi) : "h"((uint16_t)(w >> 16)));
    out[0] = __half2float(__ushort_as_half((unsigned short)(lo & 0xFFFFu)));
    out[1] = __half2float(__ushort_as_half((unsigned short)(lo >> 16)));
    out[2] = __half2float(__ushort_as_half((unsigned short)(hi & 0xFFFFu)));
    out[3] = __half2float(__ushort_as_half((unsigned short)(hi >> 16)));
}

// Non-negative float -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return (uint32_t)(r & 0xFFu);
}

// E2M1 nibble -> float: magnitude index e.m with bias 1, exponent 0 subnormal.
__device__ __forceinline__ float e2m1_to_f32(uint32_t nib) {
    uint32_t mag = nib & 7u;
    uint32_t e = mag >> 1, m = mag & 1u;
    uint32_t bits = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
    bits |= (nib & 8u) << 28;
    return __uint_as_float(bits);
}

// Eight E2M1 codes of a word (nibble n = channel n) -> eight signed int8 of the
// doubled values (2 * e2m1, in [-12, 12]), as two words of four int8.
// Byte-table lookups through PRMT: magnitudes from one table, negatives from
// another, then a per-byte select on the sign bit.
__device__ __forceinline__ void e2m1x8_to_i8x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t P0 = 0x03020100u, P1 = 0x0C080604u;   // 0 1 2 3 | 4 6 8 12
    const uint32_t N0 = 0xFDFEFF00u, N1 = 0xF4F8FAFCu;   // 0 -1 -2 -3 | -4 -6 -8 -12
    uint32_t mag = w & 0x77777777u;
    uint32_t mhi = mag >> 16;
    uint32_t p, n, sel;
    p = __byte_perm(P0, P1, mag);
    n = __byte_perm(N0, N1, mag);
    sel = ((w >> 1) & 0x4444u) | 0x3210u;
    lo = __byte_perm(p, n, sel);
    p = __byte_perm(P0, P1, mhi);
    n = __byte_perm(N0, N1, mhi);
    sel = ((w >> 17) & 0x4444u) | 0x3210u;
    hi = __byte_perm(p, n, sel);
}

// ---- order keys ----------------------------------------------------------

// fp32 score -> uint32 whose unsigned order is the float order (-0 == +0).
__device__ __forceinline__ uint32_t score_key(float s) {
    s = __fadd_rn(s, 0.0f);  // -0 -> +0
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- indexer-K cache layout ---------------------------------------------
// Codes: tiles of 128 entries stored as the tensor core reads its K-major
// operand without swizzle: 8-row x 16-byte core matrices, the two 16-byte
// halves of a row 128 bytes apart, row groups of 8 at 256 bytes.  For entry e
// (counted over the whole [B][cap] cache, cap a multiple of 128), half kc of its
// 32 code bytes starts at ik_code_off(e, kc).  Scales: row-major, 4 bytes per
// entry at ik_scale_off(e).
__host__ __device__ __forceinline__ int64_t ik_code_off(int64_t e, int kc) {
    return ((e >> 7) << 12) + (((e >> 3) & 15) << 8) + ((int64_t)kc << 7) + ((e & 7) << 4);
}

__host__ __device__ __forceinline__ int64_t ik_scale_off(int64_t e) { return e * 4; }

// Maximum over the 8 lanes of an aligned lane octet (one pool block of 8
// consecutive entries), in position order: a later score replaces the running
// maximum only when strictly larger, so of equal maxima (+0 and -0) the first wins.
__device__ __forceinline__ float block_max8(float score, int lane) {
    float mx = score;
#pragma unroll
    for (int o = 1; o < kBlk; o <<= 1) {
        const float other = __shfl_xor_sync(0xFFFFFFFFu, mx, o);
        const float earlier = (lane & o) ? other : mx, later = (lane & o) ? mx : other;
        mx = later > earlier ? later : earlier;
    }
    return mx;
}

__device__ __forceinline__ int n_visible(int64_t q_pos, int64_t n_entries, int m, int64_t cap) {
    int64_t v = (q_pos + 1) / (m > 0 ? m : 1);
    if (n_entries > cap) n_entries = cap;
    if (v > n_entries) v = n_entries;
    if (v < 0) v = 0;
    return (int)v;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Programmatic dependent launch: let the next kernel of the stream be scheduled
// now (it waits in its own pdl_enter), then wait until the previous kernel of
// the stream has completed and its writes are visible.  Every kernel calls it
// before touching global memory; without a programmatic predecessor the wait
// returns at once.
__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.launch_dependents;\n\tgriddepcontrol.wait;" ::: "memory");
}

}  // namespace csa2
