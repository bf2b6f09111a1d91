// common.cuh -- device helpers shared by the sm_100a kernels: element
// conversions through the hardware cvt instructions, bf16 bit handling,
// the device error word, vector memory access.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/fpq.h"

namespace fpq {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ----------------------------------------------------------------- errors

// Record the first device-side error; later ones are dropped.
__device__ __forceinline__ void raise_device_error(uint32_t* err, uint32_t code) {
    if (err) atomicCAS(err, 0u, code);
}

// ----------------------------------------------------------------- bf16

// bf16 pattern -> fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp32 -> bf16 pattern, round to nearest even (hardware cvt, gradual underflow).
__device__ __forceinline__ uint32_t f32_to_bf16(float f) {
    uint16_t h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
    return h;
}
// two fp32 -> packed bf16x2, `lo` in the low half
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ----------------------------------------------------------------- e4m3 / e2m1

// two fp32 -> two E4M3 codes, round to nearest even, finite values saturate
// to +-448; `lo` lands in bits 0..7.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// E4M3 code (low byte of `c`) -> fp32, exact (through the f16x2 converter).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    uint32_t h2;
    uint16_t in = (uint16_t)(c & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// two E4M3 codes (bits 0..15) -> two fp32, exact.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t c2) {
    uint32_t h2;
    uint16_t in = (uint16_t)(c2 & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// two E2M1 codes (bits 0..7, element 0 in bits 0..3) -> two fp32, exact.
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t c2) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2) : "r"(c2 & 0xFFu));
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// ----------------------------------------------------------------- dependent launch

// Wait until the grids this one depends on (programmatic dependent launch)
// have completed and their memory operations are visible; a no-op for a
// kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow dependent grids to be scheduled; they still wait (pdl_wait) for this
// grid's completion before touching its results.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------- exact quotient codes
//
// The fp32-scale formats define a code as the rounding of the correctly
// rounded fp32 quotient q = fp32(x / s).  Instead of a division per element
// (which runs on the reciprocal unit), the code is read off two products
// that bracket q:
//   r = fp32(1/s), r_lo = fp32(r (1 - 2^-20)), r_hi = fp32(r (1 + 2^-20))
// give r_lo < (1/s)(1 - 2^-21) and r_hi > (1/s)(1 + 2^-21), so for x > 0
//   fp32(x r_lo) < (x/s)(1 - 2^-24) <= q <= (x/s)(1 + 2^-24) < fp32(x r_hi)
// (mirrored for x < 0; all zero for x = 0).  Rounding to a narrow format is
// monotone in the value, so when both bracket ends round to the same code,
// q rounds to it too.  Otherwise (q within about 2^-20 relative of a
// rounding boundary, rare) the code is taken from the IEEE division itself.
// Values so small that the products are fp32-subnormal are far below the
// smallest nonzero code and round to signed zero on every path.  The caller
// guarantees 1/s is a normal fp32 number (s >= 2^-126, see reciprocal_ok).

struct QuotientBracket {
    float s, lo, hi;
};

__device__ __forceinline__ QuotientBracket quotient_bracket(float s) {
    const float r = __frcp_rn(s);
    return QuotientBracket{s, __fmul_rn(r, 1.0f - 0x1p-20f), __fmul_rn(r, 1.0f + 0x1p-20f)};
}

// E4M3 codes of fp32(x0/s) (bits 0-7) and fp32(x1/s) (bits 8-15).
__device__ __forceinline__ uint32_t e4m3x2_of_quotients(float x0, float x1, const QuotientBracket& b) {
    uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(x0, b.lo), __fmul_rn(x1, b.lo));
    const uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(x0, b.hi), __fmul_rn(x1, b.hi));
    if (lo != hi) lo = f32x2_to_e4m3x2(__fdiv_rn(x0, b.s), __fdiv_rn(x1, b.s));
    return lo;
}

// Packed pairs of fp32 values in one 64-bit register (element 0 in the low
// half) for the paired fp32 instructions of sm_100: each lane of
// fma.rn.f32x2 / mul.rn.f32x2 is one IEEE round-to-nearest fma / multiply,
// exactly as the scalar instruction.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo_of(uint64_t p) { return __uint_as_float((uint32_t)p); }
__device__ __forceinline__ float hi_of(uint64_t p) { return __uint_as_float((uint32_t)(p >> 32)); }
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// The two fp32 values of a bf16x2 word (exact), as a pair.
__device__ __forceinline__ uint64_t bf16x2_pair(uint32_t w) { return pack2(bf16_lo(w), bf16_hi(w)); }

// Eight E2M1 codes (bits 4i .. 4i + 3 = element i) of four pairs of fp32
// values, round to nearest even, saturating to +-6.
__device__ __forceinline__ uint32_t e2m1x8_of_pairs(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(lo_of(p0)), "f"(hi_of(p0)), "f"(lo_of(p1)), "f"(hi_of(p1)), "f"(lo_of(p2)), "f"(hi_of(p2)),
          "f"(lo_of(p3)), "f"(hi_of(p3)));
    return r;
}

// Four E4M3 codes (byte i = element i) of two pairs of fp32 values, round
// to nearest even, finite values saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x4_of_pairs(uint64_t p0, uint64_t p1) {
    uint32_t r;
    asm("{\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
        "mov.b32 %0, {h0, h1};\n\t}"
        : "=r"(r) : "f"(lo_of(p0)), "f"(hi_of(p0)), "f"(lo_of(p1)), "f"(hi_of(p1)));
    return r;
}

// E4M3 codes of fp32(x / s) for the eight bf16 values of four words (byte i
// of out = element i), from the products with both ends of the quotient
// bracket (lo2 / hi2: the ends as packed pairs), formed two at a time.
// Returns false when any element's two ends give different codes (a
// quotient close to a rounding boundary); `out` is then unusable and the
// caller encodes these elements from correctly rounded divisions.
__device__ __forceinline__ bool e4m3x8_bracketed(const uint32_t (&w)[4], uint64_t lo2, uint64_t hi2, uint2& out) {
    const uint64_t x0 = bf16x2_pair(w[0]), x1 = bf16x2_pair(w[1]), x2 = bf16x2_pair(w[2]), x3 = bf16x2_pair(w[3]);
    out.x = e4m3x4_of_pairs(mul2(x0, lo2), mul2(x1, lo2));
    out.y = e4m3x4_of_pairs(mul2(x2, lo2), mul2(x3, lo2));
    const uint32_t u0 = e4m3x4_of_pairs(mul2(x0, hi2), mul2(x1, hi2));
    const uint32_t u1 = e4m3x4_of_pairs(mul2(x2, hi2), mul2(x3, hi2));
    return ((out.x ^ u0) | (out.y ^ u1)) == 0u;
}

// E4M3 codes of fp32(x / s) for the eight bf16 values of four words, from
// correctly rounded divisions.
__device__ __forceinline__ uint2 e4m3x8_divided(const uint32_t (&w)[4], float s) {
    uint64_t q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = pack2(__fdiv_rn(bf16_lo(w[j]), s), __fdiv_rn(bf16_hi(w[j]), s));
    return make_uint2(e4m3x4_of_pairs(q[0], q[1]), e4m3x4_of_pairs(q[2], q[3]));
}

// ----------------------------------------------------------------- per-block scale tables
//
// For a bf16 amax a = (1 + m/128) 2^(E-127) (m: 7-bit mantissa field, E:
// exponent field) the quotient a / d by a constant d is
// fp32((1 + m/128) / d) 2^(E-127) exactly whenever the result is a normal
// fp32 number (scaling by a power of two commutes with rounding there), and
// likewise the reciprocal and the bracket ends of a scale.  So the per-block
// divisions reduce to 128-entry tables indexed by m plus an exponent add.

struct ScaleTables {
    uint32_t s[128];     // fp32((1 + m/128) / d)
    uint32_t lo[128];    // bracket ends for quotients by s: r (1 - 2^-20), r (1 + 2^-20), r = fp32(1 / s)
    uint32_t hi[128];
};

// Threads 0..127 each fill one entry; the caller synchronizes afterwards.
__device__ __forceinline__ void init_scale_tables(ScaleTables& t, float d) {
    const int m = threadIdx.x;
    if (m < 128) {
        const float sm = __fdiv_rn(1.0f + (float)m * 0x1p-7f, d);
        const float r = __frcp_rn(sm);
        t.s[m] = __float_as_uint(sm);
        t.lo[m] = __float_as_uint(__fmul_rn(r, 1.0f - 0x1p-20f));
        t.hi[m] = __float_as_uint(__fmul_rn(r, 1.0f + 0x1p-20f));
    }
}

// Scale s = fp32(a / d) of a bf16 magnitude pattern a and its bracket ends,
// when E is in [e_min, 254] (the caller's e_min keeps s and 1/s normal);
// false otherwise (zero, tiny, infinite or NaN amax: use the division path).
__device__ __forceinline__ bool table_scale(const ScaleTables& t, uint32_t a, int e_min, float& s, float& lo,
                                            float& hi) {
    const int E = (int)(a >> 7), m = (int)(a & 0x7Fu);
    if (E < e_min || E > 254) return false;
    const int k = (E - 127) << 23;
    s = __uint_as_float(t.s[m] + (uint32_t)k);
    lo = __uint_as_float(t.lo[m] - (uint32_t)k);
    hi = __uint_as_float(t.hi[m] - (uint32_t)k);
    return true;
}

// Whether the bracket applies for divisor s (1/s a normal fp32 number).
__device__ __forceinline__ bool reciprocal_ok(float s) { return s >= 1.17549435e-38f; }

// ----------------------------------------------------------------- absmax

// Largest magnitude pattern of the two bf16 halves of each word, as a packed
// pair of 15-bit magnitudes (integer order = magnitude order for finite
// values; NaN patterns order above infinity, so a NaN propagates).
__device__ __forceinline__ uint32_t abs2(uint32_t w) { return w & 0x7FFF7FFFu; }
// Per half: a value whose magnitude is the larger of the two magnitudes
// (sign bits to be masked off by the caller), NaN if either is NaN.  One
// bf16x2 max-of-magnitudes instruction instead of a mask and an integer max.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }
__device__ __forceinline__ uint32_t hmax2(uint32_t a) { return max(a & 0xFFFFu, a >> 16); }

// ----------------------------------------------------------------- memory

__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
// L2 eviction policies for loads (createpolicy + ld.global...L2::cache_hint).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_stream_hint(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
// 16-byte store of output that is not read again soon (cache-streaming: the
// line is evicted first, so it does not displace operands other CTAs reuse).
__device__ __forceinline__ void st_v4_stream(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_v2(void* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

}  // namespace fpq
