// quant_unit.cuh -- the 16-element work unit of the streaming quantizers
// and the MXFP8 block encoder, shared by the block quantizer and the fused
// MoE dispatch.  A unit is 16 consecutive bf16 elements of a row (32 bytes)
// held by one lane as eight 32-bit words; an MXFP8 block (1x32) is the unit
// pair (2i, 2i + 1), held by adjacent lanes.
#pragma once

#include "common.cuh"

namespace fpq {

struct Unit { uint32_t w[8]; };

__device__ __forceinline__ Unit load_unit(const uint4* x, int64_t u) {
    uint4 a = ld_stream(x + 2 * u), b = ld_stream(x + 2 * u + 1);
    return Unit{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}

// Largest magnitude pattern of the unit's 16 values (15 bits; a NaN
// anywhere gives a NaN pattern, which every caller treats as NaN whatever
// its payload).
__device__ __forceinline__ uint32_t unit_absmax(const Unit& v) {
    uint32_t m = absmax_bf16x2(v.w[0], v.w[1]);
#pragma unroll
    for (int i = 2; i < 8; ++i) m = absmax_bf16x2(m, v.w[i]);
    return hmax2(abs2(m));
}

// Reduce a magnitude pattern over `width` adjacent lanes (power of two).
template <int width>
__device__ __forceinline__ uint32_t group_max(uint32_t m) {
#pragma unroll
    for (int o = 1; o < width; o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    return m;
}

// MXFP8 block exponent from the block's largest magnitude pattern a (15 bits
// of a bf16): e = ceil(log2(amax/448)) clamped to [-127, 127], computed from
// the exponent and mantissa fields.  With amax = mu * 2^E, mu in [1, 2):
// amax/448 = (mu/1.75) * 2^(E-8), so e = E - 8 when mu <= 1.75 and E - 7
// when mu > 1.75 (mantissa field > 0x60).  Zero and subnormal amax clamp to
// -127; infinity gives 127; NaN gives code 0xFF (returned as 128).
__device__ __forceinline__ int mx_exponent(uint32_t a) {
    if (a > 0x7F80u) return 128;
    if (a == 0x7F80u) return 127;
    uint32_t E = a >> 7;
    if (E == 0) return -127;
    int e = (int)E - 127 - 8 + ((a & 0x7Fu) > 0x60u ? 1 : 0);
    return max(-127, min(127, e));
}

// 2^-e as fp32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2_neg(int e) {
    return (e == 127) ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
}

__device__ __forceinline__ uint4 scale_to_e4m3(const Unit& v, float mul) {
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = f32x2_to_e4m3x2(bf16_lo(v.w[i]) * mul, bf16_hi(v.w[i]) * mul);
    return make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16), c[6] | (c[7] << 16));
}

// Strided operands.  Flat unit u of `batch` [rows, cols] matrices (u =
// (b rows + r) cols / 16 + c) lives at unit b bs + r ld + c of an operand
// with row stride ld and batch stride bs, both counted in units of 16
// elements (whatever the element width).  Dense operands (S = false) use u
// itself.
struct UnitStrides {
    int64_t upr, upm;          // units per row, per matrix
    int64_t in_ld, in_bs;      // the kernel's input operand
    int64_t out_ld, out_bs;    // the kernel's output operand
};

__device__ __forceinline__ int64_t unit_at(int64_t u, int64_t upr, int64_t upm, int64_t ld, int64_t bs) {
    const int64_t b = u / upm, rem = u - b * upm, r = rem / upr;
    return b * bs + r * ld + (rem - r * upr);
}

template <bool S>
__device__ __forceinline__ int64_t in_unit(const UnitStrides& m, int64_t u) {
    return S ? unit_at(u, m.upr, m.upm, m.in_ld, m.in_bs) : u;
}

template <bool S>
__device__ __forceinline__ int64_t out_unit(const UnitStrides& m, int64_t u) {
    return S ? unit_at(u, m.upr, m.upm, m.out_ld, m.out_bs) : u;
}

}  // namespace fpq
