// merge_kernel.cu -- the weight side of the QAT forward in one pass over W:
// LoRA delta (rank-r outer-product sum in fp32), merge into the bf16 base
// weight, 128x128 block amax, E4M3 quantization and the optional
// fake-quantized bf16 copy.  One CTA per 128x128 block of W; the block's r
// rows of A and 128 rows of B are staged in shared memory as fp32, and the
// rank-r delta is formed with paired fp32 fmas.
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace fpq {

namespace {

constexpr int kMaxRank = 64;
constexpr int RPT = 4;                          // rows of a block per thread
constexpr int MT = 16 * (128 / RPT);            // 128 / RPT row groups x 16 column groups of threads
constexpr int kWBytes = 128 * 128 * 2;          // the block of W in shared memory

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// One CTA per 128x128 block of W; thread (ty, tx) owns rows RPT ty .. RPT ty
// + RPT - 1 and columns 8 tx .. 8 tx + 7 of the block.  The rank is padded to R (8,
// 16, 32 or 64) with zero rows of A and columns of B: the padded terms add
// +0 to a running sum that is never -0 (it starts at +0, and a round-to-
// nearest sum is -0 only when both addends are), so they change nothing.
//
// Shared memory: W's block (bf16, copied by cp.async while the delta is
// formed), B's rows of the block as duplicated pairs {B[i][j], B[i][j]}
// ([R][128] pairs), and A's columns of the block as fp32 ([R][128], each
// row stored as two 64-column halves so that a thread's 4-column loads of
// one half are contiguous across the 16 column groups).  Per rank step j
// a thread loads RPT pairs of B and 8 values of A (RPT / 2 + 2 shared
// loads) and issues 4 RPT paired fmas, j ascending from zero as the
// definition states.
template <int R>
__global__ void __launch_bounds__(MT, 2)
lora_merge_fq_kernel(const uint16_t* __restrict__ w, const uint16_t* __restrict__ a,
                     const uint16_t* __restrict__ b, int64_t n, int64_t k, int r, float alpha_over_r,
                     uint8_t* __restrict__ wq, float* __restrict__ ws, uint16_t* __restrict__ w_fq) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* sW = reinterpret_cast<uint16_t*>(smem);                       // [128][128] bf16
    uint64_t* sB2 = reinterpret_cast<uint64_t*>(smem + kWBytes);             // [R][128] pairs
    float* sA = reinterpret_cast<float*>(smem + kWBytes + R * 128 * 8);      // [R][2][64]
    const int64_t bj = blockIdx.x, bi = blockIdx.y;
    const int64_t row0 = bi * 128, col0 = bj * 128;
    const int rmax = (int)min64(128, n - row0);
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

    // W: this thread's RPT rows x 16 bytes, into shared memory behind the delta
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rr = RPT * ty + i;
        if (rr < rmax) cp_async16(sW + rr * 128 + 8 * tx, w + (row0 + rr) * k + col0 + 8 * tx);
    }
    // A: R rows of the block's 128 columns, 16-byte loads (zero rows past r)
    constexpr int kAChunks = R * 16;
#pragma unroll
    for (int c0 = 0; c0 < kAChunks; c0 += MT) {
        const int c = c0 + tid;
        if (kAChunks % MT == 0 || c < kAChunks) {
            const int jj = c >> 4, cc = c & 15;
            const uint4 v = jj < r ? ld_stream(a + (int64_t)jj * k + col0 + 8 * cc) : make_uint4(0, 0, 0, 0);
            float* dst = sA + jj * 128 + 4 * cc;
            *reinterpret_cast<float4*>(dst) = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
            *reinterpret_cast<float4*>(dst + 64) = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
        }
    }
    // B: thread (row = tid % 128, part = tid / 128) takes ranks part * R/P
    // .. (P = MT / 128 parts); consecutive threads write consecutive pairs of
    // one rank row
    {
        constexpr int P = MT / 128;
        const int row = tid & 127, j0 = (tid >> 7) * (R / P);
        const bool row_ok = row < rmax;
        const uint16_t* brow = b + (row0 + row) * r;
#pragma unroll
        for (int jj = 0; jj < R / P; ++jj) {
            const int j = j0 + jj;
            const float f = (row_ok && j < r) ? __uint_as_float((uint32_t)brow[j] << 16) : 0.0f;
            sB2[j * 128 + row] = pack2(f, f);
        }
    }
    __syncthreads();

    uint64_t acc[RPT][4];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0;
#pragma unroll 16
    for (int j = 0; j < R; ++j) {
        const ulonglong2* bp = reinterpret_cast<const ulonglong2*>(sB2 + j * 128 + RPT * ty);
        uint64_t bb[RPT];
#pragma unroll
        for (int h = 0; h < RPT / 2; ++h) {
            const ulonglong2 bv = bp[h];
            bb[2 * h] = bv.x;
            bb[2 * h + 1] = bv.y;
        }
        const ulonglong2 a0 = *reinterpret_cast<const ulonglong2*>(sA + j * 128 + 4 * tx);
        const ulonglong2 a1 = *reinterpret_cast<const ulonglong2*>(sA + j * 128 + 64 + 4 * tx);
        const uint64_t aa[4] = {a0.x, a0.y, a1.x, a1.y};
#pragma unroll
        for (int i = 0; i < RPT; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][e] = fma2(bb[i], aa[e], acc[i][e]);
    }

    // merge, round to bf16, block amax
    cp_async_wait_all();     // this thread's own copies of W
    const uint64_t al2 = pack2(alpha_over_r, alpha_over_r);
    uint32_t v[RPT][4];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const uint4 wv = *reinterpret_cast<const uint4*>(sW + (RPT * ty + i) * 128 + 8 * tx);
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint64_t x = fma2(al2, acc[i][e], pack2(bf16_lo(ww[e]), bf16_hi(ww[e])));
            v[i][e] = f32x2_to_bf16x2(lo_of(x), hi_of(x));
        }
        if (RPT * ty + i < rmax)
#pragma unroll
            for (int e = 0; e < 4; ++e) m = max2(m, abs2(v[i][e]));
    }
    m = hmax2(m);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[MT / 32];
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    uint32_t am = red[0];
#pragma unroll
    for (int i = 1; i < MT / 32; ++i) am = max(am, red[i]);
    const float sc = am == 0 ? 1.0f : __fdiv_rn(__uint_as_float(am << 16), 448.0f);
    if (tid == 0) ws[bi * (k / 128) + bj] = sc;
    const bool fast = reciprocal_ok(sc);
    const QuotientBracket br = quotient_bracket(fast ? sc : 1.0f);
    const uint64_t lo2 = pack2(br.lo, br.lo), hi2 = pack2(br.hi, br.hi);

    // E4M3 codes of fp32(v / sc): the quotient bracketed by products with
    // the reciprocal's two neighbours; where a row's codes of the two ends
    // differ anywhere (a quotient near a rounding boundary), the row's 8
    // elements are encoded from correctly rounded divisions
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rr = RPT * ty + i;
        if (rr < rmax) {
            uint2 cw;
            if (!fast || !e4m3x8_bracketed(v[i], lo2, hi2, cw)) cw = e4m3x8_divided(v[i], sc);
            const int64_t off = (row0 + rr) * k + col0 + 8 * tx;
            st_v2(wq + off, cw);
            if (w_fq) {
                const uint32_t c[4] = {cw.x & 0xFFFFu, cw.x >> 16, cw.y & 0xFFFFu, cw.y >> 16};
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = e4m3x2_to_f32x2(c[e]);
                    h[e] = f32x2_to_bf16x2(f.x * sc, f.y * sc);
                }
                st_v4(w_fq + off, make_uint4(h[0], h[1], h[2], h[3]));
            }
        }
    }
}

template <int R>
cudaError_t launch_r(const void* w, const void* a, const void* b, int64_t n, int64_t k, int r, float alpha_over_r,
                     void* wq, float* ws, void* w_fq, cudaStream_t st) {
    const size_t smem = (size_t)kWBytes + (size_t)R * 128 * 12;
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(lora_merge_fq_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    dim3 grid((unsigned)(k / 128), (unsigned)((n + 127) / 128));
    lora_merge_fq_kernel<R><<<grid, MT, smem, st>>>((const uint16_t*)w, (const uint16_t*)a, (const uint16_t*)b, n,
                                                     k, r, alpha_over_r, (uint8_t*)wq, ws, (uint16_t*)w_fq);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_lora_merge_fakequant(const void* w, const void* a, const void* b, int64_t n,
                                        int64_t k, int r, float alpha_over_r, void* wq, float* ws,
                                        void* w_fq, int sms, cudaStream_t st) {
    (void)sms;
    if (r < 1 || r > kMaxRank) return cudaErrorInvalidValue;
    if (r <= 8) return launch_r<8>(w, a, b, n, k, r, alpha_over_r, wq, ws, w_fq, st);
    if (r <= 16) return launch_r<16>(w, a, b, n, k, r, alpha_over_r, wq, ws, w_fq, st);
    if (r <= 32) return launch_r<32>(w, a, b, n, k, r, alpha_over_r, wq, ws, w_fq, st);
    return launch_r<64>(w, a, b, n, k, r, alpha_over_r, wq, ws, w_fq, st);
}

}  // namespace fpq
