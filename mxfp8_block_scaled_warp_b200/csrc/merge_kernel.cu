// merge_kernel.cu -- the weight side of the QAT forward in one pass over W:
// LoRA delta (rank-r outer-product sum in fp32), merge into the bf16 base
// weight, 128x128 block amax, E4M3 quantization and the optional
// fake-quantized bf16 copy.  One CTA per 128x128 block of W; the block's r
// rows of A and 128 rows of B are staged in shared memory as fp32.
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace fpq {

namespace {

constexpr int kMaxRank = 64;

__global__ void __launch_bounds__(256, 2)
lora_merge_fq_kernel(const uint16_t* __restrict__ w, const uint16_t* __restrict__ a,
                     const uint16_t* __restrict__ b, int64_t n, int64_t k, int r, float alpha_over_r,
                     uint8_t* __restrict__ wq, float* __restrict__ ws, uint16_t* __restrict__ w_fq) {
    extern __shared__ float sm[];
    float* sB = sm;                 // [128][r]   rows of B for this block row
    float* sA = sm + 128 * r;       // [r][128]   columns of A for this block column
    const int64_t bj = blockIdx.x, bi = blockIdx.y;
    const int64_t row0 = bi * 128, col0 = bj * 128;
    const int rmax = (int)min64(128, n - row0);

    // this thread's 8 chunks of W, loaded before the shared-memory staging so
    // the HBM latency overlaps it
    uint4 wv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + 256 * i, rr = c >> 4, c8 = (c & 15) * 8;
        wv[i] = rr < rmax ? ld_stream(w + (row0 + rr) * k + col0 + c8) : make_uint4(0, 0, 0, 0);
    }

    for (int i = threadIdx.x; i < 128 * r; i += 256) {
        int rr = i / r, j = i - rr * r;
        sB[i] = rr < rmax ? __uint_as_float((uint32_t)b[(row0 + rr) * r + j] << 16) : 0.0f;
        int jj = i >> 7, cc = i & 127;
        sA[i] = __uint_as_float((uint32_t)a[(int64_t)jj * k + col0 + cc] << 16);
    }
    __syncthreads();

    // merged bf16 weight of this thread's 8 chunks of 8 elements
    uint32_t v[8][4];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + 256 * i, rr = c >> 4, c8 = (c & 15) * 8;
        if (rr < rmax) {
            float d[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) d[e] = 0.0f;
#pragma unroll 4
            for (int j = 0; j < r; ++j) {
                const float bj_ = sB[rr * r + j];
                const float4 a0 = *reinterpret_cast<const float4*>(sA + j * 128 + c8);
                const float4 a1 = *reinterpret_cast<const float4*>(sA + j * 128 + c8 + 4);
                d[0] = __fmaf_rn(bj_, a0.x, d[0]); d[1] = __fmaf_rn(bj_, a0.y, d[1]);
                d[2] = __fmaf_rn(bj_, a0.z, d[2]); d[3] = __fmaf_rn(bj_, a0.w, d[3]);
                d[4] = __fmaf_rn(bj_, a1.x, d[4]); d[5] = __fmaf_rn(bj_, a1.y, d[5]);
                d[6] = __fmaf_rn(bj_, a1.z, d[6]); d[7] = __fmaf_rn(bj_, a1.w, d[7]);
            }
            const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float lo = __fmaf_rn(alpha_over_r, d[2 * e], bf16_lo(ww[e]));
                float hi = __fmaf_rn(alpha_over_r, d[2 * e + 1], bf16_hi(ww[e]));
                v[i][e] = f32x2_to_bf16x2(lo, hi);
                m = max2(m, abs2(v[i][e]));
            }
        }
    }

    // 128x128 block amax -> fp32 scale
    m = hmax2(m);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[8];
    __shared__ float sc_sh;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t am = red[0];
        for (int i = 1; i < 8; ++i) am = max(am, red[i]);
        const float sc = am == 0 ? 1.0f : __fdiv_rn(__uint_as_float(am << 16), 448.0f);
        sc_sh = sc;
        ws[bi * (k / 128) + bj] = sc;
    }
    __syncthreads();
    const float sc = sc_sh;
    const bool fast = reciprocal_ok(sc);
    const float rc = fast ? __frcp_rn(sc) : 0.0f;

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + 256 * i, rr = c >> 4, c8 = (c & 15) * 8;
        if (rr < rmax) {
            uint32_t e[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                e[j] = fast ? e4m3x2_of_quotients(bf16_lo(v[i][j]), bf16_hi(v[i][j]), sc, rc)
                            : f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(v[i][j]), sc), __fdiv_rn(bf16_hi(v[i][j]), sc));
            const int64_t off = (row0 + rr) * k + col0 + c8;
            st_v2(wq + off, make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16)));
            if (w_fq) {
                uint32_t h[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = e4m3x2_to_f32x2(e[j]);
                    h[j] = f32x2_to_bf16x2(f.x * sc, f.y * sc);
                }
                st_v4(w_fq + off, make_uint4(h[0], h[1], h[2], h[3]));
            }
        }
    }
}

}  // namespace

cudaError_t launch_lora_merge_fakequant(const void* w, const void* a, const void* b, int64_t n,
                                        int64_t k, int r, float alpha_over_r, void* wq, float* ws,
                                        void* w_fq, cudaStream_t st) {
    if (r < 1 || r > kMaxRank) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * 2 * 128 * (size_t)r;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(lora_merge_fq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)(k / 128), (unsigned)((n + 127) / 128));
    lora_merge_fq_kernel<<<grid, 256, smem, st>>>((const uint16_t*)w, (const uint16_t*)a, (const uint16_t*)b,
                                                  n, k, r, alpha_over_r, (uint8_t*)wq, ws, (uint16_t*)w_fq);
    return cudaGetLastError();
}

}  // namespace fpq
