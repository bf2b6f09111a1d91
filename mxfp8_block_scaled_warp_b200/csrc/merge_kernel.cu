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
constexpr int RPT = 8;                          // rows of the block per thread
constexpr int MT = 16 * (128 / RPT);            // threads per CTA
constexpr int MERGE_MIN_BLOCKS = 2;

// One CTA per 128x128 block of W, MT threads as a (128 / RPT) x 16 grid:
// thread (ty, tx) owns rows RPT ty .. RPT ty + RPT - 1 and columns 8 tx ..
// 8 tx + 7 of the block, so each rank step j costs it RPT / 4 + 2 16-byte
// shared loads (B column j of its rows, A row j of its columns) for 8 RPT
// fused multiply-adds; few rows per thread keep many warps resident.  The delta is
// accumulated in fp32 with j ascending from zero, exactly as the definition
// states, then merged into W and rounded to bf16; the block's amax, scale and
// E4M3 codes follow, and optionally the fake-quantized bf16 copy.
__global__ void __launch_bounds__(MT, MERGE_MIN_BLOCKS)
lora_merge_fq_kernel(const uint16_t* __restrict__ w, const uint16_t* __restrict__ a,
                     const uint16_t* __restrict__ b, int64_t n, int64_t k, int r, float alpha_over_r,
                     uint8_t* __restrict__ wq, float* __restrict__ ws, uint16_t* __restrict__ w_fq) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    extern __shared__ __align__(16) float sm[];
    float* sBt = sm;                // [r][128]  B^T for this block row: sBt[j][i] = B[row0 + i][j]
    float* sA = sm + 128 * r;       // [r][128]  A for this block column: sA[j][c] = A[j][col0 + c]
    const int64_t bj = blockIdx.x, bi = blockIdx.y;
    const int64_t row0 = bi * 128, col0 = bj * 128;
    const int rmax = (int)min64(128, n - row0);
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;

    // this thread's RPT rows x 8 columns of W (one 16-byte load per row),
    // issued first so the HBM latency overlaps the staging and the product
    uint4 wv[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rr = RPT * ty + i;
        wv[i] = rr < rmax ? ld_stream(w + (row0 + rr) * k + col0 + 8 * tx) : make_uint4(0, 0, 0, 0);
    }
    // stage the block's B rows ([128, r] contiguous) transposed, and A's r rows
    // of 128 columns, as fp32; every 16-byte load is issued before any store
    constexpr int kMaxChunks = (128 * kMaxRank * 2 / 16 + MT - 1) / MT;   // per operand at r = 64
    const int chunks = 128 * r * 2 / 16;                               // 16-byte chunks per operand
    uint4 bc[kMaxChunks], ac[kMaxChunks];
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
        const int c = threadIdx.x + MT * i;
        if (c < chunks) {
            // B elements e .. e+7 of the block (row (e+h) / r, rank (e+h) % r);
            // only the block's first rmax * r elements exist
            const int e = 8 * c, valid = rmax * r;
            if (e + 8 <= valid) {
                bc[i] = ld_stream(b + row0 * r + e);
            } else {
                uint16_t h[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) h[t] = (e + t < valid) ? b[row0 * r + e + t] : (uint16_t)0;
                bc[i] = make_uint4(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16),
                                   h[4] | ((uint32_t)h[5] << 16), h[6] | ((uint32_t)h[7] << 16));
            }
            const int jj = c >> 4, cc = 8 * (c & 15);                  // A row jj, columns cc .. cc + 7
            ac[i] = ld_stream(a + (int64_t)jj * k + col0 + cc);
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
        const int c = threadIdx.x + MT * i;
        if (c < chunks) {
            const uint32_t bw[4] = {bc[i].x, bc[i].y, bc[i].z, bc[i].w};
            const int e = 8 * c;
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const int rr = (e + h) / r, j = (e + h) - rr * r;
                sBt[j * 128 + rr] = (h & 1) ? bf16_hi(bw[h >> 1]) : bf16_lo(bw[h >> 1]);
            }
            const uint32_t aw[4] = {ac[i].x, ac[i].y, ac[i].z, ac[i].w};
            float* dst = sA + (c >> 4) * 128 + 8 * (c & 15);
            *reinterpret_cast<float4*>(dst) = make_float4(bf16_lo(aw[0]), bf16_hi(aw[0]), bf16_lo(aw[1]), bf16_hi(aw[1]));
            *reinterpret_cast<float4*>(dst + 4) = make_float4(bf16_lo(aw[2]), bf16_hi(aw[2]), bf16_lo(aw[3]), bf16_hi(aw[3]));
        }
    }
    __syncthreads();

    float d[RPT][8];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) d[i][e] = 0.0f;
#pragma unroll 2
    for (int j = 0; j < r; ++j) {
        float bv[RPT];
#pragma unroll
        for (int i = 0; i < RPT; i += 4) {
            const float4 b4 = *reinterpret_cast<const float4*>(sBt + j * 128 + RPT * ty + i);
            bv[i] = b4.x;
            if (i + 1 < RPT) bv[i + 1] = b4.y;
            if (i + 2 < RPT) bv[i + 2] = b4.z;
            if (i + 3 < RPT) bv[i + 3] = b4.w;
        }
        const float4 a0 = *reinterpret_cast<const float4*>(sA + j * 128 + 8 * tx);
        const float4 a1 = *reinterpret_cast<const float4*>(sA + j * 128 + 8 * tx + 4);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int i = 0; i < RPT; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) d[i][e] = __fmaf_rn(bv[i], av[e], d[i][e]);
    }

    // merge, round to bf16, block amax
    uint32_t v[RPT][4];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __fmaf_rn(alpha_over_r, d[i][2 * e], bf16_lo(ww[e]));
            const float hi = __fmaf_rn(alpha_over_r, d[i][2 * e + 1], bf16_hi(ww[e]));
            v[i][e] = f32x2_to_bf16x2(lo, hi);
        }
        if (RPT * ty + i < rmax)
#pragma unroll
            for (int e = 0; e < 4; ++e) m = max2(m, abs2(v[i][e]));
    }
    m = hmax2(m);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[MT / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    uint32_t am = red[0];
#pragma unroll
    for (int i = 1; i < MT / 32; ++i) am = max(am, red[i]);
    const float sc = am == 0 ? 1.0f : __fdiv_rn(__uint_as_float(am << 16), 448.0f);
    if (threadIdx.x == 0) ws[bi * (k / 128) + bj] = sc;
    const bool fast = reciprocal_ok(sc);
    const QuotientBracket br = quotient_bracket(fast ? sc : 1.0f);

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rr = RPT * ty + i;
        if (rr < rmax) {
            uint32_t e[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                e[j] = fast ? e4m3x2_of_quotients(bf16_lo(v[i][j]), bf16_hi(v[i][j]), br)
                            : f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(v[i][j]), sc), __fdiv_rn(bf16_hi(v[i][j]), sc));
            const int64_t off = (row0 + rr) * k + col0 + 8 * tx;
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
                                        void* w_fq, int sms, cudaStream_t st) {
    (void)sms;
    if (r < 1 || r > kMaxRank) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * 2 * 128 * (size_t)r;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(lora_merge_fq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)(k / 128), (unsigned)((n + 127) / 128));
    lora_merge_fq_kernel<<<grid, MT, smem, st>>>((const uint16_t*)w, (const uint16_t*)a, (const uint16_t*)b,
                                                  n, k, r, alpha_over_r, (uint8_t*)wq, ws, (uint16_t*)w_fq);
    return cudaGetLastError();
}

}  // namespace fpq
