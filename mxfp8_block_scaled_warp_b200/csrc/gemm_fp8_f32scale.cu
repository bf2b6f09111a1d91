// gemm_fp8_f32scale.cu -- FP8 GEMM with fine-grained fp32 scales (1x128
// tiles of A, 128x128 blocks of B): C[m,n] = sum_kb sA[m,kb] * sB[n/128,kb] *
// (sum_{k in kb} qA[m,k] qB[n,k]).
//
// The tensor core produces each 128-wide K block's partial sum
// (tcgen05.mma kind::f8f6f4, 4 x K=32, fresh accumulator) into one of NBUF
// rotating TMEM buffers; the epilogue warps read it back (tcgen05.ld),
// multiply by the product of the two block scales and accumulate in fp32
// registers -- the promotion of FP8 partial products to higher precision
// before the final accumulation.  The MMA runs up to NBUF K blocks ahead of
// the promotion.
//
// Per CTA one 128 x 256 output tile (the wider N halves the shared-memory
// operand bytes per FLOP against a 128 x 128 tile).  Warp roles: warp 0 TMA
// producer, warp 1 TMEM allocator + MMA issuer, warps 2-9 promotion and
// epilogue (warp w owns TMEM lane quadrant w % 4 and the 128-column half
// (w - 2) / 4 of the tile, i.e. one 128-wide block of B and its scale).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int STAGES = 4;
constexpr int NBUF = 2;
constexpr int A_TILE = BM * BK, B_TILE = BN * BK;
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int EPI_COLS = 128;               // columns per promotion warp
constexpr int CHUNK = 16;                   // columns per tcgen05.ld
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[NBUF];
    uint64_t acc_empty[NBUF];
    uint32_t tmem_base;
};

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ bool wait_or_timeout(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kTimeoutNs) {
            raise_device_error(err, FPQ_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

// 10 warps: two SM sub-partitions hold three warps each, so a thread gets at
// most 168 registers (16 K registers per sub-partition); a promotion thread
// keeps 128 fp32 accumulators plus one 16-column TMEM chunk.
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_fp8_f32scale_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const float* __restrict__ sA, const float* __restrict__ sB, int64_t M, int64_t N,
                         int64_t K, void* __restrict__ C, int c_f32, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int mt = blockIdx.x / n_tiles, nt = blockIdx.x - mt * n_tiles;
    const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
    const int KT = (int)(K / BK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], NUM_EPI_WARPS);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) break;
                mbar_arrive_expect_tx(&sm.full[s], A_TILE + B_TILE);
                tma_load_2d(sm.a[s], &tmA, &sm.full[s], kt * BK, (int32_t)m0);
                tma_load_2d(sm.b[s], &tmB, &sm.full[s], kt * BK, (int32_t)n0);
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = idesc_f8f6f4(BM, BN);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                const int b = kt % NBUF;
                const uint32_t pb = (uint32_t)(kt / NBUF) & 1u;
                if (!wait_or_timeout(&sm.full[s], ph, err)) break;
                if (!wait_or_timeout(&sm.acc_empty[b], pb ^ 1u, err)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
                const uint32_t d = tmem + (uint32_t)(b * BN);
#pragma unroll
                for (int k = 0; k < BK / 32; ++k)
                    mma_f8f6f4(d, desc_kmajor_sw128(a_base + 32 * k), desc_kmajor_sw128(b_base + 32 * k), idesc,
                               k > 0 ? 1u : 0u);
                mma_commit(&sm.empty[s]);
                mma_commit(&sm.acc_full[b]);
            }
        }
    } else {
        const int ew = warp - 2;
        const int q = warp & 3, half = ew >> 2;
        const int64_t row = m0 + 32 * q + lane;
        const bool row_ok = row < M;
        const int64_t kts = K / 128;
        const int64_t nb = n0 / 128 + half;                 // this warp's 128-wide block of B
        const bool half_ok = nb * 128 < N;
        const float* sa_row = sA + (row_ok ? row : 0) * kts;
        const float* sb_row = sB + (half_ok ? nb : 0) * kts;
        uint64_t acc[EPI_COLS / 2];          // pairs of fp32 accumulators (packed f32x2 FMAs)
#pragma unroll
        for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = 0ull;
        float sa_next = row_ok ? __ldg(sa_row) : 0.0f;
        float sb_next = __ldg(sb_row);
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
            const float sc = sa_next * sb_next;
            const uint64_t sc2 = pack_f32x2(sc, sc);
            if (kt + 1 < KT) {
                sa_next = row_ok ? __ldg(sa_row + kt + 1) : 0.0f;
                sb_next = __ldg(sb_row + kt + 1);
            }
            const int b = kt % NBUF;
            const uint32_t pb = (uint32_t)(kt / NBUF) & 1u;
            if (!wait_or_timeout(&sm.acc_full[b], pb, err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t t = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN + EPI_COLS * half);
#pragma unroll
            for (int c = 0; c < EPI_COLS / CHUNK; ++c) {
                uint32_t p[CHUNK];
                tmem_ld_32x32b_x16(t + (uint32_t)(CHUNK * c), p);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < CHUNK / 2; ++j)
                    acc[CHUNK / 2 * c + j] = fma_f32x2(pack_u32x2(p[2 * j], p[2 * j + 1]), sc2, acc[CHUNK / 2 * c + j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
        }
        const int64_t col0 = n0 + EPI_COLS * half;
        if (ok && row_ok && col0 < N) {
            if (c_f32) {
                float* out = reinterpret_cast<float*>(C) + row * N + col0;
#pragma unroll
                for (int v = 0; v < EPI_COLS / 4; ++v)
                    if (col0 + 4 * v < N)
                        st_v4(out + 4 * v, make_uint4((uint32_t)acc[2 * v], (uint32_t)(acc[2 * v] >> 32),
                                                      (uint32_t)acc[2 * v + 1], (uint32_t)(acc[2 * v + 1] >> 32)));
            } else {
                uint16_t* out = reinterpret_cast<uint16_t*>(C) + row * N + col0;
#pragma unroll
                for (int v = 0; v < EPI_COLS / 8; ++v) {
                    uint32_t h[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        h[j] = f32x2_to_bf16x2(__uint_as_float((uint32_t)acc[4 * v + j]),
                                               __uint_as_float((uint32_t)(acc[4 * v + j] >> 32)));
                    if (col0 + 8 * v < N) st_v4(out + 8 * v, make_uint4(h[0], h[1], h[2], h[3]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

int smem_bytes() { return (int)sizeof(Smem) + 1024; }

}  // namespace

cudaError_t launch_gemm_fp8_f32scale(const void* aq, const float* as, const void* bq, const float* bs, int64_t m,
                                     int64_t n, int64_t k, void* c, int c_f32, uint32_t* err, int sms,
                                     cudaStream_t st) {
    (void)sms;
    CUtensorMap ta, tb;
    cudaError_t e = make_tmap_u8_2d(&ta, aq, (uint64_t)m, (uint64_t)k, (uint64_t)k, BM, BK);
    if (e != cudaSuccess) return e;
    e = make_tmap_u8_2d(&tb, bq, (uint64_t)n, (uint64_t)k, (uint64_t)k, BN, BK);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_fp8_f32scale_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
    if (e != cudaSuccess) return e;
    const int64_t grid = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    gemm_fp8_f32scale_kernel<<<(unsigned)grid, NUM_THREADS, smem_bytes(), st>>>(ta, tb, as, bs, m, n, k, c, c_f32,
                                                                                err);
    return cudaGetLastError();
}

}  // namespace fpq
