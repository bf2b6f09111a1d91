// gemm_fp8_f32scale.cu -- FP8 GEMM with fine-grained fp32 scales (1x128
// tiles of A, 128x128 blocks of B): C[m,n] = sum_kb sA[m,kb] * sB[n/128,kb] *
// (sum_{k in kb} qA[m,k] qB[n,k]).
//
// The tensor core produces each 128-wide K block's partial sum
// (tcgen05.mma kind::f8f6f4, K=32 steps, fresh accumulator) in TMEM; the
// promotion warps read it back (tcgen05.ld), multiply by the product of the
// two block scales and accumulate in fp32 registers -- the promotion of FP8
// partial products to higher precision before the final accumulation.
//
// Per CTA one 128 x 256 output tile, MMAs of N = 256 (N = 128 MMAs do not
// keep the tensor pipe full); TMEM holds NBUF = 2 accumulator buffers of 256
// columns.  The MMA for K block kt + 2 waits until the promotion warps have
// read K block kt back.  Every mbarrier poll costs a shared-memory round
// trip, so the MMA thread polls its two barriers (stage full, buffer empty)
// back to back and only falls into the blocking wait when one is pending.
//
// Warp roles (12 warps = 3 warpgroups):
//   warp 0      TMA producer (A and B K blocks, 4-stage ring)
//   warp 1      TMEM allocator + MMA issuer (one elected thread)
//   warp 2      scale stager: reads the fp32 block scales a few K blocks
//               ahead and writes, per K block, the product
//               sA[row, kb] * sB[half, kb] of every promotion thread into a
//               shared slot tied to the TMEM buffer, so promotion never waits
//               on a global load; a buffer is full when the MMA commit and
//               the stager have both arrived on it
//   warp 3      idle
//   warps 4-11  promotion and epilogue: warp w owns TMEM lane quadrant w % 4
//               and column half (w - 4) / 4
// Warpgroup 0 gives registers to warpgroups 1-2 (setmaxnreg) so that a
// promotion thread can hold its 128 fp32 accumulators without spilling.
//
// Epilogue: once every MMA has completed, the operand ring is free; each
// promotion warp converts its 32 x 128 block of C, writes it into the ring
// in the 128-byte-swizzled box layout and issues TMA stores (rows or columns
// past the end of C are not written by the TMA unit).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 128, HN = 128;   // HN: width of one block of B
constexpr int STAGES = 4;
constexpr int NBUF = 2;
constexpr int A_TILE = BM * BK, B_TILE = BN * BK;
constexpr uint32_t TMEM_COLS = 512;
constexpr int NUM_EPI_WARPS = 8;
constexpr int WARPS_PER_HALF = NUM_EPI_WARPS / 2;
constexpr int SCALE_WARP = 2;
constexpr int FIRST_EPI_WARP = 4;
constexpr int NUM_THREADS = 32 * (FIRST_EPI_WARP + NUM_EPI_WARPS);
// Register split: launched with LAUNCH_REGS per thread (384 threads -> a
// 64512-register pool); warpgroup 0 shrinks to CTRL_REGS, warpgroups 1-2
// grow to EPI_REGS: 128 * 56 + 256 * 224 = 384 * 168.  Per SM sub-partition
// (one warp of each warpgroup): 32 * (56 + 2 * 224) = 16128 <= 16384.
constexpr int LAUNCH_REGS = 168, CTRL_REGS = 56, EPI_REGS = 224;
static_assert(128 * CTRL_REGS + 256 * EPI_REGS <= NUM_THREADS * LAUNCH_REGS, "register split exceeds the pool");
static_assert(32 * (CTRL_REGS + 2 * EPI_REGS) <= 16384, "register split exceeds a sub-partition");
constexpr int SCALE_AHEAD = 4;              // K blocks of scales the stager holds in flight
constexpr int EPI_COLS = 128;               // columns per promotion warp
constexpr int CHUNK = 16;                   // columns per tcgen05.ld
constexpr int EPI_WARP_BYTES = 32 * EPI_COLS * 4;   // staging per warp (fp32 worst case)
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    float sc[NBUF][32 * NUM_EPI_WARPS];     // per promotion thread: sA[row, kb] * sB[half, kb]
    uint64_t acc_full[NBUF];
    uint64_t acc_empty[NBUF];
    uint32_t tmem_base;
};
static_assert(NUM_EPI_WARPS * EPI_WARP_BYTES <= STAGES * (A_TILE + B_TILE), "epilogue staging exceeds the ring");

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

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_fp8_f32scale_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmC, const float* __restrict__ sA,
                         const float* __restrict__ sB, int64_t M, int64_t N, int64_t K, int c_f32, uint32_t* err) {
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
            mbar_init(&sm.acc_full[b], 2);
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
    // Everything above touched only shared memory and TMEM; global inputs
    // and the output are accessed after the preceding grids complete.
    pdl_wait();

    if (warp == 0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CTRL_REGS));
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
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
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CTRL_REGS));
        if (elect_one()) {
            const uint32_t idesc = idesc_f8f6f4(BM, BN);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                const int b = kt % NBUF;
                const uint32_t pb = (uint32_t)(kt / NBUF) & 1u;
                const bool f = mbar_test_wait(&sm.full[s], ph);
                const bool e = mbar_test_wait(&sm.acc_empty[b], pb ^ 1u);
                if (!f && !wait_or_timeout(&sm.full[s], ph, err)) break;
                if (!e && !wait_or_timeout(&sm.acc_empty[b], pb ^ 1u, err)) break;
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
    } else if (warp == SCALE_WARP) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CTRL_REGS));
        // Lane l serves promotion thread p = 32 e + l of every promotion
        // warp e = w - 4: row m0 + 32 (e % 4) + l, column half e / 4.
        const int64_t kts = K / 128;
        const float* pa[4];
        const float* pb2[2];
        bool a_ok[4], b_ok[2];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t row = m0 + 32 * q + lane;
            a_ok[q] = row < M;
            pa[q] = sA + (a_ok[q] ? row : 0) * kts;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t nb = n0 / 128 + h;
            b_ok[h] = nb * 128 < N;
            pb2[h] = sB + (b_ok[h] ? nb : 0) * kts;
        }
        float sa[SCALE_AHEAD][4], sb[SCALE_AHEAD][2];
#pragma unroll
        for (int j = 0; j < SCALE_AHEAD; ++j) {
#pragma unroll
            for (int q = 0; q < 4; ++q) sa[j][q] = (j < KT && a_ok[q]) ? __ldg(pa[q] + j) : 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) sb[j][h] = (j < KT && b_ok[h]) ? __ldg(pb2[h] + j) : 0.0f;
        }
        bool alive = true;
        for (int kt0 = 0; kt0 < KT && alive; kt0 += SCALE_AHEAD) {
#pragma unroll
            for (int j = 0; j < SCALE_AHEAD; ++j) {
                const int kt = kt0 + j;
                if (alive && kt < KT) {
                    const int b = kt % NBUF;
                    const uint32_t pb = (uint32_t)(kt / NBUF) & 1u;
                    if (wait_or_timeout(&sm.acc_empty[b], pb ^ 1u, err)) {
#pragma unroll
                        for (int e = 0; e < NUM_EPI_WARPS; ++e)
                            sm.sc[b][32 * e + lane] = sa[j][e & 3] * sb[j][e / WARPS_PER_HALF];
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.acc_full[b]);
                    } else {
                        alive = false;
                    }
                    const int kn = kt + SCALE_AHEAD;
#pragma unroll
                    for (int q = 0; q < 4; ++q) sa[j][q] = (kn < KT && a_ok[q]) ? __ldg(pa[q] + kn) : 0.0f;
#pragma unroll
                    for (int h = 0; h < 2; ++h) sb[j][h] = (kn < KT && b_ok[h]) ? __ldg(pb2[h] + kn) : 0.0f;
                }
            }
        }
    } else if (warp < FIRST_EPI_WARP) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CTRL_REGS));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(EPI_REGS));
        const int ew = warp - FIRST_EPI_WARP;
        const int q = warp & 3, half = ew / WARPS_PER_HALF;
        uint64_t acc[EPI_COLS / 2];          // pairs of fp32 accumulators (packed f32x2 FMAs)
#pragma unroll
        for (int j = 0; j < EPI_COLS / 2; ++j) acc[j] = 0ull;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
            const int b = kt % NBUF;
            const uint32_t pb = (uint32_t)(kt / NBUF) & 1u;
            // all lanes leave together (the TMEM loads below are warp-collective)
            if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.acc_full[b], pb, err))) { ok = false; break; }
            tc_fence_after();
            const float sc = sm.sc[b][32 * ew + lane];
            const uint64_t sc2 = pack_f32x2(sc, sc);
            const uint32_t t = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN + HN * half);
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
        // The last acc_full wait above saw the last MMA complete, so the
        // operand ring is free for the epilogue staging.
        const int64_t row0 = m0 + 32 * q, col0 = n0 + HN * half;
        if (ok && row0 < M && col0 < N) {
            uint8_t* stage = &sm.a[0][0] + ew * EPI_WARP_BYTES;
            if (c_f32) {
#pragma unroll
                for (int c = 0; c < EPI_COLS / 4; ++c)     // 16-byte chunk c = fp32 columns 4c .. 4c + 3
                    *reinterpret_cast<uint4*>(stage + (c / 8) * 4096 + sw128_offset(lane, c % 8)) =
                        make_uint4((uint32_t)acc[2 * c], (uint32_t)(acc[2 * c] >> 32), (uint32_t)acc[2 * c + 1],
                                   (uint32_t)(acc[2 * c + 1] >> 32));
            } else {
#pragma unroll
                for (int c = 0; c < EPI_COLS / 8; ++c) {   // 16-byte chunk c = bf16 columns 8c .. 8c + 7
                    uint32_t h[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        h[j] = f32x2_to_bf16x2(__uint_as_float((uint32_t)acc[4 * c + j]),
                                               __uint_as_float((uint32_t)(acc[4 * c + j] >> 32)));
                    *reinterpret_cast<uint4*>(stage + (c / 8) * 4096 + sw128_offset(lane, c % 8)) =
                        make_uint4(h[0], h[1], h[2], h[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int boxes = c_f32 ? 4 : 2, box_cols = c_f32 ? 32 : 64;
                for (int x = 0; x < boxes; ++x)
                    if (col0 + x * box_cols < N)
                        tma_store_2d(&tmC, stage + x * 4096, (int32_t)(col0 + x * box_cols), (int32_t)row0);
                bulk_commit_group();
                bulk_wait_group_read0();     // the staging must stay valid until read
            }
            __syncwarp();
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
    // Per-device one-time setup: the shared-memory opt-in, and a check that
    // the kernel was built with exactly LAUNCH_REGS registers per thread (the
    // register split is sized for that pool; with any other count
    // setmaxnreg.inc could wait for registers that do not exist).
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(gemm_fp8_f32scale_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) return e;
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, gemm_fp8_f32scale_kernel);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != LAUNCH_REGS) return cudaErrorNotSupported;
        configured[dev] = 1;
    }
    CUtensorMap ta, tb, tc;
    e = make_tmap_u8_2d(&ta, aq, (uint64_t)m, (uint64_t)k, (uint64_t)k, BM, BK);
    if (e != cudaSuccess) return e;
    e = make_tmap_u8_2d(&tb, bq, (uint64_t)n, (uint64_t)k, (uint64_t)k, BN, BK);
    if (e != cudaSuccess) return e;
    if (c_f32)
        e = make_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)m, (uint64_t)n, (uint64_t)n * 4, 32, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    else
        e = make_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)m, (uint64_t)n, (uint64_t)n * 2, 32, 64,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const int64_t grid = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    return launch_pdl(gemm_fp8_f32scale_kernel, dim3((unsigned)grid), dim3(NUM_THREADS), smem_bytes(), st, ta, tb, tc,
                      as, bs, m, n, k, c_f32, err);
}

}  // namespace fpq
