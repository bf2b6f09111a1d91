// gemm_bf16.cu -- bf16 GEMM on the 5th-generation tensor cores for the
// backward of the QAT step: C = alpha * (P * Q^T), P [M, K] and Q [N, K]
// bf16, K-major, fp32 accumulation in TMEM, bf16 output (round to nearest
// even).  With the straight-through estimator the fake-quantizers pass
// gradients unchanged, so the backward of y = fq(x) fq(W_eff)^T is plain
// bf16 products of the gradient with the fake-quantized operands
// ("DeepSeek R1 and V3 get quantization-aware fine-tuning on Fireworks",
// Synopsis: the LoRA adapters are trained through the quantized forward).
//
// One 128 x 256 output tile per CTA; the K loop runs over 64-wide K tiles
// through a 4-stage TMA ring; four tcgen05.mma kind::f16 (bf16 x bf16 ->
// fp32, K = 16 each) per K tile.  Either operand may be K-major (stored
// [rows, K], a K tile = one TMA box of 128-byte rows) or MN-major (stored
// [K, rows]: its K tile = boxes of 64 rows-of-the-product x 64 K, each K row
// 128 bytes, 128-byte swizzle; the MMA reads it through an MN-major shared
// memory descriptor: 8 K rows of 128 bytes per 1 KB swizzle atom, atoms
// 1 KB apart along K (SBO), 64-element blocks 8 KB apart along M or N (LBO)),
// so the backward products need no transposed copies.
// Warp roles: warp 0 TMA producer, warp 2 TMEM allocator and MMA issuer
// (one elected thread); then all eight warps run the epilogue: TMEM lanes
// 32 (w & 3) .. + 31 and columns 128 (w >> 2) .. + 127 of the accumulator,
// times alpha, to bf16, staged in 128-byte-swizzled boxes and written by
// TMA stores (which clip rows past M and columns past N).
// Split-K mode, for products with few output tiles and a long contraction
// (the LoRA gradients): the grid is tiles x slices, each CTA runs its slice
// of the K tiles and stores its fp32 sums (without alpha) to a partial
// buffer; reduce_partials_kernel then adds the slices in slice order, times
// alpha, to bf16, so results do not depend on scheduling.
// Without split-K the product runs on a persistent grid (one CTA per SM):
// TMEM holds two 256-column accumulators, so the MMA warp starts tile i + 1
// while four epilogue warps read tile i's accumulator, convert it and store
// it through a staging buffer of their own; the tile's prologue and
// epilogue leave the tensor pipe's path.  CTA c walks tiles c, c + G, ...,
// or, given a zeroed tile counter, each CTA claims its next tile from the
// counter, so that CTAs which start late (the SMs of a product running
// beside this one) take fewer tiles.
// Every wait on an mbarrier is bounded by wall time (4 s); on expiry the
// kernel records FPQ_ERR_DEVICE_TIMEOUT in the device error word and unwinds.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64;           // BK in bf16 elements (128 bytes)
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2, B_TILE = BN * BK * 2;
constexpr uint32_t TMEM_COLS = 256;
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP_BYTES = 32 * 128 * 4;        // a warp's 32 x 128 block of C (fp32 partials: 16 KB)
constexpr uint64_t kTimeoutNs = 4000000000ull;

constexpr int MN_BOX = 64 * BK * 2;                 // one MN-major box: 64 rows-of-the-product x 64 K
struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t guard[32768];      // keeps any descriptor-addressed read of the last stage inside the allocation
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full;
    uint32_t tmem_base;
};
static_assert(8 * EPI_WARP_BYTES <= STAGES * (A_TILE + B_TILE), "epilogue staging exceeds the ring");

// Persistent kernel: the ring, then the epilogue warps' staging (4 warps x
// two 4 KB boxes of 32 rows x 64 bf16 columns), which also keeps any
// descriptor-addressed read of the last stage inside the allocation.
constexpr int P_EPI_WARP0 = 4;
constexpr uint32_t P_TMEM_COLS = 2 * BN;
constexpr int P_IDS = 4;                            // tile indices in flight from the producer to the others
struct __align__(1024) PSmem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t stage[4][8192];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t id_full[P_IDS];
    uint64_t id_empty[P_IDS];
    int tile_id[P_IDS];                             // -1: no more tiles
    uint32_t tmem_base;
};

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 and 10-12 = 1), A / B MN-major (bits 15 / 16), N >> 3 at bit
// 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Shared-memory descriptor of K step kk (16 K) of an operand tile.
template <bool MN>
__device__ __forceinline__ uint64_t op_desc(uint32_t base, int kk) {
    return MN ? smem_desc(base + 2048u * (uint32_t)kk, 8192, 1024, kLayoutSw128)
              : desc_kmajor_sw128(base + 32u * (uint32_t)kk);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

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

// Split-K (partial != nullptr): CTA b takes tile b / splits and the K tiles
// [kts (b % splits), kts (b % splits + 1)) and writes its fp32 sums, without
// alpha, to partial[b % splits][M][N] (rows past M and columns past N
// skipped); reduce_partials_kernel adds the slices in order.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, int64_t M, int64_t N, int64_t K, float alpha,
                 uint32_t* err, float* __restrict__ partial, int splits, int kts) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int tile = (int)blockIdx.x / splits, split = (int)blockIdx.x - tile * splits;
    const int mt = tile / n_tiles, nt = tile - mt * n_tiles;
    const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
    const int KT_all = (int)((K + BK - 1) / BK);
    const int kt0 = partial ? split * kts : 0;
    const int KT = partial ? min(KT_all, kt0 + kts) - kt0 : KT_all;     // >= 1 by the launcher's choice

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.tmem_full, 1);
        fence_barrier_init();
    }
    if (warp == 2) {
        tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    pdl_wait();

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) break;
                mbar_arrive_expect_tx(&sm.full[s], A_TILE + B_TILE);
                const int kk = (kt0 + kt) * BK;
                if (A_MN) {
#pragma unroll
                    for (int j = 0; j < BM / 64; ++j)
                        tma_load_2d(sm.a[s] + j * MN_BOX, &tmA, &sm.full[s], (int32_t)(m0 + 64 * j), kk);
                } else {
                    tma_load_2d(sm.a[s], &tmA, &sm.full[s], kk, (int32_t)m0);
                }
                if (B_MN) {
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        tma_load_2d(sm.b[s] + j * MN_BOX, &tmB, &sm.full[s], (int32_t)(n0 + 64 * j), kk);
                } else {
                    tma_load_2d(sm.b[s], &tmB, &sm.full[s], kk, (int32_t)n0);
                }
            }
        }
    } else if (warp == 2) {
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16(BM, BN, A_MN, B_MN);
            bool ok = true;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.full[s], ph, err)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_bf16(tmem, op_desc<A_MN>(a_base, k), op_desc<B_MN>(b_base, k), idesc,
                             (kt > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.empty[s]);
            }
            if (ok) mma_commit(&sm.tmem_full);
        }
    }

    __syncwarp();     // the role warps' other lanes wait here for the elected lane, without polling
    {
        const int q = warp & 3, half = warp >> 2;
        const int64_t row0 = m0 + 32 * q, col0 = n0 + 128 * half;
        const bool ok = __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.tmem_full, 0, err));
        if (ok && row0 < M && col0 < N) {
            tc_fence_after();
            uint8_t* stage = &sm.a[0][0] + warp * EPI_WARP_BYTES;
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * half + 32 * c), r[c]);
            tmem_ld_wait();
            if (partial) {
                // fp32 sums staged row-major (512-byte rows, 16-byte chunk x of
                // row l at position x ^ l), then written a row at a time
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(stage + lane * 512 + 16 * ((8 * c + j) ^ lane)) =
                            make_uint4(r[c][4 * j], r[c][4 * j + 1], r[c][4 * j + 2], r[c][4 * j + 3]);
                __syncwarp();
                float* out = partial + (int64_t)split * M * N;
                for (int rr = 0; rr < 32; ++rr) {
                    const int64_t row = row0 + rr, col = col0 + 4 * lane;
                    if (row < M && col < N)
                        st_v4(out + row * N + col, *reinterpret_cast<const uint4*>(stage + rr * 512 + 16 * (lane ^ rr)));
                }
                __syncwarp();
            } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {     // columns 32c + 8j .. + 7 = box c / 2, chunk 4 (c % 2) + j
                    uint32_t h[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        h[e] = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(r[c][8 * j + 2 * e]), alpha),
                                               __fmul_rn(__uint_as_float(r[c][8 * j + 2 * e + 1]), alpha));
                    *reinterpret_cast<uint4*>(stage + (c / 2) * 4096 + sw128_offset(lane, 4 * (c % 2) + j)) =
                        make_uint4(h[0], h[1], h[2], h[3]);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                for (int x = 0; x < 2; ++x)
                    if (col0 + x * 64 < N) tma_store_2d(&tmC, stage + x * 4096, (int32_t)(col0 + x * 64), (int32_t)row0);
                bulk_commit_group();
                bulk_wait_group_read0();     // the staging must stay valid until read
            }
            __syncwarp();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

int smem_bytes() { return (int)sizeof(Smem) + 1024; }
int p_smem_bytes() { return (int)sizeof(PSmem) + 1024; }

// Persistent product C = alpha P Q^T (no split-K): warp 0 TMA producer,
// warp 1 TMEM allocator (512 columns) and MMA issuer, warps 4-7 epilogue
// (TMEM lanes 32 (w & 3) .. + 31, all 256 columns in two halves); tile i of
// the CTA uses accumulator i & 1.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_bf16_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmC, int64_t M, int64_t N, int64_t K, float alpha,
                            uint32_t* err, int* tile_counter) {
    extern __shared__ uint8_t smem_raw[];
    PSmem& sm = *reinterpret_cast<PSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int tiles = (int)((M + BM - 1) / BM) * n_tiles;
    const int G = (int)gridDim.x;
    const int KT = (int)((K + BK - 1) / BK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 4);
        }
        for (int j = 0; j < P_IDS; ++j) {
            mbar_init(&sm.id_full[j], 1);
            mbar_init(&sm.id_empty[j], 5);           // the MMA thread and the four epilogue warps
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, P_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                // the next tile: claimed from the counter, or CTA c's i-th
                const int slot = i % P_IDS;
                if (!wait_or_timeout(&sm.id_empty[slot], ((uint32_t)(i / P_IDS) & 1u) ^ 1u, err)) break;
                int tile = tile_counter ? atomicAdd(tile_counter, 1) : (int)blockIdx.x + i * G;
                if (tile >= tiles) tile = -1;
                sm.tile_id[slot] = tile;
                mbar_arrive(&sm.id_full[slot]);
                if (tile < 0) break;
                const int mt = tile / n_tiles, nt = tile - mt * n_tiles;
                const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
                    if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sm.full[s], A_TILE + B_TILE);
                    const int kk = kt * BK;
                    if (A_MN) {
#pragma unroll
                        for (int j = 0; j < BM / 64; ++j)
                            tma_load_2d(sm.a[s] + j * MN_BOX, &tmA, &sm.full[s], (int32_t)(m0 + 64 * j), kk);
                    } else {
                        tma_load_2d(sm.a[s], &tmA, &sm.full[s], kk, (int32_t)m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_2d(sm.b[s] + j * MN_BOX, &tmB, &sm.full[s], (int32_t)(n0 + 64 * j), kk);
                    } else {
                        tma_load_2d(sm.b[s], &tmB, &sm.full[s], kk, (int32_t)n0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16(BM, BN, A_MN, B_MN);
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int slot = i % P_IDS;
                if (!wait_or_timeout(&sm.id_full[slot], (uint32_t)(i / P_IDS) & 1u, err)) break;
                const int tile = sm.tile_id[slot];
                mbar_arrive(&sm.id_empty[slot]);
                if (tile < 0) break;
                const uint32_t b = (uint32_t)i & 1u;
                if (!wait_or_timeout(&sm.acc_empty[b], (((uint32_t)i >> 1) & 1u) ^ 1u, err)) break;
                tc_fence_after();
                const uint32_t acc = tmem + b * (uint32_t)BN;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
                    if (!wait_or_timeout(&sm.full[s], ph, err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16(acc, op_desc<A_MN>(a_base, k), op_desc<B_MN>(b_base, k), idesc,
                                 (kt > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                }
                if (ok) mma_commit(&sm.acc_full[b]);
            }
        }
    } else if (warp >= P_EPI_WARP0) {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;
        uint8_t* stage = sm.stage[q];
        for (int i = 0;; ++i) {
            const int slot = i % P_IDS;
            if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.id_full[slot], (uint32_t)(i / P_IDS) & 1u, err))) break;
            const int tile = sm.tile_id[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.id_empty[slot]);
            if (tile < 0) break;
            const int mt = tile / n_tiles, nt = tile - mt * n_tiles;
            const int64_t row0 = (int64_t)mt * BM + 32 * q, n0 = (int64_t)nt * BN;
            const uint32_t b = (uint32_t)i & 1u;
            if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.acc_full[b], ((uint32_t)i >> 1) & 1u, err))) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + b * (uint32_t)BN;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + (uint32_t)(128 * h + 32 * c), r[c]);
                tmem_ld_wait();
                if (h == 1) {            // the accumulator is in registers: hand it back to the MMA warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
                }
                if (lane == 0) bulk_wait_group_read0();      // the previous half's stores have read the staging
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {     // columns 32c + 8j .. + 7 = box c / 2, chunk 4 (c % 2) + j
                        uint32_t hw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            hw[e] = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(r[c][8 * j + 2 * e]), alpha),
                                                    __fmul_rn(__uint_as_float(r[c][8 * j + 2 * e + 1]), alpha));
                        *reinterpret_cast<uint4*>(stage + (c / 2) * 4096 + sw128_offset(lane, 4 * (c % 2) + j)) =
                            make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                const int64_t col0 = n0 + 128 * h;
                if (lane == 0 && row0 < M) {
                    for (int x = 0; x < 2; ++x)
                        if (col0 + x * 64 < N)
                            tma_store_2d(&tmC, stage + x * 4096, (int32_t)(col0 + x * 64), (int32_t)row0);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group_read0();
    }

    __syncwarp();     // the role warps' other lanes wait here for the elected lane, without polling
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, P_TMEM_COLS);
    }
}

// out[i] = bf16(alpha * sum_s part[s][i]), s ascending; four elements per
// thread (count is a multiple of 4).
__global__ void __launch_bounds__(256)
reduce_partials_kernel(const float4* __restrict__ part, int splits, int64_t count4, float alpha,
                       uint2* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < count4; i += (int64_t)gridDim.x * 256) {
        float4 acc = __ldcg(part + i);
        for (int s = 1; s < splits; ++s) {
            const float4 v = __ldcg(part + s * count4 + i);
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
        }
        out[i] = make_uint2(f32x2_to_bf16x2(__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha)),
                            f32x2_to_bf16x2(__fmul_rn(acc.z, alpha), __fmul_rn(acc.w, alpha)));
    }
}

template <bool A_MN, bool B_MN>
cudaError_t launch_t(const void* p, const void* q, int64_t m, int64_t n, int64_t k, float alpha, void* c,
                     uint32_t* err, float* partial, int splits, int kts, int* tile_counter, cudaStream_t st) {
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(gemm_bf16_kernel<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes());
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    CUtensorMap ta, tb, tc;
    // K-major [rows, k], box 128 or 256 rows x 64 K; MN-major [k, rows], box 64 K x 64 rows
    e = A_MN ? make_tmap_2d(&ta, p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)k, (uint64_t)m, (uint64_t)m * 2,
                            BK, 64, CU_TENSOR_MAP_SWIZZLE_128B)
             : make_tmap_2d(&ta, p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)m, (uint64_t)k, (uint64_t)k * 2,
                            BM, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = B_MN ? make_tmap_2d(&tb, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)k, (uint64_t)n, (uint64_t)n * 2,
                            BK, 64, CU_TENSOR_MAP_SWIZZLE_128B)
             : make_tmap_2d(&tb, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)n, (uint64_t)k, (uint64_t)k * 2,
                            BN, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)m, (uint64_t)n, (uint64_t)n * 2, 32, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    if (!partial) {
        static int p_sms[64] = {0};          // SM count of the device, once configured
        if (!p_sms[dev]) {
            e = cudaFuncSetAttribute(gemm_bf16_persistent_kernel<A_MN, B_MN>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, p_smem_bytes());
            if (e != cudaSuccess) return e;
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            p_sms[dev] = sms > 0 ? sms : 1;
        }
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, p_sms[dev]));
        return launch_pdl(gemm_bf16_persistent_kernel<A_MN, B_MN>, dim3((unsigned)grid), dim3(NUM_THREADS),
                          p_smem_bytes(), st, ta, tb, tc, m, n, k, alpha, err, tile_counter);
    }
    const int64_t grid = tiles * splits;
    return launch_pdl(gemm_bf16_kernel<A_MN, B_MN>, dim3((unsigned)grid), dim3(NUM_THREADS), smem_bytes(), st, ta,
                      tb, tc, m, n, k, alpha, err, partial, splits, kts);
}

}  // namespace

namespace {
cudaError_t launch_any(const void* p, bool p_mn, const void* q, bool q_mn, int64_t m, int64_t n, int64_t k,
                       float alpha, void* c, uint32_t* err, float* partial, int splits, int kts, int* counter,
                       cudaStream_t st) {
    if (p_mn) return q_mn ? launch_t<true, true>(p, q, m, n, k, alpha, c, err, partial, splits, kts, counter, st)
                          : launch_t<true, false>(p, q, m, n, k, alpha, c, err, partial, splits, kts, counter, st);
    return q_mn ? launch_t<false, true>(p, q, m, n, k, alpha, c, err, partial, splits, kts, counter, st)
                : launch_t<false, false>(p, q, m, n, k, alpha, c, err, partial, splits, kts, counter, st);
}
}  // namespace

cudaError_t launch_gemm_bf16(const void* p, bool p_mn, const void* q, bool q_mn, int64_t m, int64_t n, int64_t k,
                             float alpha, void* c, uint32_t* err, cudaStream_t st, int* tile_counter) {
    return launch_any(p, p_mn, q, q_mn, m, n, k, alpha, c, err, nullptr, 1, 0, tile_counter, st);
}

int bf16_split_bound(int64_t m, int64_t n, int64_t k) {
    const int64_t tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int64_t kt = (k + BK - 1) / BK;
    // at most kSplitSms / tiles slices (kSplitSms is above any SM count), at
    // most kMaxSplits, at least two K tiles each
    return (int)std::max<int64_t>(1, std::min<int64_t>(kSplitSms / tiles, std::min<int64_t>(kMaxSplits, kt / 2)));
}

int bf16_split_count(int64_t m, int64_t n, int64_t k, int sms) {
    const int64_t tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int64_t splits = (int64_t)std::min(sms, kSplitSms) / tiles;     // one wave (one CTA per SM)
    return (int)std::max<int64_t>(1, std::min<int64_t>(splits, bf16_split_bound(m, n, k)));
}

cudaError_t launch_gemm_bf16_splitk(const void* p, bool p_mn, const void* q, bool q_mn, int64_t m, int64_t n,
                                    int64_t k, float alpha, void* c, float* partial, int splits, uint32_t* err,
                                    cudaStream_t st) {
    const int64_t kt = (k + BK - 1) / BK;
    const int kts = (int)((kt + splits - 1) / splits);
    splits = (int)((kt + kts - 1) / kts);                             // every slice non-empty
    cudaError_t e = launch_any(p, p_mn, q, q_mn, m, n, k, alpha, c, err, partial, splits, kts, nullptr, st);
    if (e != cudaSuccess) return e;
    const int64_t count4 = m * n / 4;
    const int grid = (int)std::min<int64_t>((count4 + 255) / 256, 1184);
    return launch_pdl(reduce_partials_kernel, dim3((unsigned)grid), dim3(256), 0, st, (const float4*)partial, splits,
                      count4, alpha, (uint2*)c);
}

}  // namespace fpq
