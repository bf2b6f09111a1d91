// gemm_nvfp4.cu -- block-scaled NVFP4 GEMM on the 5th-generation tensor
// cores: C = gA gB (A * B^T) with A [M, K], B [N, K] packed E2M1 codes (two
// per byte, element 2i in the low nibble), one E4M3 scale per 16 K-elements
// of every row and one fp32 tensor scale per operand ("fireworks-prequant
// 0.1.0", Formats: packed FP4 + FP8 block scales); fp32 accumulation in
// TMEM, bf16 (round-to-nearest-even) or fp32 output.
//
// Per CTA one 128 x 256 output tile; the K loop runs over 256-wide K tiles
// (128 bytes of codes per row) through a STAGES-deep shared-memory ring.
// One tcgen05.mma kind::mxf4nvf4 covers K = 64 and reads, for row m of its
// operand, the 32-bit TMEM word holding the row's four block scales of those
// 64 elements: lane m mod 32 of the scale columns, column base + m / 32.  A
// K tile therefore needs four such scale atoms for A (4 columns each) and
// four for B (8 columns each: 256 rows).
//
// Warp roles:
//   warp 0  TMA producer: A and B code tiles (128-byte swizzle, no multicast)
//   warp 2  TMEM allocator and MMA issuer (one elected thread): tcgen05.cp of
//           the scale atoms, 4 x tcgen05.mma per K tile, tcgen05.commit
//   warps 4-7 during the K loop, scale loaders: warp 4 + i serves ring stage
//           i (K tiles i, i + 4, ...), reading the row-major E4M3 scales of
//           the tile's rows one K tile ahead and writing them in the
//           shared-memory atom layout the shared->TMEM copy expects (lane l:
//           rows l, l+32, l+64, l+96), so four K tiles of scale loads are in
//           flight; afterwards, the epilogue: tcgen05.ld of the accumulator,
//           times gA gB, convert, stage in the freed operand ring, store C a
//           row at a time
// Every wait on an mbarrier is bounded by wall time (4 s); on expiry the
// kernel records FPQ_ERR_DEVICE_TIMEOUT in the device error word and unwinds.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 256;          // BK in elements (128 bytes of codes)
constexpr int BKB = BK / 2;                          // code bytes per row per K tile
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BKB, B_TILE = BN * BKB;
constexpr int MMAS_PER_TILE = BK / 64;               // K = 64 per instruction
constexpr int ATOM_BYTES = 512;                      // 128 rows x 4 scale bytes
constexpr int SFA_BYTES = MMAS_PER_TILE * ATOM_BYTES;          // 4 atoms
constexpr int SFB_BYTES = MMAS_PER_TILE * 2 * ATOM_BYTES;      // 8 atoms (256 rows)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = BN;                     // scale columns follow the accumulator
constexpr uint32_t SFA_COLS = 4 * MMAS_PER_TILE;     // per stage
constexpr uint32_t SFB_COLS = 8 * MMAS_PER_TILE;
constexpr uint32_t SF_COLS_PER_STAGE = SFA_COLS + SFB_COLS;
static_assert(SF_COL0 + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM columns");
constexpr int NUM_THREADS = 256;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t sfa[STAGES][SFA_BYTES];
    uint8_t sfb[STAGES][SFB_BYTES];
    uint64_t full[STAGES];     // operand tiles (and, with TMA scales, the scale rows) have landed
    uint64_t sfr[STAGES];      // scale atoms written
    uint64_t empty[STAGES];
    uint64_t tmem_full;
    uint32_t tmem_base;
};
constexpr int EPI_WARP_BYTES = 32 * 128 * 4;       // a warp's 32 x 128 block of C, fp32
static_assert(8 * EPI_WARP_BYTES <= STAGES * (A_TILE + B_TILE), "epilogue staging exceeds the ring");

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

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// The 16 scale bytes of row `row` for K tile kt (K elements [256 kt, 256 kt
// + 256)); rows outside [0, nrows) and bytes past the row's end read as 0.
__device__ __forceinline__ uint4 load_sf_tile(const uint8_t* sf, int64_t row, int64_t nrows, int64_t pitch, int kt,
                                              bool vec16) {
    if (row < 0 || row >= nrows) return make_uint4(0, 0, 0, 0);
    const uint8_t* p = sf + row * pitch + (int64_t)kt * 16;
    if (vec16) return *reinterpret_cast<const uint4*>(p);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = ((int64_t)kt * 16 + 4 * j + 4 <= pitch) ? *reinterpret_cast<const uint32_t*>(p + 4 * j) : 0u;
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Writes the scale atoms of one ring stage from 16-byte row chunks: ca[i] =
// the K tile's scales of A row lane + 32 i, cb[i] those of B row lane + 32 i.
__device__ __forceinline__ void write_atoms(uint8_t* sfa_s, uint8_t* sfb_s, const uint4 (&ca)[4],
                                            const uint4 (&cb)[8], int lane) {
#pragma unroll
    for (int j = 0; j < MMAS_PER_TILE; ++j) {
        *reinterpret_cast<uint4*>(sfa_s + j * ATOM_BYTES + lane * 16) =
            make_uint4(word(ca[0], j), word(ca[1], j), word(ca[2], j), word(ca[3], j));
#pragma unroll
        for (int h = 0; h < 2; ++h)
            *reinterpret_cast<uint4*>(sfb_s + (2 * j + h) * ATOM_BYTES + lane * 16) =
                make_uint4(word(cb[4 * h], j), word(cb[4 * h + 1], j), word(cb[4 * h + 2], j),
                           word(cb[4 * h + 3], j));
    }
}

// Epilogue of one warp: its 32 accumulator rows x 128 columns (r[c] = TMEM
// columns 32c .. 32c + 31 of the warp's half, row = lane) times gab, staged in
// 128-byte-swizzled boxes of 32 rows (fp32: 32 columns, bf16: 64) and
// written by TMA stores at (col0, row0); the stores clip at M and N.
__device__ __forceinline__ void stage_and_store(uint8_t* stage, const uint32_t (&r)[4][32], float gab, int c_f32,
                                                int lane, const CUtensorMap* tmC, int64_t col0, int64_t row0,
                                                int64_t N) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __fmul_rn(__uint_as_float(r[c][e]), gab);
        if (c_f32) {     // columns 32c .. 32c + 31 = box c, chunks 0..7
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(stage + c * 4096 + sw128_offset(lane, j)) =
                    make_uint4(__float_as_uint(f[4 * j]), __float_as_uint(f[4 * j + 1]),
                               __float_as_uint(f[4 * j + 2]), __float_as_uint(f[4 * j + 3]));
        } else {         // columns 32c .. 32c + 31 = box c / 2, chunks 4 (c % 2) .. + 3
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) h[e] = f32x2_to_bf16x2(f[8 * j + 2 * e], f[8 * j + 2 * e + 1]);
                *reinterpret_cast<uint4*>(stage + (c / 2) * 4096 + sw128_offset(lane, 4 * (c % 2) + j)) =
                    make_uint4(h[0], h[1], h[2], h[3]);
            }
        }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        const int boxes = c_f32 ? 4 : 2, box_cols = c_f32 ? 32 : 64;
        for (int x = 0; x < boxes; ++x)
            if (col0 + x * box_cols < N)
                tma_store_2d(tmC, stage + x * 4096, (int32_t)(col0 + x * box_cols), (int32_t)row0);
        bulk_commit_group();
        bulk_wait_group_read0();     // the staging must stay valid until read
    }
    __syncwarp();
}

// TMA_SF: the scale rows of each K tile arrive by TMA with the operand tiles
// (dense, row r at 16 r) and the stage's loader warp rearranges them in place
// into atoms; otherwise (scale rows not 16-byte aligned) the loader warps
// read them from global memory themselves.
template <bool TMA_SF>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                  const __grid_constant__ CUtensorMap tmC,
                  const uint8_t* __restrict__ sfa, const float* __restrict__ ga, const uint8_t* __restrict__ sfb,
                  const float* __restrict__ gb, int64_t M, int64_t N, int64_t K, void* __restrict__ C, int c_f32,
                  uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int mt = blockIdx.x / n_tiles, nt = blockIdx.x - mt * n_tiles;
    const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
    const int KT = (int)((K + BK - 1) / BK);
    const int64_t sf_pitch = K / 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);     // TMA bytes
            mbar_init(&sm.sfr[s], 1);      // scale loader
            mbar_init(&sm.empty[s], 1);    // tcgen05.commit
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
    // Everything above touched only shared memory and TMEM; global inputs
    // and the output are accessed after the preceding grids complete.
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
            if (TMA_SF) {
                tma_prefetch_desc(&tmSA);
                tma_prefetch_desc(&tmSB);
            }
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) break;
                mbar_arrive_expect_tx(&sm.full[s], A_TILE + B_TILE + (TMA_SF ? SFA_BYTES + SFB_BYTES : 0));
                tma_load_2d(sm.a[s], &tmA, &sm.full[s], kt * BKB, (int32_t)m0);
                tma_load_2d(sm.b[s], &tmB, &sm.full[s], kt * BKB, (int32_t)n0);
                if (TMA_SF) {
                    tma_load_2d(sm.sfa[s], &tmSA, &sm.full[s], kt * 16, (int32_t)m0);
                    tma_load_2d(sm.sfb[s], &tmSB, &sm.full[s], kt * 16, (int32_t)n0);
                }
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t idesc = idesc_mxf4nvf4(BM, BN);
            bool ok = true;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.full[s], ph, err) || !wait_or_timeout(&sm.sfr[s], ph, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t col_a = tmem + SF_COL0 + SF_COLS_PER_STAGE * (uint32_t)s;
                const uint32_t col_b = col_a + SFA_COLS;
#pragma unroll
                for (int j = 0; j < MMAS_PER_TILE; ++j) {
                    tmem_cp_32x128b_warpx4(col_a + 4 * j,
                                           smem_desc(smem_u32(sm.sfa[s] + j * ATOM_BYTES), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4(col_b + 8 * j,
                                           smem_desc(smem_u32(sm.sfb[s] + 2 * j * ATOM_BYTES), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4(col_b + 8 * j + 4,
                                           smem_desc(smem_u32(sm.sfb[s] + (2 * j + 1) * ATOM_BYTES), 0, 128,
                                                     kLayoutNone));
                }
                const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                for (int j = 0; j < MMAS_PER_TILE; ++j)
                    mma_mxf4nvf4(tmem, desc_kmajor_sw128(a_base + 32 * j), desc_kmajor_sw128(b_base + 32 * j), idesc,
                                 col_a + 4 * j, col_b + 8 * j, (kt > 0 || j > 0) ? 1u : 0u);
                mma_commit(&sm.empty[s]);
            }
            if (ok) mma_commit(&sm.tmem_full);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------- scale loader
        // Lane l holds rows l + 32 i of A (i < 4) and of B (i < 8); atom j of a
        // K tile (the scales of MMA j) is, per lane, the j-th 32-bit word of
        // each of its rows: 16 bytes = rows l, l+32, l+64, l+96.
        if (TMA_SF) {
            const int s = warp - 4;                   // this warp's ring stage
            for (int kt = s; kt < KT; kt += STAGES) {
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.full[s], ph, err))) break;
                uint4 ca[4], cb[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) ca[i] = *reinterpret_cast<const uint4*>(sm.sfa[s] + (lane + 32 * i) * 16);
#pragma unroll
                for (int i = 0; i < 8; ++i) cb[i] = *reinterpret_cast<const uint4*>(sm.sfb[s] + (lane + 32 * i) * 16);
                __syncwarp();
                write_atoms(sm.sfa[s], sm.sfb[s], ca, cb, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sfr[s]);
            }
        } else {
            const int s = warp - 4;
            const bool vec16 = (sf_pitch % 16) == 0;
            uint4 ca[4], cb[8];
            if (s < KT) {
#pragma unroll
                for (int i = 0; i < 4; ++i) ca[i] = load_sf_tile(sfa, m0 + lane + 32 * i, M, sf_pitch, s, vec16);
#pragma unroll
                for (int i = 0; i < 8; ++i) cb[i] = load_sf_tile(sfb, n0 + lane + 32 * i, N, sf_pitch, s, vec16);
            }
            for (int kt = s; kt < KT; kt += STAGES) {
                uint4 na[4], nb[8];
                if (kt + STAGES < KT) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        na[i] = load_sf_tile(sfa, m0 + lane + 32 * i, M, sf_pitch, kt + STAGES, vec16);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        nb[i] = load_sf_tile(sfb, n0 + lane + 32 * i, N, sf_pitch, kt + STAGES, vec16);
                }
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.empty[s], ph ^ 1u, err))) break;
                write_atoms(sm.sfa[s], sm.sfb[s], ca, cb, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sfr[s]);
#pragma unroll
                for (int i = 0; i < 4; ++i) ca[i] = na[i];
#pragma unroll
                for (int i = 0; i < 8; ++i) cb[i] = nb[i];
            }
        }
    }

    // -------------------------------------------------------------- epilogue
    // All eight warps, once the last MMA has completed (the operand ring is
    // then free): warp w reads TMEM lanes 32 (w & 3) .. + 31 (rows of C) and
    // columns 128 (w >> 2) .. + 127, multiplies by gA gB, stages the 32 x 128
    // block in 128-byte-swizzled boxes and writes them with TMA stores (which
    // clip rows past M and columns past N).
    __syncwarp();     // the role warps' other lanes wait here for the elected lane, without polling
    {
        const int q = warp & 3, half = warp >> 2;
        const int64_t row0 = m0 + 32 * q, col0 = n0 + 128 * half;
        const bool ok = __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.tmem_full, 0, err));
        if (ok && row0 < M && col0 < N) {
            tc_fence_after();
            const float gab = __fmul_rn(__ldg(ga), __ldg(gb));
            uint8_t* stage = &sm.a[0][0] + warp * EPI_WARP_BYTES;
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * half + 32 * c), r[c]);
            tmem_ld_wait();
            stage_and_store(stage, r, gab, c_f32, lane, &tmC, col0, row0, N);
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

// ============================================================== CTA pair
// A cluster of two CTAs computes one 256 x 256 tile with tcgen05 cta_group::2:
// CTA r holds A rows m0 + 128 r .. + 127 and B rows (output columns)
// n0 + 128 r .. + 127 of each K tile in its own shared memory, and receives
// its 128 accumulator rows x 256 columns in its own TMEM.  Per SM a K tile
// is then 16 + 16 KB of codes instead of 16 + 32 KB.
//
// Scales come in chunks of SF_CH K tiles, SF_BUFS chunks in flight: one TMA
// box of (16 SF_CH)-byte scale rows for this CTA's 128 A rows and one for
// all 256 B rows of the tile (its accumulator rows meet every output
// column).  Per-row TMA requests are costly, so wider rows and fewer boxes
// matter.  Two loader warps per chunk, one per K tile, rearrange a landed
// chunk in place into the atoms of its K tiles, make them visible to the
// async proxy and arrive on the leader's sfr barrier; the leader's copy
// instruction (cta_group::2) moves each CTA's atoms into that CTA's TMEM.
// The leader's single thread issues all copies and MMAs and commits to the
// barriers of both CTAs.
//
// Warp roles in both CTAs: warp 0 code-tile TMA producer; warp 1 scale-chunk
// TMA producer; warp 2 TMEM allocator (and, in the leader, MMA issuer);
// warps 4-7 scale loaders (4-5 even chunks, 6-7 odd); then all eight warps
// run the epilogue.
constexpr int PSTAGES = 5;
constexpr int P_A_TILE = 128 * BKB, P_B_TILE = 128 * BKB;
constexpr int SF_CH = 2;                                   // K tiles per scale chunk
constexpr int SF_BUFS = 4;                                 // scale chunks in flight
constexpr int SFC_A_BYTES = 128 * 16 * SF_CH;              // dense: row r at r * 64
constexpr int SFC_BYTES = SFC_A_BYTES + 256 * 16 * SF_CH;  // + 256 B rows
constexpr int SF_TILE_ATOM_BYTES = SFA_BYTES + SFB_BYTES;  // a K tile's atoms (A then B)
static_assert(SF_CH * SF_TILE_ATOM_BYTES == SFC_BYTES, "in-place rearrangement");
constexpr uint32_t P_SF_COL0 = 256;
static_assert(P_SF_COL0 + PSTAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM columns (pair)");
static_assert(SF_CH == 2 && SF_BUFS % 2 == 0, "loader warps 4-5 take even chunks, 6-7 odd ones");

struct __align__(1024) PairSmem {
    uint8_t a[PSTAGES][P_A_TILE];
    uint8_t b[PSTAGES][P_B_TILE];
    uint8_t sfc[SF_BUFS][SFC_BYTES];
    uint64_t full[PSTAGES];    // leader's copy used: code tiles of both CTAs
    uint64_t empty[PSTAGES];   // both CTAs: the leader's commit after the stage's MMAs
    uint64_t sff[SF_BUFS];      // this CTA's scale chunk has landed
    uint64_t sfr[SF_BUFS];      // leader's copy used: atoms of both CTAs written
    uint64_t sf_empty[SF_BUFS]; // both CTAs: the leader's commit after a chunk's last MMAs
    uint64_t tmem_full;        // both CTAs: the leader's commit after the last MMA
    uint32_t tmem_base;
};
static_assert(8 * EPI_WARP_BYTES <= PSTAGES * (P_A_TILE + P_B_TILE), "epilogue staging exceeds the ring (pair)");


__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                       const __grid_constant__ CUtensorMap tmC, const float* __restrict__ ga,
                       const float* __restrict__ gb, int64_t M, int64_t N, int64_t K, int c_f32, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    PairSmem& sm = *reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int n_tiles = (int)((N + 255) / 256);
    const int pair = blockIdx.x >> 1;
    const int mt = pair / n_tiles, nt = pair - mt * n_tiles;
    const int64_t m0 = (int64_t)mt * 256 + 128 * rank;    // this CTA's A rows and accumulator rows
    const int64_t n0 = (int64_t)nt * 256;                 // the tile's first output column
    const int64_t nb0 = n0 + 128 * rank;                  // this CTA's B rows
    const int KT = (int)(K / BK);
    const int NC = (KT + SF_CH - 1) / SF_CH;              // scale chunks

    if (threadIdx.x == 0) {
        for (int s = 0; s < PSTAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < SF_BUFS; ++b) {
            mbar_init(&sm.sff[b], 1);
            mbar_init(&sm.sfr[b], 2 * SF_CH);     // SF_CH loader warps in each CTA
            mbar_init(&sm.sf_empty[b], 1);
        }
        mbar_init(&sm.tmem_full, 1);
        fence_barrier_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- code-tile TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % PSTAGES;
                const uint32_t ph = (uint32_t)(kt / PSTAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) break;
                if (leader) mbar_arrive_expect_tx(&sm.full[s], 2 * (P_A_TILE + P_B_TILE));
                tma_load_2d_pair(sm.a[s], &tmA, &sm.full[s], kt * BKB, (int32_t)m0);
                tma_load_2d_pair(sm.b[s], &tmB, &sm.full[s], kt * BKB, (int32_t)nb0);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- scale-chunk TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmSA);
            tma_prefetch_desc(&tmSB);
            for (int c = 0; c < NC; ++c) {
                const int b = c % SF_BUFS;
                const uint32_t ph = (uint32_t)(c / SF_BUFS) & 1u;
                if (!wait_or_timeout(&sm.sf_empty[b], ph ^ 1u, err)) break;
                mbar_arrive_expect_tx(&sm.sff[b], SFC_BYTES);
                tma_load_2d(sm.sfc[b], &tmSA, &sm.sff[b], c * 16 * SF_CH, (int32_t)m0);
                tma_load_2d(sm.sfc[b] + SFC_A_BYTES, &tmSB, &sm.sff[b], c * 16 * SF_CH, (int32_t)n0);
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------- MMA issuer (leader)
        if (leader && elect_one()) {
            const uint32_t idesc = idesc_mxf4nvf4(256, 256);
            bool ok = true;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % PSTAGES;
                const uint32_t ph = (uint32_t)(kt / PSTAGES) & 1u;
                const int c = kt / SF_CH, t = kt - c * SF_CH, b = c % SF_BUFS;
                if (!wait_or_timeout(&sm.full[s], ph, err) ||
                    (t == 0 && !wait_or_timeout(&sm.sfr[b], (uint32_t)(c / SF_BUFS) & 1u, err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t col_a = tmem + P_SF_COL0 + SF_COLS_PER_STAGE * (uint32_t)s;
                const uint32_t col_b = col_a + SFA_COLS;
                const uint8_t* at = sm.sfc[b] + t * SF_TILE_ATOM_BYTES;
#pragma unroll
                for (int j = 0; j < MMAS_PER_TILE; ++j) {
                    tmem_cp_32x128b_warpx4_pair(col_a + 4 * j,
                                                smem_desc(smem_u32(at + j * ATOM_BYTES), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4_pair(
                        col_b + 8 * j, smem_desc(smem_u32(at + SFA_BYTES + 2 * j * ATOM_BYTES), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4_pair(
                        col_b + 8 * j + 4,
                        smem_desc(smem_u32(at + SFA_BYTES + (2 * j + 1) * ATOM_BYTES), 0, 128, kLayoutNone));
                }
                const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                for (int j = 0; j < MMAS_PER_TILE; ++j)
                    mma_mxf4nvf4_pair(tmem, desc_kmajor_sw128(a_base + 32 * j), desc_kmajor_sw128(b_base + 32 * j),
                                      idesc, col_a + 4 * j, col_b + 8 * j, (kt > 0 || j > 0) ? 1u : 0u);
                mma_commit_pair_multicast(&sm.empty[s], 0x3);
                if (t == SF_CH - 1 || kt == KT - 1) mma_commit_pair_multicast(&sm.sf_empty[b], 0x3);
            }
            if (ok) mma_commit_pair_multicast(&sm.tmem_full, 0x3);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------- scale loaders
        // Warps 4-5 take the even chunks, 6-7 the odd ones; warp 4 + 2 g + t
        // handles K tile t of its chunks: lane l reads the 16 scale bytes of A
        // rows l + 32 i and B rows l + 32 i for that K tile; once both warps of
        // the pair have read (the barrier reduction), each writes its K
        // tile's atoms over the chunk.
        const int g = (warp - 4) >> 1, t = (warp - 4) & 1;
        const uint32_t leader_sfr0 = map_to_rank(smem_u32(&sm.sfr[0]), 0);
        for (int c = g; c < NC; c += 2) {
            const int b = c % SF_BUFS;
            const uint32_t ph = (uint32_t)(c / SF_BUFS) & 1u;
            const bool landed = __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.sff[b], ph, err));
            uint4 ca[4], cb[8];
            const uint8_t* dense = sm.sfc[b];
            if (landed) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    ca[i] = *reinterpret_cast<const uint4*>(dense + (lane + 32 * i) * (16 * SF_CH) + 16 * t);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    cb[i] = *reinterpret_cast<const uint4*>(dense + SFC_A_BYTES + (lane + 32 * i) * (16 * SF_CH) +
                                                            16 * t);
            }
            if (!bar_red_and(1 + g, 2 * 32, landed)) break;
            uint8_t* at = sm.sfc[b] + t * SF_TILE_ATOM_BYTES;
            write_atoms(at, at + SFA_BYTES, ca, cb, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_sfr0 + 8u * (uint32_t)b);
        }
    }

    // -------------------------------------------------------------- epilogue
    // As in the single-CTA kernel, on this CTA's 128 accumulator rows.
    __syncwarp();
    {
        const int q = warp & 3, half = warp >> 2;
        const int64_t row0 = m0 + 32 * q, col0 = n0 + 128 * half;
        const bool ok = __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.tmem_full, 0, err));
        if (ok && row0 < M && col0 < N) {
            tc_fence_after();
            const float gab = __fmul_rn(__ldg(ga), __ldg(gb));
            uint8_t* stage = &sm.a[0][0] + warp * EPI_WARP_BYTES;
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * half + 32 * c), r[c]);
            tmem_ld_wait();
            stage_and_store(stage, r, gab, c_f32, lane, &tmC, col0, row0, N);
        }
    }

    // both CTAs done: no MMA, copy, TMEM read or remote arrival outstanding
    tc_fence_before();
    cluster_sync();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

int pair_smem_bytes() { return (int)sizeof(PairSmem) + 1024; }


}  // namespace

cudaError_t launch_gemm_nvfp4(const void* aq, const void* as, const float* ag, const void* bq, const void* bs,
                              const float* bg, int64_t m, int64_t n, int64_t k, void* c, int c_f32, uint32_t* err,
                              cudaStream_t st) {
    static int configured[64] = {0};
    // Scale rows can come by TMA when every row starts on a 16-byte boundary
    // (the matrices themselves are 16-byte aligned).
    const bool tma_sf = (k / 16) % 16 == 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(gemm_nvfp4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_nvfp4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_nvfp4_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 pair_smem_bytes());
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    // CTA pairs (256 x 256 tiles) need the scale rows by TMA and pay off once
    // M spans more than one 128-row tile.
    const bool use_pair = tma_sf && m > BM;
    CUtensorMap ta, tb;
    e = make_tmap_u8_2d(&ta, aq, (uint64_t)m, (uint64_t)(k / 2), (uint64_t)(k / 2), BM, BKB);
    if (e != cudaSuccess) return e;
    e = make_tmap_u8_2d(&tb, bq, (uint64_t)n, (uint64_t)(k / 2), (uint64_t)(k / 2), use_pair ? 128 : BN, BKB);
    if (e != cudaSuccess) return e;
    CUtensorMap tsa, tsb;
    std::memset(&tsa, 0, sizeof(tsa));
    std::memset(&tsb, 0, sizeof(tsb));
    if (tma_sf) {
        e = make_tmap_2d(&tsa, as, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)m, (uint64_t)(k / 16), (uint64_t)(k / 16),
                         BM, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e != cudaSuccess) return e;
        e = make_tmap_2d(&tsb, bs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)n, (uint64_t)(k / 16), (uint64_t)(k / 16),
                         BN, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap tc;
    if (c_f32)
        e = make_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)m, (uint64_t)n, (uint64_t)n * 4, 32, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    else
        e = make_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)m, (uint64_t)n, (uint64_t)n * 2, 32, 64,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    if (use_pair) {
        e = make_tmap_2d(&tsa, as, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)m, (uint64_t)(k / 16), (uint64_t)(k / 16),
                         128, 16 * SF_CH, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e != cudaSuccess) return e;
        e = make_tmap_2d(&tsb, bs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)n, (uint64_t)(k / 16), (uint64_t)(k / 16),
                         256, 16 * SF_CH, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e != cudaSuccess) return e;
        const int64_t pairs = ((m + 255) / 256) * ((n + 255) / 256);
        return launch_pdl(gemm_nvfp4_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(NUM_THREADS), pair_smem_bytes(),
                          st, ta, tb, tsa, tsb, tc, ag, bg, m, n, k, c_f32, err);
    }
    const int64_t grid = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    return launch_pdl(tma_sf ? gemm_nvfp4_kernel<true> : gemm_nvfp4_kernel<false>, dim3((unsigned)grid),
                      dim3(NUM_THREADS), smem_bytes(), st, ta, tb, tsa, tsb, tc, (const uint8_t*)as, ag,
                      (const uint8_t*)bs, bg, m, n, k, c, c_f32, err);
}

}  // namespace fpq
