// gemm_mxfp8.cu -- block-scaled MXFP8 GEMM on the 5th-generation tensor
// cores: C = A * B^T with A [M, K], B [N, K] E4M3 codes and one E8M0 scale
// per 32 K-elements of every row of A and of B, fp32 accumulation in TMEM,
// bf16 (round-to-nearest-even) or fp32 output.  The same kernel serves the
// grouped (per-expert) product, where row ranges of A select the expert
// weight B[g].
//
// Per CTA one 128 x 256 output tile; the K loop runs over 128-wide K tiles
// through a STAGES-deep shared-memory ring.  Warp roles:
//   warp 0  TMA producer: A and B tiles (128-byte swizzle, no multicast)
//   warp 1  scale-factor loader: gathers the row-major E8M0 scales of the
//           tile's 128 A rows and 256 B rows into the 32x4x4 chunk layout the
//           shared->TMEM copy expects (rows r, r+32, r+64, r+96 interleaved)
//   warp 2  TMEM allocator and MMA issuer (one elected thread):
//           tcgen05.cp of the scales, then 4 x tcgen05.mma kind::mxf8f6f4
//           (K = 32 each, scale byte selected per MMA), tcgen05.commit
//   warps 4-7 epilogue: tcgen05.ld of the accumulator, convert, store
// Every wait on an mbarrier is bounded by wall time (4 s, or
// FPQ_WAIT_TIMEOUT_MS, read once per process); on expiry the kernel records FPQ_ERR_DEVICE_TIMEOUT in
// the device error word and unwinds (TMEM freed, no store).  For testing
// that path, FPQ_DEBUG_GEMM_STALL=1 (also read once per process, so a test sets
// it before the process's first launch) makes the producer declare more TMA bytes
// per stage than it loads, so the stage barriers never complete: every load
// it issues still lands, and the waits run out instead of hanging.
#include <cstdlib>
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
constexpr int A_TILE = BM * BK, B_TILE = BN * BK;
constexpr int SFA_BYTES = 512, SFB_BYTES = 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = BN;            // scale columns follow the accumulator
constexpr uint32_t SF_COLS_PER_STAGE = 16;  // 4 (A) + 8 (B), padded
constexpr int NUM_THREADS = 256;
constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;

constexpr int kMaxGroups = 1024;   // the C ABI rejects more groups

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t sfa[STAGES][SFA_BYTES];
    uint8_t sfb[STAGES][SFB_BYTES];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full;
    uint32_t tmem_base;
    int32_t tile_valid;
    int32_t group;
    int32_t row_begin, row_end;   // A rows owned by this tile's group
    int32_t m_tile, n_tile;
    int32_t off[kMaxGroups + 1];  // grouped: the group offsets, staged once per CTA
};

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ bool wait_or_timeout(uint64_t* bar, uint32_t parity, uint32_t* err, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > timeout_ns) {
            raise_device_error(err, FPQ_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pick(const uint4& v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Scales of one row for K tiles [4*kg, 4*kg + 4): 16 bytes (one word per K
// tile, one byte per 32-wide sub-block).  Rows outside [0, nrows) and K tiles
// past the end read as zero.
__device__ __forceinline__ uint4 load_sf_group(const uint8_t* sf, int64_t row, int64_t nrows, int sf_pitch,
                                               int kg, bool vec16) {
    if (row < 0 || row >= nrows) return make_uint4(0, 0, 0, 0);
    const uint8_t* p = sf + row * sf_pitch + kg * 16;
    if (vec16) return *reinterpret_cast<const uint4*>(p);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = (kg * 16 + 4 * j + 4 <= sf_pitch) ? *reinterpret_cast<const uint32_t*>(p + 4 * j) : 0u;
    return make_uint4(w[0], w[1], w[2], w[3]);
}

struct TileMap {
    int valid, g, mt, nt;
    int32_t rb, re;     // A rows owned by the tile's group
};

// Tile t -> (group, m tile, n tile) for row tiles of bm rows, run by one warp
// (all lanes return the same map).  Grouped (off = the offsets staged in
// shared memory): the groups are scanned 32 at a time (tile counts,
// inclusive prefix sum over the warp, ballot for the group holding tile t),
// and every group is validated: offsets must rise from 0 to M.
__device__ TileMap map_tile(int t, int bm, const int32_t* off, bool grouped, int groups, int64_t M, int n_tiles,
                            int lane, uint32_t* err) {
    TileMap r{0, 0, 0, 0, 0, (int32_t)M};
    if (!grouped) {
        r.mt = t / n_tiles;
        r.nt = t - r.mt * n_tiles;
        r.valid = (int64_t)r.mt * bm < M;
        return r;
    }
    bool bad = off[0] != 0 || off[groups] != (int32_t)M;
    int before = 0;                          // tiles of the groups in earlier chunks
    for (int c0 = 0; c0 < groups; c0 += 32) {
        const int e = c0 + lane;
        const int32_t b0 = e < groups ? off[e] : 0, b1 = e < groups ? off[e + 1] : 0;
        if (b1 < b0) bad = true;
        const int tiles = b1 > b0 ? ((b1 - b0 + bm - 1) / bm) * n_tiles : 0;
        int incl = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        const int lo = before + incl - tiles;
        const unsigned hit = __ballot_sync(0xFFFFFFFFu, tiles > 0 && t >= lo && t < lo + tiles);
        if (hit) {
            const int src = __ffs(hit) - 1;
            const int tt = t - __shfl_sync(0xFFFFFFFFu, lo, src);
            r.g = c0 + src;
            r.rb = __shfl_sync(0xFFFFFFFFu, b0, src);
            r.re = __shfl_sync(0xFFFFFFFFu, b1, src);
            r.mt = tt / n_tiles;
            r.nt = tt - r.mt * n_tiles;
            r.valid = 1;
        }
        before += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (__any_sync(0xFFFFFFFFu, bad)) {
        if (blockIdx.x == 0 && lane == 0) raise_device_error(err, FPQ_ERR_DEVICE_BAD_INPUT);
        r.valid = 0;
    }
    return r;
}

// grouped: offsets != nullptr.  For the dense product groups = 1 and the
// single group spans rows [0, M).
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_mxfp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                  const int32_t* __restrict__ offsets, int groups, int64_t M, int64_t N, int64_t K,
                  void* __restrict__ C, int c_f32, uint32_t* err, uint64_t timeout_ns, uint32_t extra_tx) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int KT = (int)(K / BK);
    const int sf_pitch = (int)(K / 32);

    // Map this CTA to (group, m tile, n tile).  Grouped: all threads stage
    // the offsets in shared memory with one coalesced read, then warp 0
    // scans the groups 32 at a time (tile counts, inclusive prefix sum over
    // the warp, ballot for the group holding tile blockIdx.x) and validates
    // every group: offsets must rise from 0 to M.
    if (offsets != nullptr) {
        pdl_wait();    // the group offsets may come from the preceding grid
        for (int i = threadIdx.x; i <= groups; i += NUM_THREADS) sm.off[i] = offsets[i];
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 2);     // TMA bytes + scale-factor warp
            mbar_init(&sm.empty[s], 1);    // tcgen05.commit
        }
        mbar_init(&sm.tmem_full, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 0) {
        const TileMap tm = map_tile(blockIdx.x, BM, sm.off, offsets != nullptr, groups, M, n_tiles, lane, err);
        if (lane == 0) {
            sm.tile_valid = tm.valid;
            sm.group = tm.g;
            sm.m_tile = tm.mt;
            sm.n_tile = tm.nt;
            sm.row_begin = tm.rb;
            sm.row_end = tm.re;
        }
    }
    __syncthreads();
    if (!sm.tile_valid) return;

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

    const int64_t a_row0 = (int64_t)sm.row_begin + (int64_t)sm.m_tile * BM;   // first A row of the tile
    const int64_t a_rows_end = sm.row_end;                                     // rows >= this are masked
    const int64_t n0 = (int64_t)sm.n_tile * BN;
    const int64_t b_row0 = (int64_t)sm.group * N + n0;                         // first row of B (flattened)

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err, timeout_ns)) break;
                mbar_arrive_expect_tx(&sm.full[s], A_TILE + B_TILE + extra_tx);
                tma_load_2d(sm.a[s], &tmA, &sm.full[s], kt * BK, (int32_t)a_row0);
                tma_load_2d(sm.b[s], &tmB, &sm.full[s], kt * BK, (int32_t)b_row0);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- scale factors
        const bool vec16 = (sf_pitch % 16) == 0;
        const int KG = (KT + 3) / 4;
        const int64_t b_rows_valid = (int64_t)sm.group * N + N;   // B rows of this group end here
        uint4 ca[4], cb[8], na[4], nb[8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            ca[i] = load_sf_group(sfa, a_row0 + lane + 32 * i, a_rows_end, sf_pitch, 0, vec16);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            cb[i] = load_sf_group(sfb, (b_row0 + lane + 32 * i < b_rows_valid) ? b_row0 + lane + 32 * i : -1,
                                  b_rows_valid, sf_pitch, 0, vec16);
        bool alive = true;
        for (int kg = 0; kg < KG && alive; ++kg) {
            if (kg + 1 < KG) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    na[i] = load_sf_group(sfa, a_row0 + lane + 32 * i, a_rows_end, sf_pitch, kg + 1, vec16);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    nb[i] = load_sf_group(sfb, (b_row0 + lane + 32 * i < b_rows_valid) ? b_row0 + lane + 32 * i : -1,
                                          b_rows_valid, sf_pitch, kg + 1, vec16);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kt = kg * 4 + j;
                if (kt >= KT) break;
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err, timeout_ns)) { alive = false; break; }
                *reinterpret_cast<uint4*>(sm.sfa[s] + lane * 16) =
                    make_uint4(pick(ca[0], j), pick(ca[1], j), pick(ca[2], j), pick(ca[3], j));
                *reinterpret_cast<uint4*>(sm.sfb[s] + lane * 16) =
                    make_uint4(pick(cb[0], j), pick(cb[1], j), pick(cb[2], j), pick(cb[3], j));
                *reinterpret_cast<uint4*>(sm.sfb[s] + 512 + lane * 16) =
                    make_uint4(pick(cb[4], j), pick(cb[5], j), pick(cb[6], j), pick(cb[7], j));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.full[s]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) ca[i] = na[i];
#pragma unroll
            for (int i = 0; i < 8; ++i) cb[i] = nb[i];
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------- MMA issuer
        if (elect_one()) {
            bool ok = true;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!wait_or_timeout(&sm.full[s], ph, err, timeout_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sf_col = tmem + SF_COL0 + SF_COLS_PER_STAGE * (uint32_t)s;
                tmem_cp_32x128b_warpx4(sf_col + 0, smem_desc(smem_u32(sm.sfa[s]), 0, 128, kLayoutNone));
                tmem_cp_32x128b_warpx4(sf_col + 4, smem_desc(smem_u32(sm.sfb[s]), 0, 128, kLayoutNone));
                tmem_cp_32x128b_warpx4(sf_col + 8, smem_desc(smem_u32(sm.sfb[s] + 512), 0, 128, kLayoutNone));
                const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                for (int k = 0; k < BK / 32; ++k) {
                    const uint32_t idesc = idesc_mxf8f6f4(BM, BN, (uint32_t)k, (uint32_t)k);
                    mma_mxf8f6f4(tmem, desc_kmajor_sw128(a_base + 32 * k), desc_kmajor_sw128(b_base + 32 * k), idesc,
                                 (sf_col + 0) | ((uint32_t)k << 30), (sf_col + 4) | ((uint32_t)k << 30),
                                 (kt > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(&sm.empty[s]);
            }
            if (ok) mma_commit(&sm.tmem_full);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------- epilogue
        // Once the last MMA has completed the operand ring is free: each warp
        // stages its 32 x 256 block of C there (row l of the block at l *
        // row_bytes, 16-byte chunk c at position c ^ l, so neither the
        // writes by rows nor the reads along a row conflict), then writes C
        // one full row at a time (512 or 1024 contiguous bytes per store
        // instruction), skipping rows outside the group and columns past N.
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        const int64_t row0 = a_row0 + 32 * q;
        if (wait_or_timeout(&sm.tmem_full, 0, err, timeout_ns)) {
            tc_fence_after();
            uint8_t* stage = &sm.a[0][0] + (warp - 4) * (32 * BN * 4);
            const int row_bytes = c_f32 ? BN * 4 : BN * 2;
            uint8_t* my_row = stage + lane * row_bytes;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * c), r);
                tmem_ld_wait();
                if (c_f32) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(my_row + 16 * ((8 * c + j) ^ lane)) =
                            make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            h[e] = f32x2_to_bf16x2(__uint_as_float(r[8 * j + 2 * e]), __uint_as_float(r[8 * j + 2 * e + 1]));
                        *reinterpret_cast<uint4*>(my_row + 16 * ((4 * c + j) ^ lane)) = make_uint4(h[0], h[1], h[2], h[3]);
                    }
                }
            }
            __syncwarp();
            const int chunks = row_bytes / 16;                    // 32 (bf16) or 64 (fp32) per row
            const int cols_per_chunk = c_f32 ? 4 : 8;
#pragma unroll 1
            for (int rr = 0; rr < 32; ++rr) {
                const int64_t row = row0 + rr;
                if (row >= a_rows_end) break;
                const uint8_t* src_row = stage + rr * row_bytes;
                uint8_t* dst_row = reinterpret_cast<uint8_t*>(C) + (row * N + n0) * (c_f32 ? 4 : 2);
                for (int ch = lane; ch < chunks; ch += 32)
                    if (n0 + (int64_t)ch * cols_per_chunk < N)
                        st_v4(dst_row + 16 * ch, *reinterpret_cast<const uint4*>(src_row + 16 * (ch ^ rr)));
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

// ============================================================== CTA pairs, persistent
// A cluster of two CTAs computes 256 x 256 output tiles with tcgen05
// cta_group::2 (grouped: 256 rows of one group), walking the tile list
// pair, pair + P, pair + 2P, ... (P = the pairs launched, at most one per
// two SMs).  CTA r of the pair stages A rows row_begin + 256 mt + 128 r and
// B rows n0 + 128 r of every 128-wide K tile in its own shared memory and
// receives its 128 accumulator rows in its own TMEM; per SM a K tile is
// 16 + 16 KB of codes instead of the one-CTA kernel's 16 + 32 KB (the TMA
// feed from L2 is what bounds that kernel).  The leader issues the MMAs
// (M = 256, N = 256, 4 x K = 32 per K tile, scale byte selected per MMA) and
// the scale copies, and commits to the barriers of both CTAs.
//
// Scales: chunks of P_SF_CH K tiles, one TMA box of (4 P_SF_CH)-byte scale
// rows for this CTA's 128 A rows and one for the tile's 256 B rows (every
// output column meets this CTA's rows), two chunks in flight; loader warps
// 4-7 rearrange a landed chunk in place into the TMEM-copy atoms of its K
// tiles (warp 4 + i: K tiles 2i, 2i + 1) and arrive on the leader's sfr.
//
// TMEM holds one 256-column accumulator and the scale columns of the ring's
// stages, so the accumulator is handed over instead of double-buffered: the
// eight epilogue warps (8-15; warp w reads TMEM lanes 32 (w & 3) .. + 31 and
// columns 128 ((w - 8) >> 2) .. + 127) read their block into registers,
// arrive on the leader's tmem_empty, and only then convert and store to C,
// while the code and scale producers, which run ahead by the ring's depth,
// and the MMAs of the next tile proceed.  Each thread stores one row segment
// (rows outside the group and columns past N skipped) with cache-streaming
// stores, so that C does not push out of L2 the operand tiles that the tiles
// in flight share.
//
// Warp roles in both CTAs: warp 0 code-tile TMA producer; warp 1 scale-chunk
// TMA producer; warp 2 TMEM allocator (leader: MMA issuer); warps 4-7 scale
// loaders; warps 8-15 epilogue.  The pipeline counters (ring stage, scale
// chunk, tile parity) run on across tiles.
constexpr int P_STAGES = 6;
constexpr int P_A_TILE = 128 * BK, P_B_TILE = 128 * BK;
constexpr int P_SF_CH = 8;                                   // K tiles per scale chunk
constexpr int P_SFC_A = 128 * 4 * P_SF_CH;                   // dense: A row r at r * 32
constexpr int P_SFC_BYTES = P_SFC_A + 256 * 4 * P_SF_CH;     // + 256 B rows
constexpr int P_TILE_ATOMS = SFA_BYTES + SFB_BYTES;          // a K tile's atoms: A, B rows 0-127, B rows 128-255
static_assert(P_SF_CH * P_TILE_ATOMS == P_SFC_BYTES, "in-place rearrangement");
static_assert(P_SF_CH == 8, "loader warp 4 + i takes K tiles 2i and 2i + 1 of a chunk");
constexpr uint32_t P_SF_COL0 = 256;
static_assert(P_SF_COL0 + P_STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM columns (pair)");
constexpr int P_THREADS = 512;
constexpr int P_EPI_WARP0 = 8, P_EPI_WARPS = 8;

struct __align__(1024) PairSmem {
    uint8_t a[P_STAGES][P_A_TILE];
    uint8_t b[P_STAGES][P_B_TILE];
    uint8_t sfc[2][P_SFC_BYTES];
    uint64_t full[P_STAGES];    // leader's copy used: code tiles of both CTAs
    uint64_t empty[P_STAGES];   // both CTAs: the leader's commit after the stage's MMAs
    uint64_t sff[2];            // this CTA's scale chunk has landed
    uint64_t sfr[2];            // leader's copy used: atoms of both CTAs written (8 warps)
    uint64_t sf_empty[2];       // both CTAs: the leader's commit after a chunk's last MMAs
    uint64_t tmem_full;         // both CTAs: the leader's commit after a tile's last MMA
    uint64_t tmem_empty;        // leader's copy used: the epilogue warps of both CTAs read the accumulator
    uint32_t tmem_base;
    int32_t tiles;              // pair tiles of the whole product (0: nothing to do or malformed offsets)
    int32_t off[kMaxGroups + 1];
};

// Number of 2 BM-row tiles of the product, run by one warp; grouped offsets
// are validated as in map_tile (malformed: reported once, 0 tiles).
__device__ int count_tiles(int bm, const int32_t* off, bool grouped, int groups, int64_t M, int n_tiles, int lane,
                           uint32_t* err) {
    if (!grouped) return (int)((M + bm - 1) / bm) * n_tiles;
    bool bad = off[0] != 0 || off[groups] != (int32_t)M;
    int total = 0;
    for (int c0 = 0; c0 < groups; c0 += 32) {
        const int e = c0 + lane;
        const int32_t b0 = e < groups ? off[e] : 0, b1 = e < groups ? off[e + 1] : 0;
        if (b1 < b0) bad = true;
        int tiles = b1 > b0 ? ((b1 - b0 + bm - 1) / bm) * n_tiles : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tiles += __shfl_xor_sync(0xFFFFFFFFu, tiles, o);
        total += tiles;
    }
    if (__any_sync(0xFFFFFFFFu, bad)) {
        if (blockIdx.x == 0 && lane == 0) raise_device_error(err, FPQ_ERR_DEVICE_BAD_INPUT);
        return 0;
    }
    return total;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
gemm_mxfp8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                       const int32_t* __restrict__ offsets, int groups, int64_t M, int64_t N, int64_t K,
                       void* __restrict__ C, int c_f32, uint32_t* err, uint64_t timeout_ns, uint32_t extra_tx) {
    extern __shared__ uint8_t smem_raw[];
    PairSmem& sm = *reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const bool grouped = offsets != nullptr;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int n_tiles = (int)((N + BN - 1) / BN);
    const int KT = (int)(K / BK);
    const int NC = (KT + P_SF_CH - 1) / P_SF_CH;

    if (grouped) {
        pdl_wait();    // the group offsets may come from the preceding grid
        for (int i = threadIdx.x; i <= groups; i += P_THREADS) sm.off[i] = offsets[i];
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.sff[b], 1);
            mbar_init(&sm.sfr[b], 8);
            mbar_init(&sm.sf_empty[b], 1);
        }
        mbar_init(&sm.tmem_full, 1);
        mbar_init(&sm.tmem_empty, 2 * P_EPI_WARPS);
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 0) {
        const int t = count_tiles(2 * BM, sm.off, grouped, groups, M, n_tiles, lane, err);
        if (lane == 0) sm.tiles = t;
    }
    __syncthreads();
    // the same count in both CTAs of a pair: both leave here or neither
    const int my_tiles = sm.tiles > pair ? (sm.tiles - pair + npairs - 1) / npairs : 0;
    if (my_tiles == 0) return;

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
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
        }
        uint32_t it = 0;
        bool alive = true;
        for (int i = 0; i < my_tiles && alive; ++i) {
            const TileMap tm = map_tile(pair + i * npairs, 2 * BM, sm.off, grouped, groups, M, n_tiles, lane, err);
            const int32_t a_row0 = tm.rb + tm.mt * 2 * BM + 128 * (int32_t)rank;
            const int32_t b_row0 = (int32_t)((int64_t)tm.g * N + (int64_t)tm.nt * BN + 128 * rank);
            if (lane == 0) {
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = (int)(it % P_STAGES);
                    const uint32_t ph = (it / P_STAGES) & 1u;
                    if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err, timeout_ns)) { alive = false; break; }
                    if (leader) mbar_arrive_expect_tx(&sm.full[s], 2 * (P_A_TILE + P_B_TILE) + extra_tx);
                    tma_load_2d_pair(sm.a[s], &tmA, &sm.full[s], kt * BK, a_row0);
                    tma_load_2d_pair(sm.b[s], &tmB, &sm.full[s], kt * BK, b_row0);
                }
            }
            alive = __shfl_sync(0xFFFFFFFFu, alive, 0);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- scale-chunk TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmSA);
            tma_prefetch_desc(&tmSB);
        }
        uint32_t cc = 0;
        bool alive = true;
        for (int i = 0; i < my_tiles && alive; ++i) {
            const TileMap tm = map_tile(pair + i * npairs, 2 * BM, sm.off, grouped, groups, M, n_tiles, lane, err);
            const int32_t a_row0 = tm.rb + tm.mt * 2 * BM + 128 * (int32_t)rank;
            const int32_t bt_row0 = (int32_t)((int64_t)tm.g * N + (int64_t)tm.nt * BN);
            if (lane == 0) {
                for (int c = 0; c < NC; ++c, ++cc) {
                    const int b = (int)(cc & 1u);
                    const uint32_t ph = (cc >> 1) & 1u;
                    if (!wait_or_timeout(&sm.sf_empty[b], ph ^ 1u, err, timeout_ns)) { alive = false; break; }
                    mbar_arrive_expect_tx(&sm.sff[b], P_SFC_BYTES);
                    tma_load_2d(sm.sfc[b], &tmSA, &sm.sff[b], c * 4 * P_SF_CH, a_row0);
                    tma_load_2d(sm.sfc[b] + P_SFC_A, &tmSB, &sm.sff[b], c * 4 * P_SF_CH, bt_row0);
                }
            }
            alive = __shfl_sync(0xFFFFFFFFu, alive, 0);
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------- MMA issuer (leader)
        if (leader && elect_one()) {
            uint32_t it = 0, cc = 0;
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                // the accumulator is free once both CTAs' epilogue warps have read the previous tile
                if (!wait_or_timeout(&sm.tmem_empty, ((uint32_t)i & 1u) ^ 1u, err, timeout_ns)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = (int)(it % P_STAGES);
                    const uint32_t ph = (it / P_STAGES) & 1u;
                    const int t = kt % P_SF_CH;
                    const uint32_t ch = cc + (uint32_t)(kt / P_SF_CH);
                    const int b = (int)(ch & 1u);
                    if (!wait_or_timeout(&sm.full[s], ph, err, timeout_ns) ||
                        (t == 0 && !wait_or_timeout(&sm.sfr[b], (ch >> 1) & 1u, err, timeout_ns))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_col = tmem + P_SF_COL0 + SF_COLS_PER_STAGE * (uint32_t)s;
                    const uint8_t* at = sm.sfc[b] + t * P_TILE_ATOMS;
                    tmem_cp_32x128b_warpx4_pair(sf_col + 0, smem_desc(smem_u32(at), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4_pair(sf_col + 4, smem_desc(smem_u32(at + SFA_BYTES), 0, 128, kLayoutNone));
                    tmem_cp_32x128b_warpx4_pair(sf_col + 8,
                                                smem_desc(smem_u32(at + SFA_BYTES + 512), 0, 128, kLayoutNone));
                    const uint32_t a_base = smem_u32(sm.a[s]), b_base = smem_u32(sm.b[s]);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        const uint32_t idesc = idesc_mxf8f6f4(2 * BM, BN, (uint32_t)k, (uint32_t)k);
                        mma_mxf8f6f4_pair(tmem, desc_kmajor_sw128(a_base + 32 * k), desc_kmajor_sw128(b_base + 32 * k),
                                          idesc, (sf_col + 0) | ((uint32_t)k << 30), (sf_col + 4) | ((uint32_t)k << 30),
                                          (kt > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit_pair_multicast(&sm.empty[s], 0x3);
                    if (t == P_SF_CH - 1 || kt == KT - 1) mma_commit_pair_multicast(&sm.sf_empty[b], 0x3);
                }
                if (ok) mma_commit_pair_multicast(&sm.tmem_full, 0x3);
                cc += (uint32_t)NC;
            }
        }
    } else if (warp >= 4 && warp < P_EPI_WARP0) {
        // ---------------------------------------------------------- scale loaders
        // Lane l reads, for K tiles 2i and 2i + 1 of the chunk (i = warp - 4),
        // the 8 scale bytes of A rows l + 32 q (q < 4) and B rows l + 32 q
        // (q < 8); once all four warps have read (the barrier reduction) each
        // writes its two K tiles' atoms: word q of lane l = row l + 32 q.
        const int i2 = 2 * (warp - 4);
        const uint32_t leader_sfr0 = map_to_rank(smem_u32(&sm.sfr[0]), 0);
        const uint32_t chunks = (uint32_t)my_tiles * (uint32_t)NC;
        for (uint32_t cc = 0; cc < chunks; ++cc) {
            const int b = (int)(cc & 1u);
            const uint32_t ph = (cc >> 1) & 1u;
            const bool landed = __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.sff[b], ph, err, timeout_ns));
            uint2 ra[4], rb[8];
            const uint8_t* dense = sm.sfc[b];
            if (landed) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    ra[q] = *reinterpret_cast<const uint2*>(dense + (lane + 32 * q) * (4 * P_SF_CH) + 4 * i2);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    rb[q] = *reinterpret_cast<const uint2*>(dense + P_SFC_A + (lane + 32 * q) * (4 * P_SF_CH) + 4 * i2);
            }
            if (!bar_red_and(1, 4 * 32, landed)) break;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint8_t* at = sm.sfc[b] + (i2 + h) * P_TILE_ATOMS;
                auto w = [&](const uint2& v) { return h ? v.y : v.x; };
                *reinterpret_cast<uint4*>(at + lane * 16) = make_uint4(w(ra[0]), w(ra[1]), w(ra[2]), w(ra[3]));
                *reinterpret_cast<uint4*>(at + SFA_BYTES + lane * 16) =
                    make_uint4(w(rb[0]), w(rb[1]), w(rb[2]), w(rb[3]));
                *reinterpret_cast<uint4*>(at + SFA_BYTES + 512 + lane * 16) =
                    make_uint4(w(rb[4]), w(rb[5]), w(rb[6]), w(rb[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_sfr0 + 8u * (uint32_t)b);
        }
    } else if (warp >= P_EPI_WARP0) {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3, half = (warp - P_EPI_WARP0) >> 2;
        const uint32_t leader_empty = map_to_rank(smem_u32(&sm.tmem_empty), 0);
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * half);
        for (int i = 0; i < my_tiles; ++i) {
            const TileMap tm = map_tile(pair + i * npairs, 2 * BM, sm.off, grouped, groups, M, n_tiles, lane, err);
            const int64_t row = (int64_t)tm.rb + (int64_t)tm.mt * 2 * BM + 128 * (int64_t)rank + 32 * q + lane;
            const int64_t col0 = (int64_t)tm.nt * BN + 128 * half;
            const bool row_ok = row < (int64_t)tm.re;
            if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.tmem_full, (uint32_t)i & 1u, err, timeout_ns))) break;
            tc_fence_after();
            if (!c_f32) {
                uint32_t h[64];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    // two loads in flight per wait: four TMEM round trips instead of eight
                    uint32_t r[16], r2[16];
                    tmem_ld_32x32b_x16(taddr + (uint32_t)(16 * c), r);
                    tmem_ld_32x32b_x16(taddr + (uint32_t)(16 * c + 16), r2);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        h[8 * c + e] = f32x2_to_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                        h[8 * c + 8 + e] = f32x2_to_bf16x2(__uint_as_float(r2[2 * e]), __uint_as_float(r2[2 * e + 1]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(leader_empty);
                if (row_ok) {
                    uint8_t* dst = reinterpret_cast<uint8_t*>(C) + (row * N + col0) * 2;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (col0 + 8 * j < N)
                            st_v4_stream(dst + 16 * j, make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]));
                }
            } else {
                uint8_t* dst = reinterpret_cast<uint8_t*>(C) + (row * N + col0) * 4;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + (uint32_t)(32 * c), r);
                    tmem_ld_wait();
                    if (row_ok) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            if (col0 + 32 * c + 4 * j < N)
                                st_v4_stream(dst + 128 * c + 16 * j,
                                             make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(leader_empty);
            }
        }
    }

    // both CTAs done: no MMA, copy, TMEM read or remote arrival outstanding
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

int pair_smem_bytes() { return (int)sizeof(PairSmem) + 1024; }

// Wait limit and the stall switch for the timeout test (see the file header),
// read from the environment once per process, at the first launch.
uint64_t wait_timeout_ns() {
    static const uint64_t ns = [] {
        const char* v = std::getenv("FPQ_WAIT_TIMEOUT_MS");
        const long ms = v ? std::atol(v) : 0;
        return ms > 0 ? (uint64_t)ms * 1000000ull : kDefaultTimeoutNs;
    }();
    return ns;
}
uint32_t debug_extra_tx() {
    static const uint32_t tx = [] {
        const char* v = std::getenv("FPQ_DEBUG_GEMM_STALL");
        return (v && v[0] == '1') ? 16u : 0u;
    }();
    return tx;
}

// CTA pairs need the scale rows on 16-byte boundaries (K a multiple of 512)
// and pay off once M spans more than one 128-row tile.
bool use_pair(int64_t M, int64_t K) { return K % 512 == 0 && M > BM; }

cudaError_t launch(const void* aq, const void* as, const void* bq, const void* bs, const int32_t* offsets,
                   int groups, int64_t M, int64_t N, int64_t K, void* c, int c_f32, uint32_t* err,
                   int64_t tiles, int64_t pair_tiles, int sms, cudaStream_t st) {
    const bool pair = use_pair(M, K);
    CUtensorMap ta, tb;
    cudaError_t e = make_tmap_u8_2d(&ta, aq, (uint64_t)M, (uint64_t)K, (uint64_t)K, BM, BK);
    if (e != cudaSuccess) return e;
    e = make_tmap_u8_2d(&tb, bq, (uint64_t)(groups * N), (uint64_t)K, (uint64_t)K, pair ? 128 : BN, BK);
    if (e != cudaSuccess) return e;
    if (!pair) {
        e = cudaFuncSetAttribute(gemm_mxfp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
        if (e != cudaSuccess) return e;
        if (tiles < 1) return cudaSuccess;
        return launch_pdl(gemm_mxfp8_kernel, dim3((unsigned)tiles), dim3(NUM_THREADS), smem_bytes(), st, ta, tb,
                          (const uint8_t*)as, (const uint8_t*)bs, offsets, groups, M, N, K, c, c_f32, err,
                          wait_timeout_ns(), debug_extra_tx());
    }
    CUtensorMap tsa, tsb;
    e = make_tmap_2d(&tsa, as, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)M, (uint64_t)(K / 32), (uint64_t)(K / 32),
                     128, 4 * P_SF_CH, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&tsb, bs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(groups * N), (uint64_t)(K / 32),
                     (uint64_t)(K / 32), 256, 4 * P_SF_CH, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_mxfp8_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pair_smem_bytes());
    if (e != cudaSuccess) return e;
    if (pair_tiles < 1) return cudaSuccess;
    // persistent: at most one pair per two SMs; the kernel counts the real
    // tiles (grouped: from the device-side offsets) and walks them
    const int64_t pairs = min64(pair_tiles, (int64_t)(sms > 1 ? sms / 2 : 1));
    return launch_pdl(gemm_mxfp8_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(P_THREADS), pair_smem_bytes(),
                      st, ta, tb, tsa, tsb, offsets, groups, M, N, K, c, c_f32, err, wait_timeout_ns(),
                      debug_extra_tx());
}

}  // namespace

cudaError_t launch_gemm_mxfp8(const void* aq, const void* as, const void* bq, const void* bs, int64_t m,
                              int64_t n, int64_t k, void* c, int c_f32, uint32_t* err, int sms, cudaStream_t st) {
    const int64_t n_tiles = (n + BN - 1) / BN;
    return launch(aq, as, bq, bs, nullptr, 1, m, n, k, c, c_f32, err, ((m + BM - 1) / BM) * n_tiles,
                  ((m + 2 * BM - 1) / (2 * BM)) * n_tiles, sms, st);
}

cudaError_t launch_grouped_gemm_mxfp8(const void* aq, const void* as, const void* bq, const void* bs,
                                      const int32_t* offsets, int groups, int64_t total_m, int64_t n, int64_t k,
                                      void* c, int c_f32, uint32_t* err, int sms, cudaStream_t st) {
    // Upper bounds on the tile counts without reading the device-side
    // offsets: every group adds at most one partial row tile.
    const int64_t n_tiles = (n + BN - 1) / BN;
    return launch(aq, as, bq, bs, offsets, groups, total_m, n, k, c, c_f32, err,
                  ((total_m + BM - 1) / BM + groups) * n_tiles, ((total_m + 2 * BM - 1) / (2 * BM) + groups) * n_tiles,
                  sms, st);
}

}  // namespace fpq
