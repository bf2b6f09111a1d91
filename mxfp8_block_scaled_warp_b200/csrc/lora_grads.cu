// lora_grads.cu -- the two LoRA gradients of the QAT backward in one pass
// over dW_eff ("DeepSeek R1 and V3 get quantization-aware fine-tuning on
// Fireworks", Synopsis: the adapters are trained through the quantized
// forward; with W_eff = W + (alpha / r) B A the weight gradient reaches them
// as dA = (alpha / r) B^T dW_eff and dB = (alpha / r) dW_eff A^T):
//   dA [r, k] = (alpha / r) sum_n B[n, .]^T dW[n, .]
//   dB [n, r] = (alpha / r) sum_k dW[., k] A[., k]^T
// Both contract dW_eff [n, k] (bf16) with a rank-r factor, so one CTA per
// (128-row strip of dW, range of 128-wide K tiles) loads each dW tile once
// (TMA, 128-byte swizzle) and issues two tcgen05 bf16 products from it:
//   dB: M = the tile's 128 rows, N = r (padded to 16), K = its 128 columns,
//       dW read K-major, A's tile K-major; accumulated in TMEM over the
//       CTA's K tiles;
//   dA^T: M = the tile's 128 columns, N = r, K = its 128 rows, the same dW
//       tile read MN-major (its 64-column halves 16 KB apart), B^T of the
//       strip K-major (built once per CTA in shared memory); a fresh
//       accumulator per K tile, double-buffered so the epilogue warps read
//       one while the next is computed.
// The epilogue warps write fp32 partial sums (dA^T per strip, dB per K
// range); a second kernel adds them in a fixed order, times alpha / r, to
// bf16, so results do not depend on scheduling.  Every mbarrier wait is
// bounded by wall time (4 s); on expiry the kernel records
// FPQ_ERR_DEVICE_TIMEOUT and unwinds.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

using namespace sm100;

constexpr int TK = 128;                       // K tile (columns of dW) and strip height (rows of dW)
constexpr int DW_TILE = TK * TK * 2;          // 32 KB: two boxes of 64 columns x 128 rows
constexpr int DW_BOX = DW_TILE / 2;
constexpr int MAX_RP = 64;                    // padded rank handled here
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr uint64_t kTimeoutNs = 4000000000ull;

// Ring depth: as many 32 KB tiles of dW (plus A's tile) in flight as shared
// memory holds, so that a CTA's K range (about six tiles when the strips x
// K ranges fill the SMs) is requested from HBM almost at once.
__host__ __device__ constexpr int ring_stages(int rp) { return rp <= 16 ? 6 : rp <= 32 ? 5 : 4; }

template <int RP>
struct __align__(1024) Smem {
    static constexpr int ST = ring_stages(RP);
    uint8_t dw[ST][DW_TILE];
    uint8_t a[ST][2 * RP * 128];              // A's K tile: two boxes of 64 columns x RP rows
    uint8_t bt[2 * RP * 128];                 // B^T of the strip: two boxes of 64 rows-of-dW x RP rows
    uint64_t full[ST];
    uint64_t empty[ST];
    uint64_t da_full[2];
    uint64_t da_empty[2];
    uint64_t db_full;
    uint32_t tmem_base;
};

// kind::f16, bf16 x bf16 -> fp32: D fp32 (bits 4-5), A and B bf16 (7-9,
// 10-12), A / B MN-major (15 / 16), N >> 3 at 17, M >> 4 at 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
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

// Read RP fp32 accumulator columns of this warp's 32 TMEM lanes and store
// them as one row of RP floats per lane (rows past `rows` skipped).
template <int RP>
__device__ __forceinline__ void store_acc_rows(uint32_t taddr, float* dst_row, bool row_ok) {
#pragma unroll
    for (int c = 0; c < RP / 16; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + 16u * (uint32_t)c, v);
        tmem_ld_wait();
        if (row_ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_v4(dst_row + 16 * c + 4 * j, make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
    }
}

// Grid: strips (128 rows of dW each) x splits (kts K tiles each).
// part_a [strips][k][RP] (dA^T partials), part_b [splits][n][RP].
template <int RP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
lora_grads_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                  const uint16_t* __restrict__ lora_b, int64_t n, int64_t k, int r, int splits, int kts,
                  float* __restrict__ part_a, float* __restrict__ part_b, uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    Smem<RP>& sm = *reinterpret_cast<Smem<RP>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int STAGES = Smem<RP>::ST;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int strip = (int)blockIdx.x / splits, split = (int)blockIdx.x - strip * splits;
    const int64_t n0 = (int64_t)strip * TK;
    const int KT_all = (int)((k + TK - 1) / TK);
    const int kt0 = split * kts, kt1 = min(KT_all, kt0 + kts);
    const int KT = kt1 - kt0;                     // >= 1 by the launcher's choice
    constexpr uint32_t A_BOX = RP * 128;          // one 64-column box of A's tile (and of B^T)
    constexpr uint32_t TMEM_COLS = (3 * RP <= 32) ? 32 : (3 * RP <= 64) ? 64 : (3 * RP <= 128) ? 128 : 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.da_full[b], 1);
            mbar_init(&sm.da_empty[b], 4);
        }
        mbar_init(&sm.db_full, 1);
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
    const uint32_t t_db = tmem, t_da0 = tmem + RP;
    pdl_wait();       // dW (and possibly the factors) come from preceding grids

    if (warp != 0) {
        // B^T of the strip, K-major with the 128-byte swizzle: row j (rank),
        // K = the strip's rows nn (two boxes of 64); ranks past r and rows
        // past n zero.  Warps 1-7 build it while warp 0 already streams dW;
        // the MMA warp waits for it on a named barrier of these 224 threads.
        // A 16-byte chunk is 8 ranks of one row of B (r is a multiple of 8).
        constexpr int kChunks = RP * TK / 8, kPer = (kChunks + 223) / 224;
        const int t = (int)threadIdx.x - 32;
        uint4 v[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int c = t + 224 * i, nn = c / (RP / 8), j0 = 8 * (c % (RP / 8));
            v[i] = (c < kChunks && j0 < r && n0 + nn < n)
                       ? *reinterpret_cast<const uint4*>(lora_b + (n0 + nn) * r + j0) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int c = t + 224 * i, nn = c / (RP / 8), j0 = 8 * (c % (RP / 8));
            if (c < kChunks) {
                const uint32_t wv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                const uint32_t base = (uint32_t)(nn / 64) * A_BOX + 2u * (uint32_t)(nn % 8);
#pragma unroll
                for (int h = 0; h < 8; ++h)
                    *reinterpret_cast<uint16_t*>(sm.bt + base + sw128_offset(j0 + h, (nn % 64) / 8)) =
                        (uint16_t)((h & 1) ? (wv[h >> 1] >> 16) : (wv[h >> 1] & 0xFFFFu));
            }
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 224;" ::: "memory");
    }

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmA);
            for (int i = 0; i < KT; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                if (!wait_or_timeout(&sm.empty[s], ph ^ 1u, err)) break;
                mbar_arrive_expect_tx(&sm.full[s], DW_TILE + 2 * A_BOX);
                const int32_t kk = (kt0 + i) * TK;
                tma_load_2d(sm.dw[s], &tmW, &sm.full[s], kk, (int32_t)n0);
                tma_load_2d(sm.dw[s] + DW_BOX, &tmW, &sm.full[s], kk + 64, (int32_t)n0);
                tma_load_2d(sm.a[s], &tmA, &sm.full[s], kk, 0);
                tma_load_2d(sm.a[s] + A_BOX, &tmA, &sm.full[s], kk + 64, 0);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t id_db = idesc_bf16(TK, RP, false, false);
            const uint32_t id_da = idesc_bf16(TK, RP, true, false);
            const uint32_t bt_base = smem_u32(sm.bt);
            bool ok = true;
            for (int i = 0; i < KT && ok; ++i) {
                const int s = i % STAGES, b = i & 1;
                const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
                if (!wait_or_timeout(&sm.full[s], ph, err) ||
                    !wait_or_timeout(&sm.da_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t w_base = smem_u32(sm.dw[s]), a_base = smem_u32(sm.a[s]);
#pragma unroll
                for (int q = 0; q < TK / 16; ++q) {
                    // dB: K step q = columns 16q .. 16q + 15 of the tile (box q / 4, 32 bytes per step)
                    const uint32_t ko = (uint32_t)(q / 4) * DW_BOX + 32u * (uint32_t)(q % 4);
                    mma_bf16(t_db, desc_kmajor_sw128(w_base + ko),
                             desc_kmajor_sw128(a_base + (uint32_t)(q / 4) * A_BOX + 32u * (uint32_t)(q % 4)), id_db,
                             (i > 0 || q > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int q = 0; q < TK / 16; ++q) {
                    // dA^T: K step q = rows 16q .. 16q + 15 of the tile (2 KB per step); M = the
                    // tile's columns in two 64-column blocks 16 KB apart
                    mma_bf16(t_da0 + (uint32_t)(b * RP), smem_desc(w_base + 2048u * (uint32_t)q, DW_BOX, 1024, kLayoutSw128),
                             desc_kmajor_sw128(bt_base + (uint32_t)(q / 4) * A_BOX + 32u * (uint32_t)(q % 4)), id_da,
                             q > 0 ? 1u : 0u);
                }
                mma_commit(&sm.empty[s]);
                mma_commit(&sm.da_full[b]);
            }
            if (ok) mma_commit(&sm.db_full);
        }
    } else if (warp >= EPI_WARP0) {
        // ---------------------------------------------------------- epilogue
        const int qd = warp & 3;                  // TMEM lane quadrant
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        bool ok = true;
        for (int i = 0; i < KT && ok; ++i) {
            const int b = i & 1;
            if (!__all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.da_full[b], (uint32_t)(i >> 1) & 1u, err))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int64_t col = (int64_t)(kt0 + i) * TK + 32 * qd + lane;        // a column of dW = a k of dA
            store_acc_rows<RP>(t_da0 + (uint32_t)(b * RP) + lane_off,
                               part_a + ((int64_t)strip * k + col) * RP, col < k);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.da_empty[b]);
        }
        if (ok && __all_sync(0xFFFFFFFFu, wait_or_timeout(&sm.db_full, 0, err))) {
            tc_fence_after();
            const int64_t row = n0 + 32 * qd + lane;
            store_acc_rows<RP>(t_db + lane_off, part_b + ((int64_t)split * n + row) * RP, row < n);
        }
    }

    __syncwarp();     // the role warps' other lanes wait here for the elected lane, without polling
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// sum_s p[s * stride + 0..3] for s = 0 .. S-1, added in s order; the
// partial vectors are loaded eight at a time so their L2 round trips overlap
__device__ __forceinline__ float4 ordered_sum4(const float* p, int64_t stride, int S) {
    float4 acc = __ldcg(reinterpret_cast<const float4*>(p));
    for (int s0 = 1; s0 < S; s0 += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (s0 + u < S) v[u] = __ldcg(reinterpret_cast<const float4*>(p + (int64_t)(s0 + u) * stride));
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (s0 + u < S) {
                acc.x = __fadd_rn(acc.x, v[u].x);
                acc.y = __fadd_rn(acc.y, v[u].y);
                acc.z = __fadd_rn(acc.z, v[u].z);
                acc.w = __fadd_rn(acc.w, v[u].w);
            }
    }
    return acc;
}

// dA[j][c] = bf16(alpha * sum_s part_a[s][c][j]) and dB[row][j] =
// bf16(alpha * sum_s part_b[s][row][j]), s ascending; one thread per four
// consecutive ranks of one column of dA or one row of dB (r is a multiple
// of 8, rows of the partials are rp floats, rp a multiple of 16).
__global__ void __launch_bounds__(256)
lora_grads_reduce_kernel(const float* __restrict__ part_a, const float* __restrict__ part_b, int strips,
                         int splits, int64_t n, int64_t k, int r, int rp, float alpha, uint16_t* __restrict__ da,
                         uint16_t* __restrict__ db) {
    pdl_trigger();
    pdl_wait();
    const int rq = r / 4;
    const int64_t na = k * rq, total = na + n * rq;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (int64_t)gridDim.x * 256) {
        if (i < na) {
            const int64_t c = i / rq;
            const int j = 4 * (int)(i - c * rq);
            const float4 a = ordered_sum4(part_a + c * rp + j, k * rp, strips);
            da[(int64_t)j * k + c] = (uint16_t)f32_to_bf16(__fmul_rn(a.x, alpha));
            da[(int64_t)(j + 1) * k + c] = (uint16_t)f32_to_bf16(__fmul_rn(a.y, alpha));
            da[(int64_t)(j + 2) * k + c] = (uint16_t)f32_to_bf16(__fmul_rn(a.z, alpha));
            da[(int64_t)(j + 3) * k + c] = (uint16_t)f32_to_bf16(__fmul_rn(a.w, alpha));
        } else {
            const int64_t e = i - na, row = e / rq;
            const int j = 4 * (int)(e - row * rq);
            const float4 b = ordered_sum4(part_b + row * rp + j, n * rp, splits);
            *reinterpret_cast<uint2*>(db + row * r + j) =
                make_uint2(f32x2_to_bf16x2(__fmul_rn(b.x, alpha), __fmul_rn(b.y, alpha)),
                           f32x2_to_bf16x2(__fmul_rn(b.z, alpha), __fmul_rn(b.w, alpha)));
        }
    }
}

template <int RP>
int smem_bytes() { return (int)sizeof(Smem<RP>) + 1024; }

inline int pad16(int r) { return (r + 15) / 16 * 16; }

struct Plan {
    int strips, splits, kts;
};
Plan plan(int64_t n, int64_t k, int sms) {
    Plan p;
    p.strips = (int)((n + TK - 1) / TK);
    const int kt = (int)((k + TK - 1) / TK);
    int s = (int)max64(1, min64(kt, (int64_t)(sms > 0 ? sms : 1) / p.strips));
    p.kts = (kt + s - 1) / s;
    p.splits = (kt + p.kts - 1) / p.kts;            // every split non-empty
    return p;
}

template <int RP>
cudaError_t launch_rp(const void* dw, const void* a, const void* b, int64_t n, int64_t k, int r, float alpha,
                      void* da, void* db, void* ws, uint32_t* err, int sms, cudaStream_t st) {
    static int configured[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(lora_grads_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem_bytes<RP>());
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    const Plan p = plan(n, k, sms);
    CUtensorMap tw, ta;
    e = make_tmap_2d(&tw, dw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)n, (uint64_t)k, (uint64_t)k * 2, TK, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)r, (uint64_t)k, (uint64_t)k * 2, RP, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    float* part_a = static_cast<float*>(ws);
    float* part_b = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                             ((size_t)p.strips * (size_t)k * RP * 4 + 255) / 256 * 256);
    e = launch_pdl(lora_grads_kernel<RP>, dim3((unsigned)(p.strips * p.splits)), dim3(NUM_THREADS),
                   smem_bytes<RP>(), st, tw, ta, (const uint16_t*)b, n, k, r, p.splits, p.kts, part_a, part_b, err);
    if (e != cudaSuccess) return e;
    const int64_t total = (n + k) * (r / 4);
    const int grid = (int)min64((total + 255) / 256, (int64_t)(sms > 0 ? sms : 1) * 8);
    return launch_pdl(lora_grads_reduce_kernel, dim3((unsigned)grid), dim3(256), 0, st, (const float*)part_a,
                      (const float*)part_b, p.strips, p.splits, n, k, r, RP, alpha, (uint16_t*)da, (uint16_t*)db);
}

}  // namespace

bool lora_grads_fused(int64_t r) { return r >= 1 && r <= MAX_RP; }

size_t lora_grads_workspace_bytes(int64_t n, int64_t k, int64_t r, int sms) {
    if (!lora_grads_fused(r)) return 0;
    const Plan p = plan(n, k, sms);
    const size_t rp = (size_t)pad16((int)r);
    return ((size_t)p.strips * (size_t)k * rp * 4 + 255) / 256 * 256 + (size_t)p.splits * (size_t)n * rp * 4;
}

cudaError_t launch_lora_grads(const void* dw, const void* lora_a, const void* lora_b, int64_t n, int64_t k, int r,
                              float alpha_over_r, void* da, void* db, void* workspace, uint32_t* err, int sms,
                              cudaStream_t st) {
    switch (pad16(r)) {
    case 16: return launch_rp<16>(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, err, sms, st);
    case 32: return launch_rp<32>(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, err, sms, st);
    case 48: return launch_rp<48>(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, err, sms, st);
    case 64: return launch_rp<64>(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, err, sms, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace fpq
