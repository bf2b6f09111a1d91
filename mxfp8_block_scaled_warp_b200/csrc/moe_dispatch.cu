// moe_dispatch.cu -- the FP8 MoE dispatch ("DeepSeek-V3 Blog 5: Low-Precision
// Training", Reducing Communication Overhead in MoE with FP8: token
// activations are quantized to FP8 before they are sent to the GPUs that
// hold their experts).  Format: MXFP8 (E4M3 codes, E8M0 scale per 32), the
// input of the grouped expert GEMM.
//
// Order of the rows (the page fixes none): a receiving rank holds its local
// experts' rows in expert order; each expert's rows come from source rank 0,
// 1, ... in turn; from one source, the (token, choice) pairs routed to that
// expert in token order, then choice order.  A pair's index among its
// source's pairs of the same expert is its slot.
//
// Three steps on the source rank:
//   1. route: per-chunk expert histograms (a chunk is a run of consecutive
//      tokens handled by one warp), then per expert an exclusive scan over
//      the chunks: the slot of a chunk's first pair of each expert, and the
//      per-expert counts that the ranks exchange.
//   2. layout: from every rank's counts, the row of slot 0 of each expert in
//      its destination buffer (a receiver's expert-grouped buffer, or this
//      rank's own expert-major send buffer), and this rank's group offsets.
//   3. dispatch: one warp per chunk reads each token row once, quantizes it
//      to MXFP8 and stores codes and scales to each of its top-k
//      destinations (pointers per destination rank: local memory, or a
//      peer's memory mapped into this process).
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "quant_unit.cuh"

namespace fpq {

namespace {

constexpr int kWarps = 8;                 // warps per CTA of the count and dispatch kernels
constexpr int kDispatchUnits = 7;         // units per lane in flight per batch (a 7168 row: 2 batches)

// pairs of chunk c: tokens [c tpc, min(T, (c + 1) tpc)) x topk choices
__global__ void __launch_bounds__(32 * kWarps)
moe_count_kernel(const int32_t* __restrict__ ids, int64_t tokens, int topk, int experts, int64_t tpc,
                 int64_t chunks, int32_t* __restrict__ hist, uint32_t* err) {
    extern __shared__ int32_t sh[];                         // [kWarps][experts]
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* h = sh + warp * experts;
    for (int e = lane; e < experts; e += 32) h[e] = 0;
    __syncwarp();
    pdl_wait();
    const int64_t c = (int64_t)blockIdx.x * kWarps + warp;
    if (c >= chunks) return;
    const int64_t p0 = c * tpc * topk, p1 = min64(tokens, (c + 1) * tpc) * topk;
    for (int64_t p = p0 + lane; p < p1; p += 32) {
        const int e = ids[p];
        if (e < 0 || e >= experts) {
            raise_device_error(err, FPQ_ERR_DEVICE_BAD_INPUT);
            continue;
        }
        atomicAdd(&h[e], 1);
    }
    __syncwarp();
    for (int e = lane; e < experts; e += 32) hist[(int64_t)e * chunks + c] = h[e];
}

// One CTA per expert: base[e][c] = sum of hist[e][c'] over c' < c, and
// counts[e] = the total.  Thread i owns a contiguous run of chunks.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
moe_scan_kernel(const int32_t* __restrict__ hist, int64_t chunks, int32_t* __restrict__ base,
                int32_t* __restrict__ counts) {
    __shared__ int32_t warp_tot[kScanThreads / 32];
    pdl_trigger();
    pdl_wait();
    const int e = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t per = (chunks + kScanThreads - 1) / kScanThreads;
    const int64_t c0 = min64(chunks, t * per), c1 = min64(chunks, c0 + per);
    const int32_t* hrow = hist + (int64_t)e * chunks;
    int32_t mine = 0;
    for (int64_t c = c0; c < c1; ++c) mine += hrow[c];
    // exclusive scan of `mine` over the block
    int32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = warp_tot[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;                             // exclusive over warps
        if (lane == 31) counts[e] = wi;
    }
    __syncthreads();
    int32_t run = warp_tot[warp] + incl - mine;
    int32_t* brow = base + (int64_t)e * chunks;
    for (int64_t c = c0; c < c1; ++c) {
        brow[c] = run;
        run += hrow[c];
    }
}

// One CTA; thread e per expert.  counts_all [world][experts].
//   DIRECT: dst_row0[e] = rows of experts before e on e's rank (all sources)
//           + rows of e from sources before `rank`.
//   PACK:   dst_row0[e] = rows of this rank's experts before e.
//   recv_offsets[l] (l = 0 .. L): rows of this rank's local experts before l.
__global__ void __launch_bounds__(1024)
moe_layout_kernel(const int32_t* __restrict__ counts_all, int world, int experts, int rank, int pack,
                  int64_t* __restrict__ dst_row0, int32_t* __restrict__ recv_offsets) {
    extern __shared__ int64_t tot[];                        // [experts]: rows of e over all sources
    pdl_trigger();
    pdl_wait();
    const int L = experts / world;
    for (int e = threadIdx.x; e < experts; e += blockDim.x) {
        int64_t s = 0;
        for (int r = 0; r < world; ++r) s += counts_all[(int64_t)r * experts + e];
        tot[e] = s;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < experts; e += blockDim.x) {
        int64_t row = 0;
        if (pack) {
            for (int f = 0; f < e; ++f) row += counts_all[(int64_t)rank * experts + f];
        } else {
            const int first = (e / L) * L;
            for (int f = first; f < e; ++f) row += tot[f];
            for (int r = 0; r < rank; ++r) row += counts_all[(int64_t)r * experts + e];
        }
        dst_row0[e] = row;
    }
    for (int l = threadIdx.x; l <= L; l += blockDim.x) {
        int64_t row = 0;
        for (int f = rank * L; f < rank * L + l; ++f) row += tot[f];
        recv_offsets[l] = (int32_t)row;
    }
}

// One warp per chunk.  Per token: lane j < topk computes choice j's
// destination (rank d = e / experts_per_dest, row dst_row0[e] + slot) and the
// row pointers there; then the row is quantized in batches of 32 x
// kDispatchUnits units and every batch is stored to all topk destinations.
// Slots advance in token order, then choice order, from the chunk's bases.
__global__ void __launch_bounds__(32 * kWarps)
moe_dispatch_mxfp8_kernel(const uint4* __restrict__ x, int64_t tokens, int64_t hidden,
                          const int32_t* __restrict__ ids, int topk, int experts, const int32_t* __restrict__ base,
                          int64_t tpc, int64_t chunks, const int64_t* __restrict__ dst_row0, int experts_per_dest,
                          uint8_t* const* __restrict__ dst_codes, uint8_t* const* __restrict__ dst_scales,
                          const int64_t* __restrict__ dst_capacity, uint32_t* err) {
    extern __shared__ int32_t sh[];                         // [kWarps][experts] running slots
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c = (int64_t)blockIdx.x * kWarps + warp;
    if (c >= chunks) return;
    int32_t* run = sh + warp * experts;
    for (int e = lane; e < experts; e += 32) run[e] = base[(int64_t)e * chunks + c];
    __syncwarp();
    const int64_t units_row = hidden / 16;                  // even: hidden is a multiple of 32
    const int64_t t1 = min64(tokens, (c + 1) * tpc);
    for (int64_t t = c * tpc; t < t1; ++t) {
        // destinations of the token's choices, choice j in lane j
        uint8_t* qdst = nullptr;
        uint8_t* sdst = nullptr;
        int e_l = lane < topk ? ids[t * topk + lane] : -1;
        bool ok_l = e_l >= 0 && e_l < experts;
        for (int j = 0; j < topk; ++j) {                     // slots in choice order
            const int e = __shfl_sync(0xFFFFFFFFu, e_l, j);
            const bool ok = __shfl_sync(0xFFFFFFFFu, ok_l, j);
            int32_t slot = 0;
            if (ok) {
                slot = run[e];
                __syncwarp();
                if (lane == 0) run[e] = slot + 1;
                __syncwarp();
            }
            if (lane == j && ok) {
                const int d = e / experts_per_dest;
                const int64_t row = dst_row0[e] + slot;
                if (row < 0 || row >= dst_capacity[d]) {
                    raise_device_error(err, FPQ_ERR_DEVICE_BAD_INPUT);
                    ok_l = false;
                } else {
                    qdst = dst_codes[d] + row * hidden;
                    sdst = dst_scales[d] + row * (hidden / 32);
                }
            }
        }
        if (!ok_l) qdst = nullptr;
        const uint4* xrow = x + t * (hidden / 8);
        for (int64_t u0 = 0; u0 < units_row; u0 += 32 * kDispatchUnits) {
            Unit v[kDispatchUnits];
#pragma unroll
            for (int i = 0; i < kDispatchUnits; ++i) {
                const int64_t u = u0 + 32 * i + lane;
                if (u < units_row) v[i] = load_unit(xrow, u);
            }
            uint4 q[kDispatchUnits];
            uint32_t sc[kDispatchUnits];
#pragma unroll
            for (int i = 0; i < kDispatchUnits; ++i) {
                const int64_t u = u0 + 32 * i + lane;
                // lanes 2i and 2i + 1 are in or out of the row together (units_row is even)
                const uint32_t a = group_max<2>(u < units_row ? unit_absmax(v[i]) : 0u);
                const int e = mx_exponent(a);
                q[i] = (e == 128) ? make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu)
                                  : scale_to_e4m3(v[i], pow2_neg(e));
                sc[i] = (uint32_t)(e + 127);
            }
            for (int j = 0; j < topk; ++j) {
                uint8_t* qd = (uint8_t*)__shfl_sync(0xFFFFFFFFu, (unsigned long long)qdst, j);
                uint8_t* sd = (uint8_t*)__shfl_sync(0xFFFFFFFFu, (unsigned long long)sdst, j);
                if (qd == nullptr) continue;                 // uniform over the warp
#pragma unroll
                for (int i = 0; i < kDispatchUnits; ++i) {
                    const int64_t u = u0 + 32 * i + lane;
                    if (u < units_row) {
                        st_v4(qd + 16 * u, q[i]);
                        if ((u & 1) == 0) sd[u >> 1] = (uint8_t)sc[i];
                    }
                }
            }
        }
    }
}

// Regroup (the receiving side of a rank-to-rank exchange): rows that
// arrived source-major -- all of source 0's rows for this rank's experts,
// expert-major in slot order, then source 1's, ... -- into the receive
// layout (expert-major; within an expert, source 0, 1, ...).  Segment
// (l, s) of C[s][rank L + l] rows moves from
//   src = sum_{s' < s, l'} C[s'][rank L + l'] + sum_{l' < l} C[s][rank L + l']
// to
//   dst = sum_{l' < l, s'} C[s'][rank L + l'] + sum_{s' < s} C[s'][rank L + l].
// One column of CTAs per segment (blockIdx.y = l world + s), warp 0 works out
// the segment's rows and starts; then each warp copies one row at a time
// (codes, then its E8M0 scales) with 16-byte vectors.  Negative counts or a
// segment outside `rows` are reported and not copied.
__global__ void __launch_bounds__(32 * kWarps)
moe_regroup_kernel(const uint8_t* __restrict__ src_q, const uint8_t* __restrict__ src_s,
                   const int32_t* __restrict__ counts_all, int world, int experts, int rank, int64_t hidden,
                   int64_t rows, uint8_t* __restrict__ dst_q, uint8_t* __restrict__ dst_s, uint32_t* err) {
    __shared__ int64_t seg[3];      // rows, src start, dst start (-1 rows: malformed)
    const int L = experts / world;
    const int l = (int)blockIdx.y / world, s = (int)blockIdx.y - l * world;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t* c = counts_all;
    const int e0 = rank * L;
    if (warp == 0) {
        int64_t src = 0, dst = 0;
        bool bad = false;
        for (int i = lane; i < s * L; i += 32) {           // sources before s, all local experts
            const int32_t v = c[(int64_t)(i / L) * experts + e0 + i % L];
            bad |= v < 0;
            src += v;
        }
        for (int i = lane; i < l; i += 32) src += c[(int64_t)s * experts + e0 + i];
        for (int i = lane; i < l * world; i += 32) {       // local experts before l, all sources
            const int32_t v = c[(int64_t)(i % world) * experts + e0 + i / world];
            bad |= v < 0;
            dst += v;
        }
        for (int i = lane; i < s; i += 32) dst += c[(int64_t)i * experts + e0 + l];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            src += __shfl_xor_sync(0xFFFFFFFFu, src, o);
            dst += __shfl_xor_sync(0xFFFFFFFFu, dst, o);
        }
        bad = __any_sync(0xFFFFFFFFu, bad);
        if (lane == 0) {
            const int64_t n = c[(int64_t)s * experts + e0 + l];
            if (bad || n < 0 || src + n > rows || dst + n > rows) {
                if (blockIdx.x == 0) raise_device_error(err, FPQ_ERR_DEVICE_BAD_INPUT);
                seg[0] = -1;
            } else {
                seg[0] = n;
            }
            seg[1] = src;
            seg[2] = dst;
        }
    }
    __syncthreads();
    const int64_t n = seg[0], src = seg[1], dst = seg[2];
    if (n <= 0) return;
    const int64_t sbytes = hidden / 32;
    const bool svec = (sbytes % 16) == 0;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < n; r += (int64_t)gridDim.x * kWarps) {
        const uint4* qs = reinterpret_cast<const uint4*>(src_q + (src + r) * hidden);
        uint4* qd = reinterpret_cast<uint4*>(dst_q + (dst + r) * hidden);
        for (int64_t v = lane; v < hidden / 16; v += 32) st_v4(qd + v, ld_stream(qs + v));
        const uint8_t* ss = src_s + (src + r) * sbytes;
        uint8_t* sd = dst_s + (dst + r) * sbytes;
        if (svec) {
            for (int64_t v = lane; v < sbytes / 16; v += 32)
                *reinterpret_cast<uint4*>(sd + 16 * v) = *reinterpret_cast<const uint4*>(ss + 16 * v);
        } else {
            for (int64_t v = lane; v < sbytes; v += 32) sd[v] = ss[v];
        }
    }
}

}  // namespace

int64_t moe_tokens_per_chunk(int64_t tokens) { return max64(1, (tokens + 4735) / 4736); }

int64_t moe_chunks(int64_t tokens) {
    const int64_t tpc = moe_tokens_per_chunk(tokens);
    return (tokens + tpc - 1) / tpc;
}

size_t moe_route_workspace_bytes(int64_t tokens, int experts) {
    return 2 * (size_t)experts * (size_t)max64(1, moe_chunks(tokens)) * sizeof(int32_t);
}

cudaError_t launch_moe_route(const int32_t* ids, int64_t tokens, int topk, int experts, int32_t* counts,
                             void* workspace, uint32_t* err, cudaStream_t st) {
    const int64_t tpc = moe_tokens_per_chunk(tokens), chunks = moe_chunks(tokens);
    int32_t* hist = static_cast<int32_t*>(workspace);
    int32_t* base = hist + (size_t)experts * (size_t)max64(1, chunks);
    cudaError_t e;
    if (chunks > 0) {
        const int smem = kWarps * experts * (int)sizeof(int32_t);
        e = launch_pdl(moe_count_kernel, dim3((unsigned)((chunks + kWarps - 1) / kWarps)), dim3(32 * kWarps), smem, st,
                       ids, tokens, topk, experts, tpc, chunks, hist, err);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(moe_scan_kernel, dim3((unsigned)experts), dim3(kScanThreads), 0, st, (const int32_t*)hist,
                      chunks, base, counts);
}

cudaError_t launch_moe_layout(const int32_t* counts_all, int world, int experts, int rank, int pack,
                              int64_t* dst_row0, int32_t* recv_offsets, cudaStream_t st) {
    return launch_pdl(moe_layout_kernel, dim3(1), dim3(1024), experts * (int)sizeof(int64_t), st, counts_all, world,
                      experts, rank, pack, dst_row0, recv_offsets);
}

cudaError_t launch_moe_dispatch_mxfp8(const void* x, int64_t tokens, int64_t hidden, const int32_t* ids, int topk,
                                      int experts, const void* workspace, const int64_t* dst_row0, int n_dest,
                                      void* const* dst_codes, void* const* dst_scales, const int64_t* dst_capacity,
                                      uint32_t* err, cudaStream_t st) {
    const int64_t tpc = moe_tokens_per_chunk(tokens), chunks = moe_chunks(tokens);
    if (chunks == 0) return cudaSuccess;
    const int32_t* base = static_cast<const int32_t*>(workspace) + (size_t)experts * (size_t)chunks;
    const int smem = kWarps * experts * (int)sizeof(int32_t);
    return launch_pdl(moe_dispatch_mxfp8_kernel, dim3((unsigned)((chunks + kWarps - 1) / kWarps)), dim3(32 * kWarps),
                      smem, st, (const uint4*)x, tokens, hidden, ids, topk, experts, base, tpc, chunks, dst_row0,
                      experts / n_dest, (uint8_t* const*)dst_codes, (uint8_t* const*)dst_scales, dst_capacity, err);
}

cudaError_t launch_moe_regroup(const void* src_q, const void* src_s, const int32_t* counts_all, int world,
                               int experts, int rank, int64_t hidden, int64_t rows, void* dst_q, void* dst_s,
                               uint32_t* err, int sms, cudaStream_t st) {
    // about four CTAs per SM over all segments (experts / world * world = experts of them)
    const int gx = (int)max64(1, min64(65535, (int64_t)4 * (sms > 0 ? sms : 1) / experts));
    moe_regroup_kernel<<<dim3((unsigned)gx, (unsigned)experts), 32 * kWarps, 0, st>>>(
        (const uint8_t*)src_q, (const uint8_t*)src_s, counts_all, world, experts, rank, hidden, rows,
        (uint8_t*)dst_q, (uint8_t*)dst_s, err);
    return cudaGetLastError();
}

}  // namespace fpq
