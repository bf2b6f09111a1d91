// quant_kernels.cu -- block quantize / dequantize kernels for sm_100a.
//
// Every kernel here streams HBM: 16-byte vector loads, several independent
// loads in flight per thread (an unrolled grid-stride loop), absmax of a
// block reduced with warp shuffles, packed hardware conversion to E4M3 or
// E2M1, and 8/16-byte stores with the scales written alongside.
//
// Work unit: 16 consecutive bf16 elements of a row (32 bytes), held by one
// lane as eight 32-bit words.  A block of the format is 2 units (MXFP8 1x32),
// 8 units (1x128) or 1 unit (NVFP4 1x16); because every row length is a
// multiple of the block, blocks never straddle rows and a flat unit index
// addresses both the data and the row-major scale arrays.  Each streaming
// kernel also has a strided instance (template flag S): data and codes then
// live at row and batch strides, the flat unit index is mapped to (matrix,
// row, column unit) once per unit, and the scales stay dense.
#include <cuda_fp16.h>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "quant_unit.cuh"
#include "tma_host.h"

namespace fpq {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;   // units in flight per thread

__device__ __forceinline__ Unit load_unit_hint(const uint4* x, int64_t u, uint64_t pol) {
    uint4 a = ld_stream_hint(x + 2 * u, pol), b = ld_stream_hint(x + 2 * u + 1, pol);
    return Unit{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}

// E4M3 codes of fp32(x / s) for the 16 elements of a unit.
__device__ __forceinline__ uint4 divide_to_e4m3(const Unit& v, float s) {
    uint32_t c[8];
    if (reciprocal_ok(s)) {
        const QuotientBracket br = quotient_bracket(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = e4m3x2_of_quotients(bf16_lo(v.w[i]), bf16_hi(v.w[i]), br);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            c[i] = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(v.w[i]), s), __fdiv_rn(bf16_hi(v.w[i]), s));
    }
    return make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16), c[6] | (c[7] << 16));
}

// fp32 block scale s = fp32(amax / 448), 1 for an all-zero block.
__device__ __forceinline__ float fp32_scale(uint32_t a) {
    return a == 0 ? 1.0f : __fdiv_rn(__uint_as_float(a << 16), 448.0f);
}

// ----------------------------------------------------------------- MXFP8

template <bool S>
__global__ void __launch_bounds__(kThreads, 3)
quant_mxfp8_kernel(const uint4* __restrict__ x, uint4* __restrict__ q, uint8_t* __restrict__ s,
                   int64_t units, UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    const int64_t stride = (int64_t)gridDim.x * kThreads * kUnroll;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kUnroll; base < units; base += stride) {
        Unit v[kUnroll];
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            int64_t u = base + i * kThreads + threadIdx.x;
            if (u < units) v[i] = load_unit(x, in_unit<S>(m, u));
        }
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            int64_t u = base + i * kThreads + threadIdx.x;
            // both lanes of a block are in range or out of range together
            // (units is even), so the shuffle below is uniform per pair
            uint32_t a = group_max<2>(u < units ? unit_absmax(v[i]) : 0u);
            if (u >= units) continue;
            int e = mx_exponent(a);
            uint4 out;
            if (e == 128) out = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            else out = scale_to_e4m3(v[i], pow2_neg(e));
            st_v4(q + out_unit<S>(m, u), out);
            if ((u & 1) == 0) s[u >> 1] = (uint8_t)(e + 127);
        }
    }
}

// ----------------------------------------------------------------- FP8 1x128

// One unit per thread per iteration, with the next iteration's unit loaded
// before this one is encoded; few registers let six CTAs share an SM, and
// the grid is sized to exactly that residency (grid-stride loop).
constexpr int Q1_MIN_BLOCKS = 6;

template <bool S>
__global__ void __launch_bounds__(kThreads, Q1_MIN_BLOCKS)
quant_fp8_1x128_kernel(const uint4* __restrict__ x, uint4* __restrict__ q,
                       float* __restrict__ s, int64_t units, UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    __shared__ ScaleTables tab;                      // s = fp32(amax / 448) and its bracket, by mantissa
    init_scale_tables(tab, 448.0f);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    Unit cur;
    if (u < units) cur = load_unit(x, in_unit<S>(m, u));
    __syncthreads();
    // The 8 lanes of a block are in range or out of range together (units
    // and stride are multiples of 8), so the shuffles stay converged.
    for (; u - threadIdx.x < units; u += stride) {
        Unit nxt;
        if (u + stride < units) nxt = load_unit(x, in_unit<S>(m, u + stride));
        const uint32_t a = group_max<8>(u < units ? unit_absmax(cur) : 0u);
        if (u < units) {
            // exponent field >= 10 keeps s = fp32(amax / 448) and 1/s normal
            float sc, lo, hi;
            uint4 out;
            if (table_scale(tab, a, 10, sc, lo, hi)) {
                const QuotientBracket br{sc, lo, hi};
                uint32_t c[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) c[j] = e4m3x2_of_quotients(bf16_lo(cur.w[j]), bf16_hi(cur.w[j]), br);
                out = make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16), c[6] | (c[7] << 16));
            } else {
                sc = fp32_scale(a);
                out = divide_to_e4m3(cur, sc);
            }
            st_v4(q + out_unit<S>(m, u), out);
            if ((u & 7) == 0) s[u >> 3] = sc;
        }
        cur = nxt;
    }
}

// ----------------------------------------------------------------- FP8 128x128

// One CTA of QB_THREADS threads per 128x128 block (grid = all blocks of all
// batch items).  Thread t owns the QB_CHUNKS 16-byte chunks c = t +
// QB_THREADS i of the block (row c / 16, columns 8 (c % 16)) and issues all
// their loads before using any.  Few chunks per thread keep many warps
// resident, which hides the latency of the encoder's dependent steps.  One
// barrier: each warp publishes its absmax, then every thread combines them
// and derives the same scale.  Rows past the end of a batch item (a short
// last block row) read as zero and are not stored.
constexpr int QB_THREADS = 512;
constexpr int QB_CHUNKS = 128 * 16 / QB_THREADS;
constexpr int QB_WARPS = QB_THREADS / 32;

// S: strided operands (row and batch strides in elements); dense otherwise.
template <bool S>
__global__ void __launch_bounds__(QB_THREADS, 2048 / QB_THREADS)
quant_fp8_128x128_kernel(const uint8_t* __restrict__ x, uint8_t* __restrict__ q, float* __restrict__ s,
                         int64_t rows, int64_t cols, int64_t ldx, int64_t bsx, int64_t ldq, int64_t bsq) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    __shared__ uint32_t red[QB_WARPS];
    const int64_t nbr = (rows + 127) / 128, nbc = cols / 128;
    const int64_t idx = blockIdx.x;
    const int64_t bj = idx % nbc, t2 = idx / nbc, bi = t2 % nbr, b = t2 / nbr;
    const int rmax = (int)min64(128, rows - bi * 128);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = b * rows + bi * 128;
    if (!S) ldx = ldq = cols;
    const uint8_t* xb = S ? x + (b * bsx + bi * 128 * ldx + bj * 128) * 2 : x + (row0 * cols + bj * 128) * 2;
    uint4 v[QB_CHUNKS];
#pragma unroll
    for (int i = 0; i < QB_CHUNKS; ++i) {
        const int c = threadIdx.x + QB_THREADS * i, r = c >> 4;
        v[i] = r < rmax ? ld_stream(xb + (int64_t)r * ldx * 2 + (c & 15) * 16) : make_uint4(0, 0, 0, 0);
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < QB_CHUNKS; ++i)
        m = max2(m, max2(max2(abs2(v[i].x), abs2(v[i].y)), max2(abs2(v[i].z), abs2(v[i].w))));
    m = group_max<32>(hmax2(m));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint32_t a = red[0];
#pragma unroll
    for (int w = 1; w < QB_WARPS; ++w) a = max(a, red[w]);
    const float sc = fp32_scale(a);
    if (threadIdx.x == 0) s[idx] = sc;
    const bool fast = reciprocal_ok(sc);
    const QuotientBracket br = quotient_bracket(fast ? sc : 1.0f);
    uint8_t* qb = S ? q + b * bsq + bi * 128 * ldq + bj * 128 : q + row0 * cols + bj * 128;
#pragma unroll
    for (int i = 0; i < QB_CHUNKS; ++i) {
        const int c = threadIdx.x + QB_THREADS * i, r = c >> 4, c8 = (c & 15) * 8;
        if (r < rmax) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            uint32_t e[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                e[j] = fast ? e4m3x2_of_quotients(bf16_lo(w[j]), bf16_hi(w[j]), br)
                            : f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[j]), sc), __fdiv_rn(bf16_hi(w[j]), sc));
            st_v2(qb + (int64_t)r * ldq + c8, make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16)));
        }
    }
}

// ----------------------------------------------------------------- NVFP4
//
// One persistent kernel per call.  The per-tensor scale g needs the amax of
// the whole matrix before any block of it can be encoded, so every matrix
// is read twice: once for its amax ("A" tiles) and once to encode it ("B"
// tiles).  Work items (tiles of 256 x upt units: 128 KB of input at the
// largest upt) are handed out
// from a global counter in the order (lookahead LA = NV_LOOKAHEAD)
//   A(0), ..., A(LA-1), A(LA), B(0), A(LA+1), B(1), ..., A(n-1), B(n-1-LA), B(n-LA), ..., B(n-1)
// (each a run over all tiles of the matrix), so the encode of matrix b
// starts LA matrices of amax work after its own amax, and its second read is
// mostly served by L2.  A B tile of matrix b waits (bounded) until all A
// tiles of b have published their amax.  An item only waits on items with
// smaller indices, and the smallest unfinished item is always being run by
// some CTA (the next index is fetched only once the current item is done),
// so the order cannot deadlock whatever the residency.
//
// Workspace (32-bit words, zeroed by the launcher): [0, 2) item counter
// (64-bit), [4, 4 + batch) amax patterns, [4 + batch, 4 + 2 batch) number of
// finished A tiles per matrix.
// Units of one item per thread (upt): NV_UNITS_PER_THREAD, halved by the
// launcher (down to 1) until every resident CTA gets about two items per
// pass.  A thread walks its units of an item one after another, so a small
// input cut into few large items would serialise that many memory latencies.
constexpr int NV_UNITS_PER_THREAD = 16;
constexpr int NV_LOOKAHEAD = 1;                // matrices of amax work ahead of the encode

// Per-tensor scale g = fp32(amax_T / 2688), 1 for an all-zero tensor.
__device__ __forceinline__ float nvfp4_tensor_scale(uint32_t a) {
    return a == 0 ? 1.0f : __fdiv_rn(__uint_as_float(a << 16), 2688.0f);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Wait until *count >= target; false (and a device error) after ~4 s.
__device__ bool wait_count(const uint32_t* count, uint32_t target, uint32_t* err) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire_u32(count) >= target) return true;
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (it == 0) t0 = now;
        else if (now - t0 > 4000000000ull) {
            raise_device_error(err, FPQ_ERR_DEVICE_TIMEOUT);
            return false;
        }
        __nanosleep(128);
    }
}

// Bracket for quotients by s from an approximation r of 1/s with relative
// error at most 2^-21: r (1 -+ 2^-20) still lands strictly outside
// (1/s)(1 -+ 2^-21), which is what the bracket argument needs.
__device__ __forceinline__ QuotientBracket bracket_from_reciprocal(float s, float r) {
    return QuotientBracket{s, __fmul_rn(r, 1.0f - 0x1p-20f), __fmul_rn(r, 1.0f + 0x1p-20f)};
}

struct NvItem {
    bool is_a;
    int64_t b, t;
};

__device__ __forceinline__ NvItem nv_decode(unsigned long long item, int64_t batch, int64_t nT) {
    NvItem r;
    const int64_t i = (int64_t)item, blk = i / nT;
    const int64_t la = min64(NV_LOOKAHEAD, batch);
    r.t = i - blk * nT;
    if (blk < la) {                                   // leading amax runs
        r.is_a = true; r.b = blk;
        return r;
    }
    const int64_t j = blk - la, pairs = 2 * (batch - la);
    if (j < pairs) {                                  // A(la + p), B(p) alternating
        r.is_a = (j & 1) == 0;
        r.b = r.is_a ? la + j / 2 : j / 2;
    } else {                                          // trailing encode runs
        r.is_a = false; r.b = batch - la + (j - pairs);
    }
    return r;
}

// Within an item each thread encodes its units one at a time, loading the
// next before encoding the current; few registers let NV_MIN_BLOCKS CTAs
// share an SM.
constexpr int NV_MIN_BLOCKS = 5;

__device__ __forceinline__ void nvfp4_encode_unit(const Unit& v, float g, bool g_ok, const QuotientBracket& gb,
                                                  float rg, const ScaleTables& tab6, const float* s_dec,
                                                  const float* s_inv, uint2* qdst, uint8_t* sdst) {
    // block scale code = E4M3(fp32(fp32(amax_b / 6) / g)), S = fp32(dec(code) g)
    const uint32_t a = unit_absmax(v);
    float tq, unused_lo, unused_hi;
    if (!table_scale(tab6, a, 4, tq, unused_lo, unused_hi)) tq = __fdiv_rn(__uint_as_float(a << 16), 6.0f);
    uint32_t code;
    if (g_ok) {
        code = f32x2_to_e4m3x2(__fmul_rn(tq, gb.lo), __fmul_rn(tq, gb.hi));
        code = ((code & 0xFFu) == (code >> 8)) ? (code & 0xFFu) : (f32x2_to_e4m3x2(__fdiv_rn(tq, g), 0.0f) & 0xFFu);
    } else {
        code = f32x2_to_e4m3x2(__fdiv_rn(tq, g), 0.0f) & 0xFFu;
    }
    const float S = code < 127u ? __fmul_rn(s_dec[code], g) : __fmul_rn(e4m3_to_f32(code), g);
    uint32_t packed[2] = {0u, 0u};
    if (S != 0.0f) {
        bool exact = true;
        if (g_ok && reciprocal_ok(S) && code < 127u) {
            // fp32(inv(code) * fp32(1/g)) is within 2^-22 of 1/S, close
            // enough for the bracket (bracket_from_reciprocal); the unit's
            // 16 products with each bracket end are formed in pairs, and the
            // unit falls back to divisions only if any code differs
            const QuotientBracket br = bracket_from_reciprocal(S, __fmul_rn(s_inv[code], rg));
            const uint64_t lo2 = pack2(br.lo, br.lo), hi2 = pack2(br.hi, br.hi);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint64_t x0 = bf16x2_pair(v.w[4 * h]), x1 = bf16x2_pair(v.w[4 * h + 1]),
                               x2 = bf16x2_pair(v.w[4 * h + 2]), x3 = bf16x2_pair(v.w[4 * h + 3]);
                packed[h] = e2m1x8_of_pairs(mul2(x0, lo2), mul2(x1, lo2), mul2(x2, lo2), mul2(x3, lo2));
                const uint32_t up = e2m1x8_of_pairs(mul2(x0, hi2), mul2(x1, hi2), mul2(x2, hi2), mul2(x3, hi2));
                exact = exact && packed[h] == up;
            }
        } else {
            exact = false;
        }
        if (!exact) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint64_t q[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    q[j] = pack2(__fdiv_rn(bf16_lo(v.w[4 * h + j]), S), __fdiv_rn(bf16_hi(v.w[4 * h + j]), S));
                packed[h] = e2m1x8_of_pairs(q[0], q[1], q[2], q[3]);
            }
        }
    }
    st_v2(qdst, make_uint2(packed[0], packed[1]));
    *sdst = (uint8_t)code;
}

template <int upt, bool S>
__global__ void __launch_bounds__(kThreads, NV_MIN_BLOCKS)
quant_nvfp4_kernel(const uint4* __restrict__ x, int64_t batch, int64_t upm, uint2* __restrict__ q,
                   uint8_t* __restrict__ s, float* __restrict__ g_out, uint32_t* __restrict__ ws,
                   uint32_t* err, UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    __shared__ ScaleTables tab6;                 // fp32(amax_b / 6) by mantissa
    __shared__ float s_dec[128];                 // dec(c) for E4M3 codes c = 0..126
    __shared__ float s_inv[128];                 // fp32(1 / dec(c)) for c = 1..126
    __shared__ uint32_t s_wmax[kThreads / 32];
    __shared__ unsigned long long s_item;
    __shared__ int s_ok;
    unsigned long long* counter = reinterpret_cast<unsigned long long*>(ws);
    uint32_t* amax = ws + 4;
    uint32_t* done = ws + 4 + batch;
    constexpr int tile = kThreads * upt;
    const int64_t nT = (upm + tile - 1) / tile;
    const unsigned long long total = (unsigned long long)(2 * batch * nT);
    init_scale_tables(tab6, 6.0f);
    if (threadIdx.x < 128) {
        const uint32_t c = threadIdx.x;
        const float d = c == 127 ? 0.0f : e4m3_to_f32(c);
        s_dec[c] = d;
        s_inv[c] = (c == 0 || c == 127) ? 0.0f : __frcp_rn(d);
    }
    if (threadIdx.x == 0) s_item = atomicAdd(counter, 1ull);
    __syncthreads();
    unsigned long long item = s_item;
    while (item < total) {
        const NvItem w = nv_decode(item, batch, nT);
        // this item's units: [base, base + n) of matrix w.b, addressed by
        // 32-bit offsets from the item's first unit
        const int64_t base = w.b * upm + w.t * tile;
        const int n = (int)min64(tile, upm - w.t * tile);
        const uint4* xi = x + 2 * base;
        const int u0 = threadIdx.x;
        // The amax pass keeps its lines in L2 (evict-last) for the encode pass,
        // which reads them a matrix later and lets them go (evict-first).
        if (w.is_a) {
            const uint64_t keep = l2_policy_evict_last();
            uint32_t am = 0;
            Unit cur;
            if (u0 < n) cur = S ? load_unit_hint(x, in_unit<S>(m, base + u0), keep) : load_unit_hint(xi, u0, keep);
#pragma unroll
            for (int i = 0; i < upt; ++i) {
                const int u = u0 + i * kThreads;
                Unit nxt;
                if (i + 1 < upt && u + kThreads < n)
                    nxt = S ? load_unit_hint(x, in_unit<S>(m, base + u + kThreads), keep)
                            : load_unit_hint(xi, u + kThreads, keep);
                if (u < n) am = max(am, unit_absmax(cur));
                cur = nxt;
            }
            am = group_max<32>(am);
            if ((threadIdx.x & 31) == 0) s_wmax[threadIdx.x >> 5] = am;
            __syncthreads();
            if (threadIdx.x == 0) {
                uint32_t mm = 0;
#pragma unroll
                for (int k = 0; k < kThreads / 32; ++k) mm = max(mm, s_wmax[k]);
                if (mm) atomicMax(amax + w.b, mm);
                __threadfence();                     // publish the amax before the count
                atomicAdd(done + w.b, 1u);
            }
        } else {
            const uint64_t drop = l2_policy_evict_first();
            Unit cur;
            if (u0 < n)                                 // the input is ready; only g must wait
                cur = S ? load_unit_hint(x, in_unit<S>(m, base + u0), drop) : load_unit_hint(xi, u0, drop);
            if (threadIdx.x == 0) s_ok = wait_count(done + w.b, (uint32_t)nT, err) ? 1 : 0;
            __syncthreads();
            if (!s_ok) return;
            const float g = nvfp4_tensor_scale(__ldcg(amax + w.b));
            if (w.t == 0 && threadIdx.x == 0) g_out[w.b] = g;
            const bool g_ok = reciprocal_ok(g);
            const QuotientBracket gb = quotient_bracket(g_ok ? g : 1.0f);
            const float rg = __frcp_rn(g_ok ? g : 1.0f);
            uint2* qi = q + base;
            uint8_t* si = s + base;
#pragma unroll 1
            for (int i = 0; i < upt; ++i) {
                const int u = u0 + i * kThreads;
                Unit nxt;
                if (i + 1 < upt && u + kThreads < n)
                    nxt = S ? load_unit_hint(x, in_unit<S>(m, base + u + kThreads), drop)
                            : load_unit_hint(xi, u + kThreads, drop);
                if (u < n)
                    nvfp4_encode_unit(cur, g, g_ok, gb, rg, tab6, s_dec, s_inv,
                                      S ? q + out_unit<S>(m, base + u) : qi + u, si + u);
                cur = nxt;
            }
        }
        __syncthreads();                             // every thread is done with s_item / s_ok
        if (threadIdx.x == 0) s_item = atomicAdd(counter, 1ull);
        __syncthreads();
        item = s_item;
    }
}

// One or two matrices: the persistent ordering buys no L2 reuse between
// matrices, and an item's units walked one after another leave little in
// flight, so the two passes are two launches instead: a streaming amax
// kernel (kUnroll units in flight per thread, CTA reduction, one atomicMax
// per matrix and CTA) and a grid-stride encode kernel whose launch follows
// the amax kernel's completion in stream order (the input's second read
// is mostly served by L2 at these sizes).  Workspace as above (only the
// amax words are used).
constexpr int NV_SMALL_BATCH = 2;

template <bool S>
__global__ void __launch_bounds__(kThreads, 3)
nvfp4_amax_kernel(const uint4* __restrict__ x, int64_t batch, int64_t upm, uint32_t* __restrict__ ws,
                  UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    __shared__ uint32_t s_wmax[NV_SMALL_BATCH][kThreads / 32];
    const int64_t units = batch * upm;
    const int64_t stride = (int64_t)gridDim.x * kThreads * kUnroll;
    uint32_t am0 = 0, am1 = 0;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kUnroll + threadIdx.x; base < units; base += stride) {
        Unit v[kUnroll];
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) v[i] = load_unit(x, in_unit<S>(m, u));
        }
#pragma unroll
        for (int i = 0; i < kUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                const uint32_t a = unit_absmax(v[i]);
                if (u < upm) am0 = max(am0, a);
                else am1 = max(am1, a);
            }
        }
    }
    am0 = group_max<32>(am0);
    am1 = group_max<32>(am1);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        s_wmax[0][warp] = am0;
        s_wmax[1][warp] = am1;
    }
    __syncthreads();
    if (threadIdx.x < batch) {
        uint32_t mm = 0;
#pragma unroll
        for (int k = 0; k < kThreads / 32; ++k) mm = max(mm, s_wmax[threadIdx.x][k]);
        if (mm) atomicMax(ws + 4 + threadIdx.x, mm);
    }
}

template <bool S>
__global__ void __launch_bounds__(kThreads, 4)
nvfp4_encode_kernel(const uint4* __restrict__ x, int64_t batch, int64_t upm, uint2* __restrict__ q,
                    uint8_t* __restrict__ s, float* __restrict__ g_out, const uint32_t* __restrict__ ws,
                    UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    __shared__ ScaleTables tab6;                 // fp32(amax_b / 6) by mantissa
    __shared__ float s_dec[128];                 // dec(c) for E4M3 codes c = 0..126
    __shared__ float s_inv[128];                 // fp32(1 / dec(c)) for c = 1..126
    init_scale_tables(tab6, 6.0f);
    if (threadIdx.x < 128) {
        const uint32_t c = threadIdx.x;
        const float d = c == 127 ? 0.0f : e4m3_to_f32(c);
        s_dec[c] = d;
        s_inv[c] = (c == 0 || c == 127) ? 0.0f : __frcp_rn(d);
    }
    const float g0 = nvfp4_tensor_scale(__ldcg(ws + 4));
    const float g1 = batch > 1 ? nvfp4_tensor_scale(__ldcg(ws + 5)) : 1.0f;
    if (blockIdx.x == 0 && threadIdx.x < batch) g_out[threadIdx.x] = threadIdx.x == 0 ? g0 : g1;
    __syncthreads();
    const bool ok0 = reciprocal_ok(g0), ok1 = reciprocal_ok(g1);
    const QuotientBracket gb0 = quotient_bracket(ok0 ? g0 : 1.0f), gb1 = quotient_bracket(ok1 ? g1 : 1.0f);
    const float rg0 = __frcp_rn(ok0 ? g0 : 1.0f), rg1 = __frcp_rn(ok1 ? g1 : 1.0f);
    const int64_t units = batch * upm;
    constexpr int kIn = 2;                       // units in flight per thread
    const int64_t stride = (int64_t)gridDim.x * kThreads * kIn;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kIn + threadIdx.x; base < units; base += stride) {
        Unit v[kIn];
#pragma unroll
        for (int i = 0; i < kIn; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) v[i] = load_unit(x, in_unit<S>(m, u));
        }
#pragma unroll
        for (int i = 0; i < kIn; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                const bool first = u < upm;
                nvfp4_encode_unit(v[i], first ? g0 : g1, first ? ok0 : ok1, first ? gb0 : gb1, first ? rg0 : rg1,
                                  tab6, s_dec, s_inv, q + out_unit<S>(m, u), s + u);
            }
        }
    }
}

// ----------------------------------------------------------------- dequantize

__device__ __forceinline__ void store_bf16x16(uint4* out, int64_t u, const float (&f)[16]) {
    uint32_t h[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = f32x2_to_bf16x2(f[2 * j], f[2 * j + 1]);
    st_v4(out + 2 * u, make_uint4(h[0], h[1], h[2], h[3]));
    st_v4(out + 2 * u + 1, make_uint4(h[4], h[5], h[6], h[7]));
}

// Units in flight per thread in the dequantizers: all of an iteration's
// code (and scale) loads are issued before any unit is decoded.
constexpr int kDqUnroll = 4;

// fmt: 0 = 1x128 (fp32 scale per 8 units), 2 = MXFP8 (E8M0 per 2 units),
// 1 = 128x128 (fp32 scale per 128x128 block).
template <int kFmt>
__device__ __forceinline__ float fp8_unit_scale(const void* __restrict__ scales, int64_t u, int64_t rows,
                                                int64_t cols) {
    if (kFmt == 2) {
        const uint32_t code = ((const uint8_t*)scales)[u >> 1];
        return code == 0xFFu ? __uint_as_float(0x7FC00000u)
             : code == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
    } else if (kFmt == 0) {
        return ((const float*)scales)[u >> 3];
    } else {
        const int64_t units_per_row = cols / 16;
        const int64_t row = u / units_per_row, colu = u - row * units_per_row;
        const int64_t b = row / rows, r = row - b * rows;
        const int64_t nbr = (rows + 127) / 128, nbc = cols / 128;
        return ((const float*)scales)[(b * nbr + r / 128) * nbc + colu / 8];
    }
}

template <int kFmt, bool S>
__global__ void __launch_bounds__(kThreads, 3)
dequant_fp8_kernel(const uint4* __restrict__ q, const void* __restrict__ scales, uint4* __restrict__ out,
                   int64_t units, int64_t rows, int64_t cols, UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    const int64_t stride = (int64_t)gridDim.x * kThreads * kDqUnroll;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kDqUnroll + threadIdx.x; base < units; base += stride) {
        uint4 c[kDqUnroll];
        float sc[kDqUnroll];
#pragma unroll
        for (int i = 0; i < kDqUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                c[i] = ld_stream(q + in_unit<S>(m, u));
                sc[i] = fp8_unit_scale<kFmt>(scales, u, rows, cols);
            }
        }
#pragma unroll
        for (int i = 0; i < kDqUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                const uint32_t w[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
                float f[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 lo = e4m3x2_to_f32x2(w[j] & 0xFFFFu), hi = e4m3x2_to_f32x2(w[j] >> 16);
                    f[4 * j + 0] = lo.x * sc[i]; f[4 * j + 1] = lo.y * sc[i];
                    f[4 * j + 2] = hi.x * sc[i]; f[4 * j + 3] = hi.y * sc[i];
                }
                store_bf16x16(out, out_unit<S>(m, u), f);
            }
        }
    }
}

template <bool S>
__global__ void __launch_bounds__(kThreads, 3)
dequant_nvfp4_kernel(const uint2* __restrict__ q, const uint8_t* __restrict__ s, const float* __restrict__ g,
                     uint4* __restrict__ out, int64_t units, int64_t units_per_matrix, UnitStrides m) {
    pdl_trigger();   // dependents may launch now; they wait for this grid to finish
    const int64_t stride = (int64_t)gridDim.x * kThreads * kDqUnroll;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kDqUnroll + threadIdx.x; base < units; base += stride) {
        uint2 c[kDqUnroll];
        float Sc[kDqUnroll];
#pragma unroll
        for (int i = 0; i < kDqUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                c[i] = q[in_unit<S>(m, u)];
                Sc[i] = e4m3_to_f32(s[u]) * g[u / units_per_matrix];
            }
        }
#pragma unroll
        for (int i = 0; i < kDqUnroll; ++i) {
            const int64_t u = base + (int64_t)i * kThreads;
            if (u < units) {
                const uint32_t w[2] = {c[i].x, c[i].y};
                float f[16];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float2 e = e2m1x2_to_f32x2((w[j >> 2] >> (8 * (j & 3))) & 0xFFu);
                    f[2 * j] = e.x * Sc[i];
                    f[2 * j + 1] = e.y * Sc[i];
                }
                store_bf16x16(out, out_unit<S>(m, u), f);
            }
        }
    }
}

int grid_for(int64_t work_items, int per_cta, int sms) {
    int64_t g = (work_items + per_cta - 1) / per_cta;
    int64_t cap = (int64_t)sms * 8;
    return (int)max64(1, min(g, cap));
}

}  // namespace

// ----------------------------------------------------------------- launchers

namespace {
// Unit strides of an operand pair; `strided` false when both are dense.
UnitStrides unit_strides(const OperandStrides* os, int64_t rows, int64_t cols, bool& strided) {
    const int64_t upr = cols / 16;
    UnitStrides m{upr, rows * upr, upr, rows * upr, upr, rows * upr};
    strided = false;
    if (os) {
        m.in_ld = os->ld_in / 16;
        m.in_bs = os->bs_in / 16;
        m.out_ld = os->ld_out / 16;
        m.out_bs = os->bs_out / 16;
        strided = m.in_ld != upr || m.in_bs != rows * upr || m.out_ld != upr || m.out_bs != rows * upr;
    }
    return m;
}
}  // namespace

cudaError_t launch_quantize(int fmt, const void* x, int64_t batch, int64_t rows, int64_t cols,
                            void* q, void* scales, float* tensor_scale, void* workspace,
                            uint32_t* err, int sms, cudaStream_t st, const OperandStrides* strides) {
    const int64_t n = batch * rows * cols, units = n / 16;
    bool sd = false;
    const UnitStrides m = unit_strides(strides, rows, cols, sd);
    switch (fmt) {
    case FPQ_MXFP8: {
        const int grid = grid_for(units, kThreads * kUnroll, sms);
        if (sd) quant_mxfp8_kernel<true><<<grid, kThreads, 0, st>>>((const uint4*)x, (uint4*)q, (uint8_t*)scales,
                                                                    units, m);
        else quant_mxfp8_kernel<false><<<grid, kThreads, 0, st>>>((const uint4*)x, (uint4*)q, (uint8_t*)scales,
                                                                  units, m);
        break;
    }
    case FPQ_FP8_1x128: {
        const int grid = (int)max64(1, min64((units + kThreads - 1) / kThreads, (int64_t)sms * Q1_MIN_BLOCKS));
        if (sd) quant_fp8_1x128_kernel<true><<<grid, kThreads, 0, st>>>((const uint4*)x, (uint4*)q, (float*)scales,
                                                                        units, m);
        else quant_fp8_1x128_kernel<false><<<grid, kThreads, 0, st>>>((const uint4*)x, (uint4*)q, (float*)scales,
                                                                      units, m);
        break;
    }
    case FPQ_FP8_128x128: {
        const int64_t nblocks = batch * ((rows + 127) / 128) * (cols / 128);
        const int64_t ldx = strides ? strides->ld_in : cols, bsx = strides ? strides->bs_in : rows * cols;
        const int64_t ldq = strides ? strides->ld_out : cols, bsq = strides ? strides->bs_out : rows * cols;
        (sd ? quant_fp8_128x128_kernel<true> : quant_fp8_128x128_kernel<false>)<<<(unsigned)nblocks, QB_THREADS, 0,
                                                                                 st>>>(
            (const uint8_t*)x, (uint8_t*)q, (float*)scales, rows, cols, ldx, bsx, ldq, bsq);
        break;
    }
    case FPQ_NVFP4: {
        const int64_t upm = rows * cols / 16;
        uint32_t* ws = (uint32_t*)workspace;
        cudaError_t e = cudaMemsetAsync(ws, 0, nvfp4_workspace_words(batch) * sizeof(uint32_t), st);
        if (e != cudaSuccess) return e;
        if (batch <= NV_SMALL_BATCH) {
            const int ga = grid_for(units, kThreads * kUnroll, sms);
            const int ge = (int)max64(1, min64((units + 2 * kThreads - 1) / (2 * kThreads), (int64_t)sms * 4));
            if (sd) {
                nvfp4_amax_kernel<true><<<ga, kThreads, 0, st>>>((const uint4*)x, batch, upm, ws, m);
                nvfp4_encode_kernel<true><<<ge, kThreads, 0, st>>>((const uint4*)x, batch, upm, (uint2*)q,
                                                                   (uint8_t*)scales, tensor_scale, ws, m);
            } else {
                nvfp4_amax_kernel<false><<<ga, kThreads, 0, st>>>((const uint4*)x, batch, upm, ws, m);
                nvfp4_encode_kernel<false><<<ge, kThreads, 0, st>>>((const uint4*)x, batch, upm, (uint2*)q,
                                                                    (uint8_t*)scales, tensor_scale, ws, m);
            }
            break;
        }
        const int64_t slots = (int64_t)sms * NV_MIN_BLOCKS;
        int upt = NV_UNITS_PER_THREAD;
        while (upt > 1 && batch * ((upm + (int64_t)kThreads * upt - 1) / ((int64_t)kThreads * upt)) < 2 * slots) upt /= 2;
        const int64_t items = 2 * batch * ((upm + (int64_t)kThreads * upt - 1) / ((int64_t)kThreads * upt));
        const int grid = (int)max64(1, min64(items, slots));
        auto kern = sd ? (upt == 16 ? quant_nvfp4_kernel<16, true> : upt == 8 ? quant_nvfp4_kernel<8, true>
                          : upt == 4 ? quant_nvfp4_kernel<4, true> : upt == 2 ? quant_nvfp4_kernel<2, true>
                          : quant_nvfp4_kernel<1, true>)
                       : (upt == 16 ? quant_nvfp4_kernel<16, false> : upt == 8 ? quant_nvfp4_kernel<8, false>
                          : upt == 4 ? quant_nvfp4_kernel<4, false> : upt == 2 ? quant_nvfp4_kernel<2, false>
                          : quant_nvfp4_kernel<1, false>);
        kern<<<grid, kThreads, 0, st>>>((const uint4*)x, batch, upm, (uint2*)q, (uint8_t*)scales, tensor_scale, ws,
                                        err, m);
        break;
    }
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize(int fmt, const void* q, const void* scales, const float* tensor_scale,
                              int64_t batch, int64_t rows, int64_t cols, void* out, int sms, cudaStream_t st,
                              const OperandStrides* strides) {
    const int64_t units = batch * rows * cols / 16;
    const int grid = grid_for(units, kThreads * kDqUnroll, sms);
    bool sd = false;
    const UnitStrides m = unit_strides(strides, rows, cols, sd);
#define FPQ_DEQ(F)                                                                                                \
    (sd ? dequant_fp8_kernel<F, true> : dequant_fp8_kernel<F, false>)<<<grid, kThreads, 0, st>>>(                 \
        (const uint4*)q, scales, (uint4*)out, units, rows, cols, m)
    switch (fmt) {
    case FPQ_MXFP8:
        FPQ_DEQ(2);
        break;
    case FPQ_FP8_1x128:
        FPQ_DEQ(0);
        break;
    case FPQ_FP8_128x128:
        FPQ_DEQ(1);
        break;
    case FPQ_NVFP4:
        (sd ? dequant_nvfp4_kernel<true> : dequant_nvfp4_kernel<false>)<<<grid, kThreads, 0, st>>>(
            (const uint2*)q, (const uint8_t*)scales, tensor_scale, (uint4*)out, units, rows * cols / 16, m);
        break;
    default:
        return cudaErrorInvalidValue;
    }
#undef FPQ_DEQ
    return cudaGetLastError();
}

}  // namespace fpq
