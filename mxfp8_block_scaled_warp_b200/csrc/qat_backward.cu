// qat_backward.cu -- the backward of the QAT step's linear layer with the
// straight-through estimator ("DeepSeek R1 and V3 get quantization-aware
// fine-tuning on Fireworks", Synopsis and Interpretation: LoRA adapters
// trained through the FP8-quantized forward, then merged).  The forward is
// y = fq(x) fq(W_eff)^T with W_eff = W + (alpha / r) B A; the fake-quantizers
// pass gradients unchanged, W is frozen, so for the output gradient dY:
//   dX     = dY Wfq                  [M, K]
//   dW_eff = dY^T Xfq                [N, K]   (bf16, also an output)
//   dA     = (alpha / r) B^T dW_eff  [r, K]
//   dB     = (alpha / r) dW_eff A^T  [N, r]
// with Xfq = fq(x), Wfq = fq(W_eff) in bf16 and fp32 accumulation, all
// results rounded to bf16.  Every product runs on the bf16 tensor-core GEMM
// (C = alpha P Q^T), which reads each operand in the layout it is stored in
// (K-major or MN-major).  The tiled bf16 transpose below is exported as a
// utility.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace fpq {

namespace {

// bf16 [R, C] -> [C, R].  One CTA of 256 threads per 64 x 64 tile: 16-byte
// row loads into shared memory (rows padded by 8 elements), then each thread
// gathers 8 consecutive elements of an output row (a column of the tile)
// and writes them as one 16-byte store.  R and C are multiples of 8.
constexpr int TT = 64;

__global__ void __launch_bounds__(256)
transpose_bf16_kernel(const uint16_t* __restrict__ in, uint16_t* __restrict__ out, int64_t R, int64_t C) {
    pdl_trigger();
    __shared__ uint16_t tile[TT][TT + 8];
    const int64_t r0 = (int64_t)blockIdx.y * TT, c0 = (int64_t)blockIdx.x * TT;
    pdl_wait();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int v = threadIdx.x + 256 * i;          // 512 chunks of 8 elements
        const int r = v >> 3, c = (v & 7) * 8;
        uint4 x = make_uint4(0, 0, 0, 0);
        if (r0 + r < R && c0 + c < C) x = *reinterpret_cast<const uint4*>(in + (r0 + r) * C + c0 + c);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            tile[r][c + 2 * j] = (uint16_t)(w[j] & 0xFFFFu);
            tile[r][c + 2 * j + 1] = (uint16_t)(w[j] >> 16);
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int v = threadIdx.x + 256 * i;
        const int oc = v >> 3, orr = (v & 7) * 8;     // output row c0 + oc, columns r0 + orr .. + 7
        if (c0 + oc < C && r0 + orr < R) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = (uint32_t)tile[orr + 2 * j][oc] | ((uint32_t)tile[orr + 2 * j + 1][oc] << 16);
            *reinterpret_cast<uint4*>(out + (c0 + oc) * R + r0 + orr) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

inline size_t round_up(size_t x) { return (x + 255) & ~size_t(255); }

// A second stream per device for the fork below, with the two events of
// the fork and the join; created on first use.  The fork-join section holds
// the mutex, so concurrent callers never interleave records and waits on
// the shared events.
constexpr int kForkDevices = 64;
struct Fork {
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
Fork g_fork[kForkDevices];
std::mutex g_fork_mu;

cudaError_t fork_state(Fork** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kForkDevices) return cudaErrorInvalidDevice;
    Fork& f = g_fork[dev];
    if (!f.side) {
        if ((e = cudaStreamCreateWithFlags(&f.side, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    *out = &f;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_transpose_bf16(const void* in, void* out, int64_t R, int64_t C, cudaStream_t st) {
    const dim3 grid((unsigned)((C + TT - 1) / TT), (unsigned)((R + TT - 1) / TT));
    return launch_pdl(transpose_bf16_kernel, grid, dim3(256), 0, st, (const uint16_t*)in, (uint16_t*)out, R, C);
}

// The skinny products dA [r, k] and dB [n, r]: for r <= 64 one kernel reads
// each tile of dW once and issues both products from it (lora_grads.cu),
// its workspace holding the fp32 partial sums; for larger r each is a
// split-K bf16 GEMM (partials of at most kMaxSplits slices each).  Every
// operand is read in the layout it is stored in (the GEMM takes K-major or
// MN-major operands).
// The workspace ends with the two tile counters of the dX and dW products
// (kCounterBytes, zeroed by the call), which share the GPU.
constexpr size_t kCounterBytes = 256;

size_t grads_workspace_bytes(int64_t n, int64_t k, int64_t r) {
    if (lora_grads_fused(r)) return round_up(lora_grads_workspace_bytes(n, k, r, current_sms()));
    return round_up((size_t)kMaxSplits * (size_t)(r * k) * 4) + round_up((size_t)kMaxSplits * (size_t)(n * r) * 4);
}

size_t qat_backward_workspace_bytes(int64_t, int64_t n, int64_t k, int64_t r) {
    return grads_workspace_bytes(n, k, r) + kCounterBytes;
}

int current_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}

cudaError_t launch_qat_backward(const void* dy, const void* x_fq, const void* w_fq, const void* lora_a,
                                const void* lora_b, int64_t m, int64_t n, int64_t k, int64_t r, float alpha_over_r,
                                void* dx, void* dw, void* da, void* db, void* ws, uint32_t* err, int sms,
                                cudaStream_t st) {
    float* part_a = static_cast<float*>(ws);
    float* part_b = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + round_up((size_t)kMaxSplits * (size_t)(r * k) * 4));
    // dX does not depend on the other three products: it runs on a second
    // stream, forked from and joined back into st, so that its tiles fill
    // the SMs that dW's last partial wave leaves idle.  Works under stream
    // capture (the fork and join become graph edges).
    std::lock_guard<std::mutex> lock(g_fork_mu);
    Fork* f = nullptr;
    cudaError_t e = fork_state(&f);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + grads_workspace_bytes(n, k, r), 0, 2 * sizeof(int), st)) !=
        cudaSuccess)
        return e;
    if ((e = cudaEventRecord(f->fork, st)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(f->side, f->fork, 0)) != cudaSuccess) return e;
    // Both products claim their tiles from counters (zeroed here, on st
    // before the fork is taken), so that dX's CTAs, which start on the SMs
    // dW's finish, take only the tiles that are left.
    int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + grads_workspace_bytes(n, k, r));
    // dW [n, k] = dY^T Xfq: contraction over m; dY [m, n] and Xfq [m, k] MN-major
    e = launch_gemm_bf16(dy, true, x_fq, true, n, k, m, 1.0f, dw, err, st, counters);
    // dX [m, k] = dY Wfq: contraction over n; dY [m, n] K-major, Wfq [n, k] MN-major
    if (e == cudaSuccess) e = launch_gemm_bf16(dy, false, w_fq, true, m, k, n, 1.0f, dx, err, f->side, counters + 1);
    if (lora_grads_fused(r)) {
        // dA and dB from one pass over dW (each tile read once, both products issued from it)
        if (e == cudaSuccess)
            e = launch_lora_grads(dw, lora_a, lora_b, n, k, (int)r, alpha_over_r, da, db, ws, err, sms, st);
    } else {
        // dA [r, k] = (alpha / r) B^T dW: contraction over n; B [n, r] and dW [n, k] MN-major
        if (e == cudaSuccess)
            e = launch_gemm_bf16_splitk(lora_b, true, dw, true, r, k, n, alpha_over_r, da, part_a,
                                        bf16_split_count(r, k, n, sms), err, st);
        // dB [n, r] = (alpha / r) dW A^T: contraction over k; dW [n, k] and A [r, k] K-major
        if (e == cudaSuccess)
            e = launch_gemm_bf16_splitk(dw, false, lora_a, false, n, r, k, alpha_over_r, db, part_b,
                                        bf16_split_count(n, r, k, sms), err, st);
    }
    // the join is made on every path, so a capture is never left forked
    cudaError_t j = cudaEventRecord(f->join, f->side);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, f->join, 0);
    return e != cudaSuccess ? e : j;
}

}  // namespace fpq
