// internal.h -- host-side launchers shared between the kernel translation
// units and the C-ABI layer (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fpq {

// 32-bit words of NVFP4 quantize workspace for `batch` matrices: a 64-bit
// work-item counter (4 words with padding), one amax word and one progress
// counter per matrix.
inline int64_t nvfp4_workspace_words(int64_t batch) { return 4 + 2 * batch; }

// Row and batch strides, in elements, of a kernel's input and output
// operands (multiples of 16); nullptr means both are dense.  Scales are
// always dense row-major.
struct OperandStrides {
    int64_t ld_in, bs_in, ld_out, bs_out;
};

// Quantize `batch` row-major bf16 matrices [rows, cols] (fmt: fpq_format).
cudaError_t launch_quantize(int fmt, const void* x, int64_t batch, int64_t rows, int64_t cols,
                            void* q, void* scales, float* tensor_scale, void* workspace,
                            uint32_t* err, int sms, cudaStream_t st, const OperandStrides* strides = nullptr);

cudaError_t launch_dequantize(int fmt, const void* q, const void* scales, const float* tensor_scale,
                              int64_t batch, int64_t rows, int64_t cols, void* out, int sms,
                              cudaStream_t st, const OperandStrides* strides = nullptr);

cudaError_t launch_lora_merge_fakequant(const void* w, const void* a, const void* b, int64_t n,
                                        int64_t k, int r, float alpha_over_r, void* wq, float* ws,
                                        void* w_fq, int sms, cudaStream_t st);

// Dense block-scaled GEMMs: C[m,n] = sum_k A[m,k] B[n,k].
cudaError_t launch_gemm_mxfp8(const void* aq, const void* as, const void* bq, const void* bs,
                              int64_t m, int64_t n, int64_t k, void* c, int c_f32,
                              uint32_t* err, int sms, cudaStream_t st);

cudaError_t launch_gemm_fp8_f32scale(const void* aq, const float* as, const void* bq,
                                     const float* bs, int64_t m, int64_t n, int64_t k, void* c,
                                     int c_f32, uint32_t* err, int sms, cudaStream_t st);

// NVFP4 GEMM: C = ga gb sum_k A[m,k] B[n,k] (packed E2M1, E4M3 per 16).
cudaError_t launch_gemm_nvfp4(const void* aq, const void* as, const float* ag, const void* bq, const void* bs,
                              const float* bg, int64_t m, int64_t n, int64_t k, void* c, int c_f32, uint32_t* err,
                              cudaStream_t st);

// C = alpha P Q^T, C [m, n] bf16.  P is [m, k] (K-major) or, with p_mn,
// stored as [k, m] (MN-major); likewise Q [n, k] or, with q_mn, [k, n].
// tile_counter: a zeroed device int from which the persistent CTAs claim
// tiles (for products that share the GPU with another); nullptr: CTA c
// takes tiles c, c + grid, ...
cudaError_t launch_gemm_bf16(const void* p, bool p_mn, const void* q, bool q_mn, int64_t m, int64_t n, int64_t k,
                             float alpha, void* c, uint32_t* err, cudaStream_t st, int* tile_counter = nullptr);

// Split-K variant for products with few output tiles: fp32 partial sums of
// `splits` K slices in `partial` ([splits, m, n] fp32), then a reduce kernel
// writes bf16(alpha * sum) to c; m * n a multiple of 4.
constexpr int kMaxSplits = 16;
constexpr int kSplitSms = 256;
int bf16_split_bound(int64_t m, int64_t n, int64_t k);          // slices the workspace must hold
int bf16_split_count(int64_t m, int64_t n, int64_t k, int sms);
cudaError_t launch_gemm_bf16_splitk(const void* p, bool p_mn, const void* q, bool q_mn, int64_t m, int64_t n,
                                    int64_t k, float alpha, void* c, float* partial, int splits, uint32_t* err,
                                    cudaStream_t st);

// MoE FP8 dispatch (moe_dispatch.cu).  The route workspace holds the
// per-chunk histograms and slot bases; a chunk is moe_tokens_per_chunk(T)
// consecutive tokens.
int64_t moe_tokens_per_chunk(int64_t tokens);
int64_t moe_chunks(int64_t tokens);
size_t moe_route_workspace_bytes(int64_t tokens, int experts);
cudaError_t launch_moe_route(const int32_t* ids, int64_t tokens, int topk, int experts, int32_t* counts,
                             void* workspace, uint32_t* err, cudaStream_t st);
cudaError_t launch_moe_layout(const int32_t* counts_all, int world, int experts, int rank, int pack,
                              int64_t* dst_row0, int32_t* recv_offsets, cudaStream_t st);
cudaError_t launch_moe_regroup(const void* src_q, const void* src_s, const int32_t* counts_all, int world,
                               int experts, int rank, int64_t hidden, int64_t rows, void* dst_q, void* dst_s,
                               uint32_t* err, int sms, cudaStream_t st);
cudaError_t launch_moe_dispatch_mxfp8(const void* x, int64_t tokens, int64_t hidden, const int32_t* ids, int topk,
                                      int experts, const void* workspace, const int64_t* dst_row0, int n_dest,
                                      void* const* dst_codes, void* const* dst_scales, const int64_t* dst_capacity,
                                      uint32_t* err, cudaStream_t st);

// bf16 [R, C] -> [C, R] (R, C multiples of 8).
cudaError_t launch_transpose_bf16(const void* in, void* out, int64_t R, int64_t C, cudaStream_t st);

// QAT backward (straight-through estimator); workspace of
// qat_backward_workspace_bytes bytes.
size_t qat_backward_workspace_bytes(int64_t m, int64_t n, int64_t k, int64_t r);
// The LoRA gradients dA = alpha B^T dW, dB = alpha dW A^T in one pass over
// dW (r <= 64); the workspace holds their fp32 partial sums.
bool lora_grads_fused(int64_t r);
size_t lora_grads_workspace_bytes(int64_t n, int64_t k, int64_t r, int sms);
cudaError_t launch_lora_grads(const void* dw, const void* lora_a, const void* lora_b, int64_t n, int64_t k, int r,
                              float alpha_over_r, void* da, void* db, void* workspace, uint32_t* err, int sms,
                              cudaStream_t st);
// SM count of the current device (0 if there is none)
int current_sms();
cudaError_t launch_qat_backward(const void* dy, const void* x_fq, const void* w_fq, const void* lora_a,
                                const void* lora_b, int64_t m, int64_t n, int64_t k, int64_t r, float alpha_over_r,
                                void* dx, void* dw, void* da, void* db, void* ws, uint32_t* err, int sms,
                                cudaStream_t st);

cudaError_t launch_grouped_gemm_mxfp8(const void* aq, const void* as, const void* bq,
                                      const void* bs, const int32_t* offsets, int groups,
                                      int64_t total_m, int64_t n, int64_t k, void* c, int c_f32,
                                      uint32_t* err, int sms, cudaStream_t st);

// Set the per-thread detail string returned by fpq_last_error_detail().
void set_error_detail(const char* what);

// Launch with programmatic dependent launch allowed: the kernel may become
// resident while the previous kernel in the stream is still finishing, so it
// must execute pdl_wait() (griddepcontrol.wait) before it touches global
// memory that earlier work writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace fpq
