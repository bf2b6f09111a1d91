/*
 * fpq.h -- C ABI of the B200 (sm_100a) library for fine-grained block-scaled
 * low-precision quantization and the block-scaled matmul that consumes it.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All data pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or keeps them past the call; it enqueues kernels
 *    on `stream` (a cudaStream_t passed as void*, NULL = the legacy default
 *    stream) and returns without synchronizing.  The caller must keep every
 *    buffer alive until the stream has passed the enqueued work.
 *  - Tensors are row-major; batched tensors are batch-major with no padding
 *    ([batch][rows][cols]), except where an entry point takes explicit row
 *    and batch strides (the *_strided calls).  bf16 values are raw 16-bit
 *    patterns.
 *  - Scratch memory is a caller-owned workspace, sized by the matching
 *    *_workspace_bytes call.
 *  - Every pointer must be 16-byte aligned.
 *  - Scales are DEQUANTIZATION MULTIPLIERS ("scale inverse"): an element's
 *    value is approximately decode(code) * scale.
 *  - Return values are synchronous status codes (fpq_status).  On any error
 *    nothing is enqueued.  FPQ_ERR_CUDA carries the CUDA error text in
 *    fpq_last_error_detail() (per thread).  Faults detected inside a kernel
 *    (a bounded wait that ran out, a malformed group offset list, an expert
 *    id out of range) are written to a device-side error word read by
 *    fpq_get_device_error().
 *  - There is no CPU fallback: a missing or non-sm_100 device gives
 *    FPQ_ERR_UNSUPPORTED.
 *
 * Numerics (all formats): round-to-nearest-even, E4M3 saturating to +-448,
 * E2M1 saturating to +-6, IEEE fp32 arithmetic with gradual underflow.
 * Element encodings are those of the OCP Microscaling (MX) v1.0 formats.
 *
 * Sources (web pages, cited by title and section):
 *  [FP]  "fireworks-prequant 0.1.0" (PyPI): "Formats" (mxfp8 = 1x32 block
 *        FP8 with E8M0 scales; nvfp4 = packed FP4 with FP8 block scales) and
 *        "Quick start" (float8_e4m3fn weight + uint8 E8M0 weight_scale_inv;
 *        only routed MoE expert projections are quantized).
 *  [DS]  "FP8 в DeepSeek V3: как низкая точность ускоряет обучение и
 *        инференс": "Как FP8 встроен в DeepSeek V3" (online
 *        per-token-per-128-channel activation quantization), "Почему обычное
 *        округление не подходит" (128x128 weight blocks, scale inverse for
 *        dequantization), "Инференс с FP8" (activation quantization, weight
 *        dequantization and FP8 matmul kernels).
 *  [B5]  "DeepSeek-V3 Blog 5: Low-Precision Training -- The FP8 Revolution":
 *        "The Solution: Block-Wise Quantization", "Hardware Optimization"
 *        (FP8 products promoted to higher precision before accumulation),
 *        "Reducing Communication Overhead in MoE with FP8" (activations sent
 *        to the experts' GPUs in FP8: the MoE dispatch calls).
 *  [QAT] "DeepSeek R1 and V3 get quantization-aware fine-tuning on
 *        Fireworks": "Synopsis"/"Interpretation" (LoRA merged into the base
 *        weight, merged bf16 weight converted to block-wise FP8, forward
 *        pass fake-quantizes merged weights and activations; the adapters
 *        are trained through it: the QAT backward calls).
 *
 * Families: block quantize / dequantize (dense and strided); the LoRA merge
 * with weight fake-quant; block-scaled GEMMs (fp32 scales, MXFP8, NVFP4,
 * grouped MXFP8); the bf16 GEMMs of the QAT backward; the MoE FP8 dispatch;
 * status and error queries.
 */
#ifndef FPQ_H
#define FPQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FPQ_API __attribute__((visibility("default")))
#else
#define FPQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t fpq_status;
enum {
    FPQ_OK = 0,
    FPQ_ERR_INVALID_ARG = 1,     /* null pointer, bad shape, bad enum value     */
    FPQ_ERR_ALIGNMENT = 2,       /* a pointer is not 16-byte aligned            */
    FPQ_ERR_UNSUPPORTED = 3,     /* no sm_100 device, or format pair not built  */
    FPQ_ERR_CUDA = 4,            /* a CUDA call failed (see detail string)      */
    FPQ_ERR_DEVICE_TIMEOUT = 5,  /* device error word: a bounded wait ran out   */
    FPQ_ERR_DEVICE_BAD_INPUT = 6,/* device error word: malformed device input   */
    FPQ_ERR_WORKSPACE = 7        /* workspace missing or too small              */
};

/* Block formats (fpq_format). */
typedef int32_t fpq_format;
enum {
    /* FP8-E4M3, one fp32 scale per 1x128 tile of a row (activations) [DS].
     * codes uint8 [B,R,C]; scales fp32 [B,R,C/128]; C % 128 == 0.
     * s = fp32(amax/448) (1.0 for an all-zero tile); q = E4M3(fp32(x / s)). */
    FPQ_FP8_1x128 = 0,
    /* FP8-E4M3, one fp32 scale per 128x128 block (weights) [DS].
     * codes uint8 [B,R,C]; scales fp32 [B,ceil(R/128),C/128]; C % 128 == 0;
     * the last block row may be short.  Same s and q rule as FPQ_FP8_1x128. */
    FPQ_FP8_128x128 = 1,
    /* MXFP8: FP8-E4M3, one E8M0 scale per 1x32 block of a row [FP].
     * codes uint8 [B,R,C]; scales uint8 [B,R,C/32]; C % 32 == 0.
     * e = clamp(ceil(log2(amax/448)), -127, 127), scale code e + 127,
     * q = E4M3(x * 2^-e) (exact scaling; no element saturates). */
    FPQ_MXFP8 = 2,
    /* NVFP4: E2M1 packed two per byte (element 2i in the low nibble), one
     * E4M3 scale per 1x16 block, one fp32 tensor scale g per batch item [FP].
     * codes uint8 [B,R,C/2]; scales uint8 [B,R,C/16]; g fp32 [B]; C % 32 == 0.
     * g = fp32(amax_T/2688) (1 for an all-zero tensor),
     * s_b = E4M3(fp32(fp32(amax_b/6)/g)), S = fp32(dec(s_b)*g),
     * q = E2M1(fp32(x/S)) (all zero when S == 0). */
    FPQ_NVFP4 = 3
};

/* GEMM output element type. */
enum { FPQ_OUT_BF16 = 0, FPQ_OUT_F32 = 1 };

/* Version of this ABI: major * 10000 + minor * 100 + patch. */
FPQ_API int32_t fpq_version(void);

/* Static text for a status code. */
FPQ_API const char* fpq_status_string(fpq_status status);

/* Detail of the last failing call on this host thread ("" if none). */
FPQ_API const char* fpq_last_error_detail(void);
/* The same text under the name of its most common use: after FPQ_ERR_CUDA
 * it holds the failing call and the CUDA error string. */
FPQ_API const char* fpq_last_cuda_error(void);

/* Bytes of device workspace fpq_quantize_block needs for `fmt` and `batch`
 * (NVFP4: 16 + 8 * batch bytes -- a work-item counter, and per batch item
 * the tensor amax and a progress counter of the amax pass; 0 otherwise). */
FPQ_API size_t fpq_quantize_workspace_bytes(fpq_format fmt, int64_t batch);

/*
 * fpq_quantize_block -- block-wise quantization of bf16 to FP8/FP4 with
 * per-block scales [B5 "The Solution: Block-Wise Quantization"; DS; FP].
 *
 *   x              bf16 [batch, rows, cols] (input, read only)
 *   q              codes, layout of `fmt` (output)
 *   scales         block scales, layout of `fmt` (output)
 *   tensor_scale   NVFP4 only: fp32 g per batch item (output); NULL otherwise
 *   workspace      NVFP4 only: >= fpq_quantize_workspace_bytes() bytes of
 *                  device memory, contents overwritten; NULL otherwise
 *
 * Outputs are bit-identical for any stream, batch split and launch history.
 * Errors: FPQ_ERR_INVALID_ARG (null pointer, batch/rows/cols < 1, cols not a
 * multiple of the format's block), FPQ_ERR_ALIGNMENT, FPQ_ERR_WORKSPACE,
 * FPQ_ERR_UNSUPPORTED, FPQ_ERR_CUDA.
 */
FPQ_API fpq_status fpq_quantize_block(fpq_format fmt, const void* x, int64_t batch, int64_t rows,
                              int64_t cols, void* q, void* scales, float* tensor_scale,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * fpq_dequantize -- out = bf16(fp32(decode(q) * scale)) per element, the
 * "scale inverse" dequantization [DS "Почему обычное округление не подходит";
 * "Практический смысл для инференс-инфраструктуры" (conversion to BF16)].
 * For NVFP4 the scale is S = fp32(dec(s_b) * g).
 *
 *   q, scales, tensor_scale   as produced by fpq_quantize_block
 *   out                       bf16 [batch, rows, cols] (output)
 *
 * Errors: as fpq_quantize_block.
 */
FPQ_API fpq_status fpq_dequantize(fpq_format fmt, const void* q, const void* scales,
                          const float* tensor_scale, int64_t batch, int64_t rows,
                          int64_t cols, void* out, void* stream);

/*
 * fpq_quantize_block_strided, fpq_dequantize_strided -- the same two
 * operations on strided matrices: the bf16 operand and the code operand each
 * have a row stride (ld_*) and a batch stride (bs_*), counted in ELEMENTS
 * (for NVFP4 codes, two elements per byte); scales stay dense row-major as
 * above.  Element (b, r, c) of the bf16 operand is at x + b*bs_x + r*ld_x + c
 * (likewise out with ld_out, bs_out), and its code at element offset
 * b*bs_q + r*ld_q + c of q.  Results are the same bytes as the dense calls
 * on the same logical matrices.
 *
 * Requires, besides the dense calls' rules: every ld and bs a multiple of 16,
 * ld >= cols, bs >= rows*ld when batch > 1.  The library does not check that
 * strided operands do not overlap.  Errors: as the dense calls.
 */
FPQ_API fpq_status fpq_quantize_block_strided(fpq_format fmt, const void* x, int64_t ld_x, int64_t bs_x,
                                              int64_t batch, int64_t rows, int64_t cols, void* q, int64_t ld_q,
                                              int64_t bs_q, void* scales, float* tensor_scale, void* workspace,
                                              size_t workspace_bytes, void* stream);
FPQ_API fpq_status fpq_dequantize_strided(fpq_format fmt, const void* q, int64_t ld_q, int64_t bs_q,
                                          const void* scales, const float* tensor_scale, int64_t batch,
                                          int64_t rows, int64_t cols, void* out, int64_t ld_out, int64_t bs_out,
                                          void* stream);

/*
 * fpq_lora_merge_fakequant -- the weight side of the QAT forward [QAT]:
 *   delta[n,k] = sum_{j<r} B[n,j] * A[j,k]   (fp32, fused multiply-adds,
 *                                              j ascending, from zero)
 *   W_eff[n,k] = bf16(fma(alpha_over_r, delta[n,k], W[n,k]))
 * then W_eff is quantized with 128x128 blocks (FPQ_FP8_128x128 rules).
 *
 *   w        bf16 [n, k] base weight (out_features x in_features)
 *   lora_a   bf16 [r, k]
 *   lora_b   bf16 [n, r]
 *   wq       uint8 e4m3 [n, k] (output)
 *   ws       fp32 [ceil(n/128), k/128] (output)
 *   w_fq     bf16 [n, k] fake-quantized weight dequant(wq, ws) (optional
 *            output for an autograd caller; NULL skips it)
 *
 * Requires k % 128 == 0, 1 <= r <= 64.  Errors: as fpq_quantize_block.
 */
FPQ_API fpq_status fpq_lora_merge_fakequant(const void* w, const void* lora_a, const void* lora_b,
                                    int64_t n, int64_t k, int32_t r, float alpha_over_r,
                                    void* wq, float* ws, void* w_fq, void* stream);

/*
 * fpq_scaled_gemm -- C = A * B^T on block-quantized operands with fp32
 * accumulation [B5 "Hardware Optimization"; DS "Инференс с FP8" (FP8
 * matrix multiplication)]:
 *   C[m,n] = sum_k decA[m,k] * decB[n,k],  dec = decode(code) * block scale.
 *
 *   aq, as   A [m, k] codes and scales in format fmt_a
 *   bq, bs   B [n, k] codes and scales in format fmt_b (weights, K-major)
 *   c        [m, n] bf16 (FPQ_OUT_BF16, round-to-nearest-even) or fp32
 *
 * Supported pairs: (FPQ_MXFP8, FPQ_MXFP8) -- the block-scaled tensor-core
 * path; (FPQ_FP8_1x128, FPQ_FP8_128x128) -- per-128-K partial sums promoted
 * to fp32 with the product of the two scales.  Others: FPQ_ERR_UNSUPPORTED.
 * Requires k % 128 == 0, n % 16 == 0, m >= 1.
 */
FPQ_API fpq_status fpq_scaled_gemm(fpq_format fmt_a, const void* aq, const void* as,
                           fpq_format fmt_b, const void* bq, const void* bs,
                           int64_t m, int64_t n, int64_t k, void* c, int32_t c_dtype,
                           void* stream);

/*
 * fpq_scaled_gemm_nvfp4 -- C = gA gB (A * B^T) on NVFP4 operands with fp32
 * accumulation ["fireworks-prequant 0.1.0" Formats: nvfp4 = packed FP4 +
 * FP8 block scales]:
 *   C[m,n] = gA gB sum_k e2m1(A[m,k]) sA[m,k/16] e2m1(B[n,k]) sB[n,k/16].
 *
 *   aq   uint8 [m, k/2] packed E2M1 (element 2i in the low nibble of byte i)
 *   as   uint8 E4M3 [m, k/16] block scales
 *   ag   fp32 device scalar: A's tensor scale g (as written by
 *        fpq_quantize_block with FPQ_NVFP4)
 *   bq, bs, bg   the same for B [n, k] (weights, K-major)
 *   c    [m, n] bf16 (FPQ_OUT_BF16, round-to-nearest-even) or fp32
 *
 * The tensor cores multiply the codes with their block scales exactly and
 * accumulate in fp32; the epilogue multiplies by fp32(gA gB).  Requires
 * k % 128 == 0, n % 16 == 0, m >= 1; ag and bg 4-byte aligned, the other
 * pointers 16-byte aligned.  Errors: as fpq_scaled_gemm.
 */
FPQ_API fpq_status fpq_scaled_gemm_nvfp4(const void* aq, const void* as, const float* ag, const void* bq,
                                         const void* bs, const float* bg, int64_t m, int64_t n, int64_t k,
                                         void* c, int32_t c_dtype, void* stream);

/*
 * fpq_gemm_bf16 -- C = alpha * (P * Q^T) on bf16 operands with fp32
 * accumulation on the tensor cores (the products of the QAT backward below).
 *
 *   p    bf16 [m, k] row-major (K contiguous)
 *   q    bf16 [n, k] row-major (K contiguous)
 *   c    bf16 [m, n] (round-to-nearest-even of fp32(alpha * fp32 sum))
 *
 * Requires m >= 1, n and k positive multiples of 8, 16-byte aligned
 * pointers.  Errors: FPQ_ERR_INVALID_ARG, FPQ_ERR_ALIGNMENT, FPQ_ERR_CUDA;
 * device-side wait timeouts go to the device error word.
 */
FPQ_API fpq_status fpq_gemm_bf16(const void* p, const void* q, int64_t m, int64_t n, int64_t k, float alpha,
                                 void* c, void* stream);

/*
 * fpq_gemm_bf16_layout -- as fpq_gemm_bf16 with each operand in either
 * layout: p_mn = 0: P stored [m, k] (K contiguous); p_mn = 1: P stored
 * [k, m] (m contiguous, i.e. the product uses its transpose); likewise q_mn
 * for Q ([n, k] or [k, n]).  Requires additionally m a multiple of 8 when
 * p_mn = 1.
 */
FPQ_API fpq_status fpq_gemm_bf16_layout(const void* p, int32_t p_mn, const void* q, int32_t q_mn, int64_t m,
                                        int64_t n, int64_t k, float alpha, void* c, void* stream);

/*
 * fpq_gemm_bf16_splitk -- as fpq_gemm_bf16_layout for products with few
 * output tiles and a long contraction (m or n small, as for the LoRA
 * gradients of the QAT backward): the contraction is cut into up to 16
 * slices spread over the SMs (about one CTA per SM; a product with many
 * output tiles takes one slice), each slice's fp32 sums go to the workspace,
 * and a second kernel adds the slices in order, multiplies by alpha and
 * rounds to bf16 (so results are repeatable run to run).
 *
 *   workspace   fpq_gemm_bf16_splitk_workspace_bytes(m, n, k) bytes,
 *               16-byte aligned, caller-owned, not read before written
 *
 * Requirements and errors: as fpq_gemm_bf16_layout, plus FPQ_ERR_WORKSPACE.
 */
FPQ_API size_t fpq_gemm_bf16_splitk_workspace_bytes(int64_t m, int64_t n, int64_t k);
FPQ_API fpq_status fpq_gemm_bf16_splitk(const void* p, int32_t p_mn, const void* q, int32_t q_mn, int64_t m,
                                        int64_t n, int64_t k, float alpha, void* c, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * fpq_transpose_bf16 -- out[c, r] = in[r, c] for bf16 [rows, cols] (the data
 * movement of the QAT backward below, exposed for callers that schedule its
 * products themselves).  Requires rows and cols positive multiples of 8,
 * 16-byte aligned pointers, in and out not overlapping.  Errors:
 * FPQ_ERR_INVALID_ARG, FPQ_ERR_ALIGNMENT, FPQ_ERR_CUDA.
 */
FPQ_API fpq_status fpq_transpose_bf16(const void* in, void* out, int64_t rows, int64_t cols, void* stream);

/*
 * fpq_qat_backward -- backward of the QAT linear layer with the
 * straight-through estimator ["DeepSeek R1 and V3 get quantization-aware
 * fine-tuning on Fireworks", Synopsis and Interpretation: LoRA adapters
 * trained through the FP8-quantized forward, the base weight frozen].  The
 * forward is y = fq(x) fq(W_eff)^T with W_eff = W + (alpha/r) B A
 * (fpq_lora_merge_fakequant + the 1x128 fake-quant of x + fpq_scaled_gemm);
 * the fake-quantizers pass gradients unchanged, so for the output gradient
 * dy:
 *   dx = dy Wfq,   dw = dy^T Xfq,   da = (alpha/r) B^T dw,   db = (alpha/r) dw A^T
 * each with fp32 accumulation and rounded to bf16; da and db use the bf16 dw.
 *
 *   dy      bf16 [m, n]      gradient of the layer output
 *   x_fq    bf16 [m, k]      fake-quantized activations (dequantized 1x128 codes)
 *   w_fq    bf16 [n, k]      fake-quantized merged weight (w_fq output of
 *                            fpq_lora_merge_fakequant)
 *   lora_a  bf16 [r, k], lora_b bf16 [n, r]
 *   dx      bf16 [m, k];  dw bf16 [n, k] (gradient of W_eff);
 *   da      bf16 [r, k];  db bf16 [n, r]
 *   workspace   fpq_qat_backward_workspace_bytes(m, n, k, r) bytes, 16-byte
 *               aligned, caller-owned, not read before written: fp32 partial
 *               sums of da and db (for r <= 64 those of fpq_qat_lora_grads,
 *               sized for the current device's SM count; for larger r the
 *               split-K slices of two bf16 GEMMs, at most 16 each), added in
 *               a fixed order by a second kernel, so results are repeatable;
 *               then the tile counters of the dX and dW products (zeroed by
 *               the call), from which their persistent CTAs claim tiles
 *
 * The products are ordered on `stream` like any other work: dx, which no
 * other product needs, runs on a library-owned second stream forked from
 * `stream` by an event and joined back before the call returns (so the call
 * may also be captured into a CUDA graph).
 *
 * Requires m, n, k positive multiples of 8 and r a multiple of 8 in [8, 256];
 * every pointer 16-byte aligned.  Errors: FPQ_ERR_INVALID_ARG,
 * FPQ_ERR_ALIGNMENT, FPQ_ERR_WORKSPACE, FPQ_ERR_CUDA; device-side wait
 * timeouts go to the device error word.
 */
/*
 * fpq_qat_lora_grads -- the two LoRA gradients of the QAT backward in one
 * pass over the weight gradient [same source, same numerics as in
 * fpq_qat_backward]:  da = (alpha/r) B^T dw,  db = (alpha/r) dw A^T, fp32
 * accumulation, bf16 out.  Each 128 x 128 tile of dw is read once and feeds
 * both tensor-core products (one CTA per 128-row strip of dw and range of K
 * tiles); the fp32 partial sums go to the workspace and a second kernel adds
 * them in a fixed order (repeatable results).
 *
 *   dw      bf16 [n, k];  lora_a bf16 [r, k];  lora_b bf16 [n, r]
 *   da      bf16 [r, k];  db bf16 [n, r]
 *   workspace   fpq_qat_lora_grads_workspace_bytes(n, k, r) bytes (the
 *               current device's SM count enters the size), 16-byte aligned,
 *               caller-owned, not read before written
 *
 * Requires n, k positive multiples of 8, r a multiple of 8 in [8, 64], every
 * pointer 16-byte aligned.  Errors: FPQ_ERR_INVALID_ARG, FPQ_ERR_ALIGNMENT,
 * FPQ_ERR_WORKSPACE, FPQ_ERR_CUDA; device-side wait timeouts go to the device
 * error word.
 */
FPQ_API size_t fpq_qat_lora_grads_workspace_bytes(int64_t n, int64_t k, int32_t r);
FPQ_API fpq_status fpq_qat_lora_grads(const void* dw, const void* lora_a, const void* lora_b, int64_t n, int64_t k,
                                      int32_t r, float alpha_over_r, void* da, void* db, void* workspace,
                                      size_t workspace_bytes, void* stream);

FPQ_API size_t fpq_qat_backward_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r);
FPQ_API fpq_status fpq_qat_backward(const void* dy, const void* x_fq, const void* w_fq, const void* lora_a,
                                    const void* lora_b, int64_t m, int64_t n, int64_t k, int32_t r,
                                    float alpha_over_r, void* dx, void* dw, void* da, void* db, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * MoE FP8 dispatch ["DeepSeek-V3 Blog 5: Low-Precision Training", Reducing
 * Communication Overhead in MoE with FP8: token activations are quantized to
 * FP8 before they are sent to the GPUs that hold their experts].  Tokens are
 * quantized to MXFP8 (E4M3 codes, E8M0 scale per 32, as fpq_quantize_block
 * FPQ_MXFP8) and each token's codes and scales are written once per chosen
 * expert, to the rows of that expert.
 *
 * Row order: with `world` ranks and E experts, rank r owns experts
 * [r L, (r + 1) L), L = E / world.  A rank's receive buffer holds its local
 * experts' rows in expert order; each expert's rows come from source rank
 * 0, 1, ... in turn; from one source, the (token, choice) pairs routed to
 * that expert in token order, then choice order (the pair's slot).  The
 * buffer is the `aq`/`as` operand of fpq_grouped_scaled_gemm (FPQ_MXFP8)
 * with `recv_offsets` as its group offsets.
 *
 * Calls, on the source rank's stream:
 *   fpq_moe_route          per-expert counts of this rank's pairs, and the
 *                          slot bases in the workspace;
 *   (the ranks exchange counts: counts_all [world, E], e.g. an all-gather)
 *   fpq_moe_dispatch_layout  destination row of slot 0 of every expert, and
 *                          this rank's group offsets;
 *   fpq_moe_dispatch_mxfp8 quantize + write every pair's row.
 *
 *   topk_ids    DEVICE int32 [tokens, topk], expert ids in [0, E); an id out
 *               of range raises FPQ_ERR_DEVICE_BAD_INPUT and its pair is
 *               dropped
 *   counts      DEVICE int32 [E] (out)
 *   workspace   fpq_moe_route_workspace_bytes(tokens, E) bytes, 16-byte
 *               aligned, caller-owned; fpq_moe_route writes it and
 *               fpq_moe_dispatch_mxfp8 (same tokens, topk, E) reads it
 *   counts_all  DEVICE int32 [world, E]: row s = source rank s's counts
 *   mode        FPQ_MOE_DIRECT: rows go straight into the receivers'
 *               buffers (one GPU, or peer memory); dst_row0[e] = row of
 *               slot 0 of expert e, from this rank, in rank e / L's buffer.
 *               FPQ_MOE_PACK: rows go into this rank's send buffer, expert-
 *               major in slot order (for a collective that moves each
 *               (expert, source) segment to its receiver); dst_row0[e] =
 *               rows of this rank's experts before e
 *   dst_row0    DEVICE int64 [E] (out);  recv_offsets DEVICE int32 [L + 1]
 *               (out): row of local expert l in this rank's receive buffer
 *   x           DEVICE bf16 [tokens, hidden], hidden a positive multiple of 32
 *   n_dest      number of destination buffers; expert e goes to buffer
 *               e / (E / n_dest) (DIRECT: n_dest = world; PACK: 1)
 *   dst_codes, dst_scales  DEVICE arrays of n_dest DEVICE pointers: uint8
 *               [rows, hidden] codes and uint8 [rows, hidden/32] E8M0 scales
 *               (16-byte aligned code buffers); peer pointers are allowed
 *   dst_capacity  DEVICE int64 [n_dest]: rows of each buffer; a row outside
 *               raises FPQ_ERR_DEVICE_BAD_INPUT and is not written
 *
 * Requires tokens >= 0, 1 <= topk <= 32, tokens * topk < 2^31 (counts and
 * group offsets are int32), 1 <= E <= 1024, world >= 1 dividing
 * E, 0 <= rank < world, n_dest >= 1 dividing E; the pointer arguments of
 * fpq_moe_dispatch_mxfp8 16-byte aligned.  Errors: FPQ_ERR_INVALID_ARG,
 * FPQ_ERR_ALIGNMENT, FPQ_ERR_WORKSPACE, FPQ_ERR_CUDA.
 */
#define FPQ_MOE_DIRECT 0
#define FPQ_MOE_PACK 1
FPQ_API size_t fpq_moe_route_workspace_bytes(int64_t tokens, int32_t num_experts);
FPQ_API fpq_status fpq_moe_route(const int32_t* topk_ids, int64_t tokens, int32_t topk, int32_t num_experts,
                                 int32_t* counts, void* workspace, size_t workspace_bytes, void* stream);
FPQ_API fpq_status fpq_moe_dispatch_layout(const int32_t* counts_all, int32_t world, int32_t num_experts,
                                           int32_t rank, int32_t mode, int64_t* dst_row0, int32_t* recv_offsets,
                                           void* stream);
FPQ_API fpq_status fpq_moe_dispatch_mxfp8(const void* x, int64_t tokens, int64_t hidden, const int32_t* topk_ids,
                                          int32_t topk, int32_t num_experts, const void* workspace,
                                          size_t workspace_bytes, const int64_t* dst_row0, int32_t n_dest,
                                          void* const* dst_codes, void* const* dst_scales,
                                          const int64_t* dst_capacity, void* stream);

/*
 * fpq_moe_regroup -- the receiving side of the exchange in the PACK mode
 * ["DeepSeek-V3 Blog 5: Low-Precision Training", Reducing Communication
 * Overhead in MoE with FP8].  A PACK send buffer holds a rank's rows expert-
 * major, so the rows bound for rank p (experts [p L, (p + 1) L)) are one
 * contiguous run, and one all-to-all with per-rank row counts delivers them.
 * The receiver then holds its rows source-major: all of source 0's rows for
 * its experts (expert-major, slot order), then source 1's, ...  This call
 * moves them into the receive layout above (expert-major; within an expert,
 * source 0, 1, ...): segment (local expert l, source s) of
 * counts_all[s][rank L + l] rows.
 *
 *   recv_codes, recv_scales  DEVICE uint8 [rows, hidden] E4M3 codes and
 *               [rows, hidden / 32] E8M0 scales, source-major (input)
 *   counts_all  DEVICE int32 [world, E] (as for fpq_moe_dispatch_layout)
 *   rows        rows of the input and of the output buffers:
 *               sum over s and l of counts_all[s][rank L + l]
 *   codes, scales  DEVICE, same shapes (output; must not overlap the input)
 *
 * Requires world >= 1 dividing E, 1 <= E <= 1024, 0 <= rank < world, hidden
 * a positive multiple of 32, 0 <= rows < 2^31, 16-byte aligned code
 * buffers.  A negative count, or a segment past `rows`, is malformed device
 * input: FPQ_ERR_DEVICE_BAD_INPUT in the device error word, that segment not
 * copied.  Errors: FPQ_ERR_INVALID_ARG, FPQ_ERR_ALIGNMENT, FPQ_ERR_CUDA.
 */
FPQ_API fpq_status fpq_moe_regroup(const void* recv_codes, const void* recv_scales, const int32_t* counts_all,
                                   int32_t world, int32_t num_experts, int32_t rank, int64_t hidden, int64_t rows,
                                   void* codes, void* scales, void* stream);

/*
 * fpq_grouped_scaled_gemm -- per-expert product over a token-permuted
 * activation matrix (MoE routed experts) [FP "Quick start": routed MoE
 * expert projections; DS "Как FP8 связан с MoE-архитектурой DeepSeek V3"]:
 *   for every expert g and row m in [off[g], off[g+1]):
 *     C[m, :] = A[m, :] * B[g]^T
 *
 *   aq, as          A [total_m, k] codes/scales (fmt)
 *   bq, bs          B [groups, n, k] codes/scales (fmt)
 *   group_offsets   DEVICE int32 [groups + 1], off[0] = 0, non-decreasing,
 *                   off[groups] = total_m (empty experts are legal);
 *                   a violation is reported through the device error word
 *                   (FPQ_ERR_DEVICE_BAD_INPUT) and C is left unspecified
 *   c               [total_m, n] bf16 or fp32
 *
 * Supported: fmt = FPQ_MXFP8.  Requires k % 128 == 0, n % 16 == 0.
 */
FPQ_API fpq_status fpq_grouped_scaled_gemm(fpq_format fmt, const void* aq, const void* as,
                                   const void* bq, const void* bs,
                                   const int32_t* group_offsets, int32_t groups,
                                   int64_t total_m, int64_t n, int64_t k, void* c,
                                   int32_t c_dtype, void* stream);

/*
 * fpq_quantize_nvfp4_noalloc -- NVFP4 quantization (same outputs, layouts and
 * errors as fpq_quantize_block with FPQ_NVFP4) for callers that cannot
 * allocate device memory and so cannot pass the amax workspace, such as a
 * plugin running inside a host application that owns the device memory pool.
 * The pages describe no such entry point; it exists for these callers only.
 *
 * Scratch: a library-owned static device array of 4 + 2 *
 * FPQ_NOALLOC_NVFP4_MAX_BATCH 32-bit words (32 KiB + 16 bytes: the NVFP4
 * workspace for the largest batch) on every GPU that loads the library, held
 * until the process
 * exits.  No call allocates or frees anything.  batch > the maximum gives
 * FPQ_ERR_INVALID_ARG.  The first call of this function on a device looks
 * up the array's device address (cudaGetSymbolAddress) with that device
 * current and caches it per device ordinal; that lookup is separate from the
 * one every other entry point makes for the device error word, so a caller
 * that has already used other entry points on the device must still make
 * one call of this function outside any stream capture before capturing it.
 * The cached address assumes the device's primary context for the life of
 * the process: after cudaDeviceReset, or under a non-primary driver context
 * on the same ordinal, it no longer names the live array.  All calls on a
 * device share the array, so calls that may overlap on the GPU (different
 * streams, no ordering between them) race and must not be issued; calls on
 * one stream are safe.
 */
#define FPQ_NOALLOC_NVFP4_MAX_BATCH 4096
FPQ_API fpq_status fpq_quantize_nvfp4_noalloc(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                              void* q, void* scales, float* tensor_scale, void* stream);

/*
 * fpq_get_device_error -- synchronize `stream`, then read and clear the
 * current device's error word.  *code receives FPQ_OK or the first
 * FPQ_ERR_DEVICE_* raised by a kernel since the last read.  Returns
 * FPQ_ERR_CUDA if the synchronization itself fails.
 */
FPQ_API fpq_status fpq_get_device_error(void* stream, int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* FPQ_H */
