// api.cu -- the C ABI declared in include/fpq.h: argument validation, status
// codes, per-device state (SM count, error-word address) and dispatch to the
// kernel launchers.  No allocation, no synchronization (except in
// fpq_get_device_error), no CPU fallback.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/fpq.h"
#include "internal.h"

namespace {

// Device-side error word: the first FPQ_ERR_DEVICE_* a kernel raises.
__device__ uint32_t g_device_error = 0;

thread_local char t_detail[512] = "";

void set_detail(const char* what, cudaError_t e) {
    std::snprintf(t_detail, sizeof(t_detail), "%s: %s (%s)", what, cudaGetErrorName(e),
                  cudaGetErrorString(e));
}
void set_detail(const char* what) { std::snprintf(t_detail, sizeof(t_detail), "%s", what); }

constexpr int kMaxDevices = 64;
struct DeviceState {
    bool ready = false;
    bool supported = false;
    int sms = 0;
    uint32_t* err = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device's state; nullptr (with the detail set) if unusable.
const DeviceState* device_state(fpq_status* st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_detail("no CUDA device", e);
        *st = FPQ_ERR_UNSUPPORTED;
        return nullptr;
    }
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        std::lock_guard<std::mutex> lock(g_dev_mu);
        if (!d.ready) {
            int major = 0, minor = 0, sms = 0;
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            d.supported = (major == 10 && minor == 0);
            d.sms = sms;
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_device_error);
            if (e != cudaSuccess) {
                set_detail("cudaGetSymbolAddress(device error word)", e);
                *st = FPQ_ERR_CUDA;
                return nullptr;
            }
            d.err = (uint32_t*)p;
            d.ready = true;
        }
    }
    if (!d.supported) {
        set_detail("device is not sm_100 (B200/GB200); this library has no other code path");
        *st = FPQ_ERR_UNSUPPORTED;
        return nullptr;
    }
    return &d;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

fpq_status check_ptrs(std::initializer_list<const void*> ps) {
    for (const void* p : ps) {
        if (!p) { set_detail("null pointer argument"); return FPQ_ERR_INVALID_ARG; }
        if (!aligned16(p)) { set_detail("pointer not 16-byte aligned"); return FPQ_ERR_ALIGNMENT; }
    }
    return FPQ_OK;
}

fpq_status from_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return FPQ_OK;
    if (e == cudaErrorNotSupported) { set_detail(what, e); return FPQ_ERR_UNSUPPORTED; }
    set_detail(what, e);
    return FPQ_ERR_CUDA;
}

int block_cols(fpq_format f) {
    switch (f) {
    case FPQ_FP8_1x128: case FPQ_FP8_128x128: return 128;
    case FPQ_MXFP8: return 32;
    case FPQ_NVFP4: return 32;
    default: return 0;
    }
}

fpq_status check_quant_shape(fpq_format fmt, int64_t batch, int64_t rows, int64_t cols) {
    const int bc = block_cols(fmt);
    if (bc == 0) { set_detail("unknown format"); return FPQ_ERR_INVALID_ARG; }
    if (batch < 1 || rows < 1 || cols < 1) { set_detail("batch, rows and cols must be >= 1"); return FPQ_ERR_INVALID_ARG; }
    if (cols % bc) { set_detail("cols is not a multiple of the format's block width"); return FPQ_ERR_INVALID_ARG; }
    if (batch > (1ll << 40) / rows / cols) { set_detail("tensor too large"); return FPQ_ERR_INVALID_ARG; }
    return FPQ_OK;
}

}  // namespace

namespace fpq {
// Lets other translation units of the library report a detail string through
// fpq_last_error_detail().
void set_error_detail(const char* what) { set_detail(what); }
}  // namespace fpq

extern "C" {

int32_t fpq_version(void) { return 10000; }

const char* fpq_status_string(fpq_status s) {
    switch (s) {
    case FPQ_OK: return "ok";
    case FPQ_ERR_INVALID_ARG: return "invalid argument";
    case FPQ_ERR_ALIGNMENT: return "misaligned pointer";
    case FPQ_ERR_UNSUPPORTED: return "unsupported device or format";
    case FPQ_ERR_CUDA: return "CUDA error";
    case FPQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case FPQ_ERR_DEVICE_BAD_INPUT: return "malformed device input";
    case FPQ_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
    }
}

const char* fpq_last_error_detail(void) { return t_detail; }
const char* fpq_last_cuda_error(void) { return t_detail; }

size_t fpq_quantize_workspace_bytes(fpq_format fmt, int64_t batch) {
    return (fmt == FPQ_NVFP4 && batch > 0) ? sizeof(uint32_t) * (size_t)fpq::nvfp4_workspace_words(batch) : 0;
}

fpq_status fpq_quantize_block(fpq_format fmt, const void* x, int64_t batch, int64_t rows, int64_t cols,
                              void* q, void* scales, float* tensor_scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
    t_detail[0] = 0;
    fpq_status st = check_quant_shape(fmt, batch, rows, cols);
    if (st != FPQ_OK) return st;
    if ((st = check_ptrs({x, q, scales})) != FPQ_OK) return st;
    if (fmt == FPQ_NVFP4) {
        if ((st = check_ptrs({tensor_scale})) != FPQ_OK) return st;
        if (!workspace || workspace_bytes < fpq_quantize_workspace_bytes(fmt, batch) || !aligned16(workspace)) {
            set_detail("NVFP4 needs a 16-byte aligned workspace of fpq_quantize_workspace_bytes() bytes");
            return FPQ_ERR_WORKSPACE;
        }
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_quantize(fmt, x, batch, rows, cols, q, scales, tensor_scale, workspace,
                                          d->err, d->sms, (cudaStream_t)stream), "quantize launch");
}

fpq_status fpq_dequantize(fpq_format fmt, const void* q, const void* scales, const float* tensor_scale,
                          int64_t batch, int64_t rows, int64_t cols, void* out, void* stream) {
    t_detail[0] = 0;
    fpq_status st = check_quant_shape(fmt, batch, rows, cols);
    if (st != FPQ_OK) return st;
    if ((st = check_ptrs({q, scales, out})) != FPQ_OK) return st;
    if (fmt == FPQ_NVFP4 && (st = check_ptrs({tensor_scale})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_dequantize(fmt, q, scales, tensor_scale, batch, rows, cols, out, d->sms,
                                            (cudaStream_t)stream), "dequantize launch");
}

namespace {
fpq_status check_strides(int64_t batch, int64_t rows, int64_t cols, int64_t ld, int64_t bs, const char* what) {
    if (ld < cols || ld % 16 || ld > (1ll << 40) || (batch > 1 && (bs < rows * ld || bs % 16 || bs > (1ll << 44)))) {
        set_detail(what);
        return FPQ_ERR_INVALID_ARG;
    }
    return FPQ_OK;
}
}  // namespace

fpq_status fpq_quantize_block_strided(fpq_format fmt, const void* x, int64_t ld_x, int64_t bs_x, int64_t batch,
                                      int64_t rows, int64_t cols, void* q, int64_t ld_q, int64_t bs_q, void* scales,
                                      float* tensor_scale, void* workspace, size_t workspace_bytes, void* stream) {
    t_detail[0] = 0;
    fpq_status st = check_quant_shape(fmt, batch, rows, cols);
    if (st != FPQ_OK) return st;
    if ((st = check_strides(batch, rows, cols, ld_x, bs_x, "x strides: need ld >= cols, ld and bs multiples of 16, "
                                                            "bs >= rows * ld")) != FPQ_OK)
        return st;
    if ((st = check_strides(batch, rows, cols, ld_q, bs_q, "q strides: need ld >= cols, ld and bs multiples of 16, "
                                                            "bs >= rows * ld")) != FPQ_OK)
        return st;
    if ((st = check_ptrs({x, q, scales})) != FPQ_OK) return st;
    if (fmt == FPQ_NVFP4) {
        if ((st = check_ptrs({tensor_scale})) != FPQ_OK) return st;
        if (!workspace || workspace_bytes < fpq_quantize_workspace_bytes(fmt, batch) || !aligned16(workspace)) {
            set_detail("NVFP4 needs a 16-byte aligned workspace of fpq_quantize_workspace_bytes() bytes");
            return FPQ_ERR_WORKSPACE;
        }
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    const fpq::OperandStrides os{ld_x, batch > 1 ? bs_x : rows * ld_x, ld_q, batch > 1 ? bs_q : rows * ld_q};
    return from_cuda(fpq::launch_quantize(fmt, x, batch, rows, cols, q, scales, tensor_scale, workspace, d->err,
                                          d->sms, (cudaStream_t)stream, &os),
                     "quantize launch");
}

fpq_status fpq_dequantize_strided(fpq_format fmt, const void* q, int64_t ld_q, int64_t bs_q, const void* scales,
                                  const float* tensor_scale, int64_t batch, int64_t rows, int64_t cols, void* out,
                                  int64_t ld_out, int64_t bs_out, void* stream) {
    t_detail[0] = 0;
    fpq_status st = check_quant_shape(fmt, batch, rows, cols);
    if (st != FPQ_OK) return st;
    if ((st = check_strides(batch, rows, cols, ld_q, bs_q, "q strides: need ld >= cols, ld and bs multiples of 16, "
                                                            "bs >= rows * ld")) != FPQ_OK)
        return st;
    if ((st = check_strides(batch, rows, cols, ld_out, bs_out, "out strides: need ld >= cols, ld and bs multiples of "
                                                                "16, bs >= rows * ld")) != FPQ_OK)
        return st;
    if ((st = check_ptrs({q, scales, out})) != FPQ_OK) return st;
    if (fmt == FPQ_NVFP4 && (st = check_ptrs({tensor_scale})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    const fpq::OperandStrides os{ld_q, batch > 1 ? bs_q : rows * ld_q, ld_out, batch > 1 ? bs_out : rows * ld_out};
    return from_cuda(fpq::launch_dequantize(fmt, q, scales, tensor_scale, batch, rows, cols, out, d->sms,
                                            (cudaStream_t)stream, &os),
                     "dequantize launch");
}

fpq_status fpq_lora_merge_fakequant(const void* w, const void* lora_a, const void* lora_b, int64_t n,
                                    int64_t k, int32_t r, float alpha_over_r, void* wq, float* ws,
                                    void* w_fq, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (n < 1 || k < 128 || k % 128 || r < 1 || r > 64) {
        set_detail("need n >= 1, k a positive multiple of 128, 1 <= r <= 64");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({w, lora_a, lora_b, wq, ws})) != FPQ_OK) return st;
    if (w_fq && !aligned16(w_fq)) { set_detail("w_fq not 16-byte aligned"); return FPQ_ERR_ALIGNMENT; }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_lora_merge_fakequant(w, lora_a, lora_b, n, k, r, alpha_over_r, wq, ws, w_fq,
                                                      d->sms, (cudaStream_t)stream), "lora merge launch");
}

fpq_status fpq_scaled_gemm(fpq_format fmt_a, const void* aq, const void* as, fpq_format fmt_b,
                           const void* bq, const void* bs, int64_t m, int64_t n, int64_t k, void* c,
                           int32_t c_dtype, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 1 || n < 16 || n % 16 || k < 128 || k % 128 || (c_dtype != FPQ_OUT_BF16 && c_dtype != FPQ_OUT_F32) ||
        m > (1 << 30) || n > (1 << 30) || k > (1 << 30)) {
        set_detail("need m >= 1, n a positive multiple of 16, k a positive multiple of 128, c_dtype BF16|F32");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({aq, as, bq, bs, c})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    const int f32 = c_dtype == FPQ_OUT_F32;
    if (fmt_a == FPQ_MXFP8 && fmt_b == FPQ_MXFP8)
        return from_cuda(fpq::launch_gemm_mxfp8(aq, as, bq, bs, m, n, k, c, f32, d->err, d->sms,
                                                (cudaStream_t)stream), "mxfp8 gemm launch");
    if (fmt_a == FPQ_FP8_1x128 && fmt_b == FPQ_FP8_128x128)
        return from_cuda(fpq::launch_gemm_fp8_f32scale(aq, (const float*)as, bq, (const float*)bs, m, n, k, c, f32,
                                                       d->err, d->sms, (cudaStream_t)stream),
                         "fp8 blockscale gemm launch");
    set_detail("supported format pairs: (MXFP8, MXFP8) and (FP8_1x128, FP8_128x128)");
    return FPQ_ERR_UNSUPPORTED;
}

fpq_status fpq_scaled_gemm_nvfp4(const void* aq, const void* as, const float* ag, const void* bq, const void* bs,
                                 const float* bg, int64_t m, int64_t n, int64_t k, void* c, int32_t c_dtype,
                                 void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 1 || n < 16 || n % 16 || k < 128 || k % 128 || (c_dtype != FPQ_OUT_BF16 && c_dtype != FPQ_OUT_F32) ||
        m > (1 << 30) || n > (1 << 30) || k > (1 << 30)) {
        set_detail("need m >= 1, n a positive multiple of 16, k a positive multiple of 128, c_dtype BF16|F32");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({aq, as, bq, bs, c})) != FPQ_OK) return st;
    if (!ag || !bg) { set_detail("null tensor scale pointer"); return FPQ_ERR_INVALID_ARG; }
    if ((reinterpret_cast<uintptr_t>(ag) & 3) || (reinterpret_cast<uintptr_t>(bg) & 3)) {
        set_detail("tensor scale pointers must be 4-byte aligned");
        return FPQ_ERR_ALIGNMENT;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_gemm_nvfp4(aq, as, ag, bq, bs, bg, m, n, k, c, c_dtype == FPQ_OUT_F32, d->err,
                                            (cudaStream_t)stream), "nvfp4 gemm launch");
}

fpq_status fpq_gemm_bf16(const void* p, const void* q, int64_t m, int64_t n, int64_t k, float alpha, void* c,
                         void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 1 || n < 8 || n % 8 || k < 8 || k % 8 || m > (1 << 30) || n > (1 << 30) || k > (1 << 30)) {
        set_detail("need m >= 1, n and k positive multiples of 8");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({p, q, c})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_gemm_bf16(p, false, q, false, m, n, k, alpha, c, d->err, (cudaStream_t)stream),
                     "bf16 gemm launch");
}

fpq_status fpq_gemm_bf16_layout(const void* p, int32_t p_mn, const void* q, int32_t q_mn, int64_t m, int64_t n,
                                int64_t k, float alpha, void* c, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 1 || n < 8 || n % 8 || k < 8 || k % 8 || (p_mn && m % 8) || m > (1 << 30) || n > (1 << 30) ||
        k > (1 << 30) || (p_mn != 0 && p_mn != 1) || (q_mn != 0 && q_mn != 1)) {
        set_detail("need n, k positive multiples of 8, m >= 1 (a multiple of 8 when P is MN-major), flags 0|1");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({p, q, c})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_gemm_bf16(p, p_mn != 0, q, q_mn != 0, m, n, k, alpha, c, d->err,
                                           (cudaStream_t)stream),
                     "bf16 gemm launch");
}

size_t fpq_moe_route_workspace_bytes(int64_t tokens, int32_t num_experts) {
    if (tokens < 0 || num_experts < 1 || num_experts > 1024) return 0;
    return fpq::moe_route_workspace_bytes(tokens, num_experts);
}

fpq_status fpq_moe_route(const int32_t* topk_ids, int64_t tokens, int32_t topk, int32_t num_experts,
                         int32_t* counts, void* workspace, size_t workspace_bytes, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (tokens < 0 || topk < 1 || topk > 32 || tokens * topk >= (1ll << 31) || num_experts < 1 ||
        num_experts > 1024) {
        set_detail("need tokens >= 0, topk in [1, 32], tokens * topk < 2^31 (int32 counts), num_experts in "
                   "[1, 1024]");
        return FPQ_ERR_INVALID_ARG;
    }
    if (!counts || (tokens > 0 && !topk_ids)) {
        set_detail("null pointer");
        return FPQ_ERR_INVALID_ARG;
    }
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < fpq::moe_route_workspace_bytes(tokens, num_experts)) {
        set_detail("need a 16-byte aligned workspace of fpq_moe_route_workspace_bytes() bytes");
        return FPQ_ERR_WORKSPACE;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_moe_route(topk_ids, tokens, topk, num_experts, counts, workspace, d->err,
                                           (cudaStream_t)stream),
                     "moe route launch");
}

fpq_status fpq_moe_dispatch_layout(const int32_t* counts_all, int32_t world, int32_t num_experts, int32_t rank,
                                   int32_t mode, int64_t* dst_row0, int32_t* recv_offsets, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (world < 1 || num_experts < 1 || num_experts > 1024 || num_experts % world || rank < 0 || rank >= world ||
        (mode != FPQ_MOE_DIRECT && mode != FPQ_MOE_PACK)) {
        set_detail("need world >= 1 dividing num_experts in [1, 1024], 0 <= rank < world, a known mode");
        return FPQ_ERR_INVALID_ARG;
    }
    if (!counts_all || !dst_row0 || !recv_offsets) {
        set_detail("null pointer");
        return FPQ_ERR_INVALID_ARG;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_moe_layout(counts_all, world, num_experts, rank, mode == FPQ_MOE_PACK, dst_row0,
                                            recv_offsets, (cudaStream_t)stream),
                     "moe layout launch");
}

fpq_status fpq_moe_dispatch_mxfp8(const void* x, int64_t tokens, int64_t hidden, const int32_t* topk_ids,
                                  int32_t topk, int32_t num_experts, const void* workspace, size_t workspace_bytes,
                                  const int64_t* dst_row0, int32_t n_dest, void* const* dst_codes,
                                  void* const* dst_scales, const int64_t* dst_capacity, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (tokens < 0 || hidden < 32 || hidden % 32 || hidden > (1 << 24) || topk < 1 || topk > 32 ||
        tokens * topk >= (1ll << 31) || num_experts < 1 || num_experts > 1024 || n_dest < 1 ||
        num_experts % n_dest) {
        set_detail("need tokens >= 0, hidden a positive multiple of 32, topk in [1, 32], num_experts in "
                   "[1, 1024], n_dest >= 1 dividing num_experts");
        return FPQ_ERR_INVALID_ARG;
    }
    if (tokens == 0) return FPQ_OK;
    if ((st = check_ptrs({x, topk_ids, dst_row0, dst_codes, dst_scales, dst_capacity})) != FPQ_OK) return st;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < fpq::moe_route_workspace_bytes(tokens, num_experts)) {
        set_detail("need the workspace that fpq_moe_route wrote");
        return FPQ_ERR_WORKSPACE;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_moe_dispatch_mxfp8(x, tokens, hidden, topk_ids, topk, num_experts, workspace,
                                                    dst_row0, n_dest, dst_codes, dst_scales, dst_capacity, d->err,
                                                    (cudaStream_t)stream),
                     "moe dispatch launch");
}

fpq_status fpq_moe_regroup(const void* recv_codes, const void* recv_scales, const int32_t* counts_all,
                           int32_t world, int32_t num_experts, int32_t rank, int64_t hidden, int64_t rows,
                           void* codes, void* scales, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (world < 1 || num_experts < 1 || num_experts > 1024 || num_experts % world || rank < 0 || rank >= world ||
        hidden < 32 || hidden % 32 || hidden > (1 << 24) || rows < 0 || rows >= (1ll << 31)) {
        set_detail("need world >= 1 dividing num_experts in [1, 1024], 0 <= rank < world, hidden a positive "
                   "multiple of 32, 0 <= rows < 2^31");
        return FPQ_ERR_INVALID_ARG;
    }
    if (rows == 0) return FPQ_OK;
    if ((st = check_ptrs({recv_codes, recv_scales, counts_all, codes, scales})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_moe_regroup(recv_codes, recv_scales, counts_all, world, num_experts, rank, hidden,
                                             rows, codes, scales, d->err, d->sms, (cudaStream_t)stream),
                     "moe regroup launch");
}

size_t fpq_gemm_bf16_splitk_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < 1) return 0;
    return (size_t)fpq::bf16_split_bound(m, n, k) * (size_t)m * (size_t)n * 4;
}

fpq_status fpq_gemm_bf16_splitk(const void* p, int32_t p_mn, const void* q, int32_t q_mn, int64_t m, int64_t n,
                                int64_t k, float alpha, void* c, void* workspace, size_t workspace_bytes,
                                void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 1 || n < 8 || n % 8 || k < 8 || k % 8 || (p_mn && m % 8) || m > (1 << 30) || n > (1 << 30) ||
        k > (1 << 30) || (p_mn != 0 && p_mn != 1) || (q_mn != 0 && q_mn != 1)) {
        set_detail("need n, k positive multiples of 8, m >= 1 (a multiple of 8 when P is MN-major), flags 0|1");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({p, q, c})) != FPQ_OK) return st;
    if (!workspace || !aligned16(workspace) || workspace_bytes < fpq_gemm_bf16_splitk_workspace_bytes(m, n, k)) {
        set_detail("need a 16-byte aligned workspace of fpq_gemm_bf16_splitk_workspace_bytes() bytes");
        return FPQ_ERR_WORKSPACE;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_gemm_bf16_splitk(p, p_mn != 0, q, q_mn != 0, m, n, k, alpha, c,
                                                  static_cast<float*>(workspace),
                                                  fpq::bf16_split_count(m, n, k, d->sms), d->err,
                                                  (cudaStream_t)stream),
                     "bf16 split-k gemm launch");
}

fpq_status fpq_transpose_bf16(const void* in, void* out, int64_t rows, int64_t cols, void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (rows < 8 || rows % 8 || cols < 8 || cols % 8 || rows > (1 << 30) || cols > (1 << 30)) {
        set_detail("need rows and cols positive multiples of 8");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({in, out})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_transpose_bf16(in, out, rows, cols, (cudaStream_t)stream), "transpose launch");
}

size_t fpq_qat_lora_grads_workspace_bytes(int64_t n, int64_t k, int32_t r) {
    if (n < 8 || k < 8 || r < 8 || r % 8 || !fpq::lora_grads_fused(r)) return 0;
    return fpq::lora_grads_workspace_bytes(n, k, r, fpq::current_sms());
}

fpq_status fpq_qat_lora_grads(const void* dw, const void* lora_a, const void* lora_b, int64_t n, int64_t k, int32_t r,
                              float alpha_over_r, void* da, void* db, void* workspace, size_t workspace_bytes,
                              void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (n < 8 || n % 8 || k < 8 || k % 8 || r < 8 || r % 8 || r > 64 || n > (1 << 30) || k > (1 << 30)) {
        set_detail("need n, k positive multiples of 8 and r a multiple of 8 in [8, 64]");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({dw, lora_a, lora_b, da, db})) != FPQ_OK) return st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    const size_t need = fpq::lora_grads_workspace_bytes(n, k, r, d->sms);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) {
        set_detail("need a 16-byte aligned workspace of fpq_qat_lora_grads_workspace_bytes() bytes");
        return FPQ_ERR_WORKSPACE;
    }
    return from_cuda(fpq::launch_lora_grads(dw, lora_a, lora_b, n, k, r, alpha_over_r, da, db, workspace, d->err,
                                            d->sms, (cudaStream_t)stream),
                     "lora gradients launch");
}

size_t fpq_qat_backward_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t r) {
    if (m < 1 || n < 1 || k < 1 || r < 1) return 0;
    return fpq::qat_backward_workspace_bytes(m, n, k, r);
}

fpq_status fpq_qat_backward(const void* dy, const void* x_fq, const void* w_fq, const void* lora_a,
                            const void* lora_b, int64_t m, int64_t n, int64_t k, int32_t r, float alpha_over_r,
                            void* dx, void* dw, void* da, void* db, void* workspace, size_t workspace_bytes,
                            void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (m < 8 || m % 8 || n < 8 || n % 8 || k < 8 || k % 8 || r < 8 || r % 8 || r > 256 || m > (1 << 30) ||
        n > (1 << 30) || k > (1 << 30)) {
        set_detail("need m, n, k positive multiples of 8 and r a multiple of 8 in [8, 256]");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({dy, x_fq, w_fq, lora_a, lora_b, dx, dw, da, db})) != FPQ_OK) return st;
    const size_t need = fpq::qat_backward_workspace_bytes(m, n, k, r);
    if (need > 0 && (!workspace || !aligned16(workspace) || workspace_bytes < need)) {
        set_detail("need a 16-byte aligned workspace of fpq_qat_backward_workspace_bytes() bytes");
        return FPQ_ERR_WORKSPACE;
    }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_qat_backward(dy, x_fq, w_fq, lora_a, lora_b, m, n, k, r, alpha_over_r, dx, dw, da,
                                              db, workspace, d->err, d->sms, (cudaStream_t)stream),
                     "qat backward launch");
}

fpq_status fpq_grouped_scaled_gemm(fpq_format fmt, const void* aq, const void* as, const void* bq,
                                   const void* bs, const int32_t* group_offsets, int32_t groups,
                                   int64_t total_m, int64_t n, int64_t k, void* c, int32_t c_dtype,
                                   void* stream) {
    t_detail[0] = 0;
    fpq_status st;
    if (groups < 1 || groups > 1024 || total_m < 1 || n < 16 || n % 16 || k < 128 || k % 128 ||
        (c_dtype != FPQ_OUT_BF16 && c_dtype != FPQ_OUT_F32) || total_m > (1 << 30) || n > (1 << 30) ||
        k > (1 << 30)) {
        set_detail("need 1 <= groups <= 1024, total_m >= 1, n a positive multiple of 16, k a positive multiple of 128");
        return FPQ_ERR_INVALID_ARG;
    }
    if ((st = check_ptrs({aq, as, bq, bs, c, group_offsets})) != FPQ_OK) return st;
    if (fmt != FPQ_MXFP8) { set_detail("grouped GEMM supports FPQ_MXFP8 only"); return FPQ_ERR_UNSUPPORTED; }
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    return from_cuda(fpq::launch_grouped_gemm_mxfp8(aq, as, bq, bs, group_offsets, groups, total_m, n, k, c,
                                                    c_dtype == FPQ_OUT_F32, d->err, d->sms, (cudaStream_t)stream),
                     "grouped gemm launch");
}

fpq_status fpq_get_device_error(void* stream, int32_t* code) {
    t_detail[0] = 0;
    if (!code) { set_detail("null code pointer"); return FPQ_ERR_INVALID_ARG; }
    fpq_status st;
    const DeviceState* d = device_state(&st);
    if (!d) return st;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return from_cuda(e, "stream synchronize");
    uint32_t v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
    if (e != cudaSuccess) return from_cuda(e, "read device error word");
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return from_cuda(e, "clear device error word");
    *code = (int32_t)v;
    return FPQ_OK;
}

}  // extern "C"
