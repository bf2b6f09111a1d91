// noalloc.cu -- NVFP4 quantization for callers that cannot allocate device
// memory.
//
// The regular entry point (fpq_quantize_block with FPQ_NVFP4) needs a small
// caller-provided workspace for the per-tensor amax.  Some callers hold only
// their input and output buffers and have no way to obtain more device
// memory: for example a C plugin loaded into a serving runtime that owns the
// whole device memory pool, where a cudaMalloc would fall outside the
// runtime's budget (or stall the device in the middle of a request).  For
// them this file keeps the amax scratch in a file-scope device array that
// every GPU loading the library holds until the process exits.
#include <mutex>

#include "../../include/fpq.h"
#include "internal.h"

namespace {

// The NVFP4 quantize workspace for up to FPQ_NOALLOC_NVFP4_MAX_BATCH
// matrices: a work-item counter plus one amax word and one progress counter
// per matrix (4 + 2 * 4096 words, 32 KiB + 16 bytes).
constexpr int kScratchWords = 4 + 2 * FPQ_NOALLOC_NVFP4_MAX_BATCH;
__device__ __align__(256) uint32_t g_noalloc_amax[kScratchWords];

constexpr int kMaxDevices = 64;
void* g_scratch[kMaxDevices] = {};
std::mutex g_mu;

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached by device ordinal.
// The cache assumes the device's primary context for the life of the
// process (no cudaDeviceReset, no other driver context on the ordinal); the
// device error word of the other entry points is cached the same way.
fpq_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        fpq::set_error_detail("no CUDA device");
        return FPQ_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_amax);
        if (e != cudaSuccess || p == nullptr) {
            fpq::set_error_detail("cudaGetSymbolAddress of the no-alloc scratch array failed");
            return FPQ_ERR_CUDA;
        }
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return FPQ_OK;
}

}  // namespace

extern "C" FPQ_API fpq_status fpq_quantize_nvfp4_noalloc(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                                         void* q, void* scales, float* tensor_scale, void* stream) {
    if (batch < 1 || batch > FPQ_NOALLOC_NVFP4_MAX_BATCH) {
        fpq::set_error_detail("fpq_quantize_nvfp4_noalloc: batch must be in [1, FPQ_NOALLOC_NVFP4_MAX_BATCH]");
        return FPQ_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    fpq_status st = scratch_on_current_device(&scratch);
    if (st != FPQ_OK) return st;
    // The quantizer zeroes the workspace words it uses before it starts.
    return fpq_quantize_block(FPQ_NVFP4, x, batch, rows, cols, q, scales, tensor_scale, scratch,
                              sizeof(uint32_t) * (size_t)kScratchWords, stream);
}
