// hqq_noalloc.cu -- hqq_quantize_noalloc: the group-stop quantiser for callers
// that cannot allocate device memory.
//
// Who needs it: code that is handed its inputs and outputs but has no way, or
// no permission, to call cudaMalloc -- for example a plugin running inside a
// host runtime that owns every device allocation, or a latency-critical loop
// where an allocation (and the implicit device synchronisation cudaMalloc and
// cudaFree can cause) is not acceptable.  hqq_quantize needs a caller-provided
// workspace; this entry point instead uses one scratch buffer that the library
// itself holds in device memory.
//
// The scratch is a file-scope __device__ array of kScratchBytes.  Every GPU
// that loads this library keeps it resident until the process exits.  In host
// code the array's name only stands for the symbol; its device address is
// obtained once per device with cudaGetSymbolAddress (done by the first call
// on that device, with that device current) and that address is what the
// kernels receive.  All calls on a device share the buffer and it keeps the
// last call's contents; the solver clears what must start at zero (the status
// header) on every call.  Two calls whose work overlaps on the GPU (different
// streams, or different host threads without ordering) race on the buffer.

#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hqq.h"
#include "hqq_internal.h"

namespace {

constexpr size_t kScratchBytes = HQQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (set up on first use).
cudaError_t scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        err = cudaGetSymbolAddress(&ptr, g_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int hqq_quantize_noalloc(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size,
                                    int axis, float p, float beta, float kappa, int iters, int stop_mode,
                                    int zero_nbits, void* W_q_packed, void* scale, void* zero, void* zero_meta,
                                    int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32,
                                    void* stream) {
    if (stop_mode == HQQ_STOP_TENSOR) return HQQ_ERR_INVALID_ARG;
    const size_t need = hqq_workspace_bytes(rows, cols, group_size, axis, stop_mode, zero_nbits);
    void* ws = nullptr;
    if (need > 0) {  // need == 0: invalid arguments, reported by quantize_entry below
        if (hqq::fit_slice(rows, cols, group_size, axis, stop_mode, zero_nbits, kScratchBytes) <= 0)
            return HQQ_ERR_WORKSPACE;
        if (scratch_for_current_device(&ws) != cudaSuccess) {
            cudaGetLastError();
            return HQQ_ERR_CUDA;
        }
    }
    // a problem whose full workspace exceeds the scratch runs in slices of groups
    return hqq::quantize_entry(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                               zero_nbits, W_q_packed, scale, zero, zero_meta, ws, ws ? kScratchBytes : 0, true,
                               debug_best_iter, debug_best_err, debug_zero_f32, stream);
}
