// hqq_api.cu -- the extern "C" entry points declared in include/hqq.h.
//
// Every argument is checked on the host before anything is launched; a bad
// argument returns an error code and touches no output.  Device pointers are
// checked with cudaPointerGetAttributes so that a host pointer never reaches a
// kernel.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/hqq.h"
#include "hqq_internal.h"

namespace {

bool valid_group_size(int g) { return g >= 8 && g <= 1024 && (g & (g - 1)) == 0; }

bool valid_nbits(int b) { return b == 1 || b == 2 || b == 3 || b == 4 || b == 8; }

// Shape checks shared by every entry point: HQQ_OK, HQQ_ERR_SHAPE or HQQ_ERR_INVALID_ARG.
int check_shape(int64_t rows, int64_t cols, int g, int axis) {
    if (rows < 0 || cols < 0) return HQQ_ERR_SHAPE;
    if (axis != 0 && axis != 1) return HQQ_ERR_INVALID_ARG;
    if (!valid_group_size(g)) return HQQ_ERR_SHAPE;
    if (axis == 1 && cols % g != 0) return HQQ_ERR_SHAPE;
    if (axis == 0 && rows % g != 0) return HQQ_ERR_SHAPE;
    if (cols > 0 && rows > (INT64_MAX / 16) / cols) return HQQ_ERR_SHAPE;
    return HQQ_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Device (or managed) memory of the current device; anything else is rejected.
bool is_device_ptr(const void* p) {
    if (p == nullptr) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    if (attr.type != cudaMemoryTypeDevice) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    return attr.device == dev;
}

}  // namespace

namespace hqq {

int check_args(int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis, float p, float beta,
               float kappa, int iters, int stop_mode, int zero_nbits) {
    if (dtype != HQQ_F16 && dtype != HQQ_BF16) return HQQ_ERR_DTYPE;
    if (!valid_nbits(nbits)) return HQQ_ERR_INVALID_ARG;
    const int sh = check_shape(rows, cols, group_size, axis);
    if (sh != HQQ_OK) return sh;
    if (!(p > 0.0f && p < 2.0f) || !(beta > 0.0f) || !std::isfinite(beta) || !(kappa >= 1.0f) ||
        !std::isfinite(kappa))
        return HQQ_ERR_INVALID_ARG;
    if (iters < 0 || iters > hqq::kMaxIters) return HQQ_ERR_INVALID_ARG;
    if (stop_mode < 0 || stop_mode > 2) return HQQ_ERR_INVALID_ARG;
    if (zero_nbits != 8 && zero_nbits != 16) return HQQ_ERR_INVALID_ARG;
    return HQQ_OK;
}

int quantize_entry(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis, float p,
                   float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* W_q_packed, void* scale,
                   void* zero, void* zero_meta, void* workspace, size_t workspace_bytes, bool allow_slices,
                   int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32, void* stream,
                   bool half) {
    const int ck = check_args(rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode, zero_nbits);
    if (ck != HQQ_OK) return ck;
    if (half) {
        if (dtype != HQQ_F16) return HQQ_ERR_DTYPE;
        if (axis != 1 || stop_mode == HQQ_STOP_TENSOR) return HQQ_ERR_INVALID_ARG;
    }
    const int64_t G = rows * cols / group_size;
    const int64_t slice =
        hqq::fit_slice(rows, cols, group_size, axis, stop_mode, zero_nbits, workspace == nullptr ? 0 : workspace_bytes);
    const size_t need = hqq::workspace_layout(rows, cols, group_size, axis, stop_mode, zero_nbits, 0).total;
    if (workspace == nullptr || (!allow_slices && workspace_bytes < need) || slice <= 0) return HQQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return HQQ_ERR_ALIGN;
    if (!is_device_ptr(workspace)) return HQQ_ERR_INVALID_ARG;
    if (zero_nbits == 8) {
        if (!is_device_ptr(zero_meta)) return HQQ_ERR_INVALID_ARG;
        if (!aligned(zero_meta, 4)) return HQQ_ERR_ALIGN;
    }
    if (G > 0) {
        if (!is_device_ptr(W) || !is_device_ptr(W_q_packed) || !is_device_ptr(scale) || !is_device_ptr(zero))
            return HQQ_ERR_INVALID_ARG;
        if (!aligned(W, 16) || !aligned(W_q_packed, 16) || !aligned(scale, 2)) return HQQ_ERR_ALIGN;
        if (zero_nbits == 16 && !aligned(zero, 2)) return HQQ_ERR_ALIGN;
        if (debug_best_iter && (!is_device_ptr(debug_best_iter) || !aligned(debug_best_iter, 4)))
            return HQQ_ERR_INVALID_ARG;
        if (debug_best_err && (!is_device_ptr(debug_best_err) || !aligned(debug_best_err, 4)))
            return HQQ_ERR_INVALID_ARG;
        if (debug_zero_f32 && (!is_device_ptr(debug_zero_f32) || !aligned(debug_zero_f32, 4)))
            return HQQ_ERR_INVALID_ARG;
    }

    hqq::SolveArgs a{};
    a.W = W;
    a.rows = rows;
    a.cols = cols;
    a.G = G;
    a.dtype = dtype;
    a.nbits = nbits;
    a.g = group_size;
    a.axis = axis;
    a.iters = iters;
    a.stop_mode = stop_mode;
    a.zero_nbits = zero_nbits;
    a.p = p;
    a.beta = beta;
    a.kappa = kappa;
    a.packed = static_cast<uint8_t*>(W_q_packed);
    a.scale = static_cast<uint16_t*>(scale);
    a.zero = zero;
    a.zero_meta = static_cast<float*>(zero_meta);
    a.ws = static_cast<uint8_t*>(workspace);
    a.slice = slice;
    a.dbg_iter = debug_best_iter;
    a.dbg_err = debug_best_err;
    a.dbg_zero = debug_zero_f32;
    a.half = half;
    const cudaError_t err = hqq::launch_solve(a, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

}  // namespace hqq

extern "C" {

size_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits, int group_size, int axis) {
    if (!valid_nbits(nbits) || check_shape(rows, cols, group_size, axis) != HQQ_OK) return 0;
    return static_cast<size_t>(rows * cols * nbits / 8);
}

int64_t hqq_num_groups(int64_t rows, int64_t cols, int group_size, int axis) {
    if (check_shape(rows, cols, group_size, axis) != HQQ_OK) return -1;
    return rows * cols / group_size;
}

size_t hqq_workspace_bytes(int64_t rows, int64_t cols, int group_size, int axis, int stop_mode, int zero_nbits) {
    if (check_shape(rows, cols, group_size, axis) != HQQ_OK) return 0;
    if (stop_mode < 0 || stop_mode > 2 || (zero_nbits != 8 && zero_nbits != 16)) return 0;
    return hqq::workspace_layout(rows, cols, group_size, axis, stop_mode, zero_nbits, 0).total;
}

int hqq_quantize(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis, float p,
                 float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* W_q_packed, void* scale,
                 void* zero, void* zero_meta, void* workspace, size_t workspace_bytes, int32_t* debug_best_iter,
                 float* debug_best_err, float* debug_zero_f32, void* stream) {
    return hqq::quantize_entry(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                               zero_nbits, W_q_packed, scale, zero, zero_meta, workspace, workspace_bytes, false,
                               debug_best_iter, debug_best_err, debug_zero_f32, stream);
}

int hqq_quantize_half(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis,
                      float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* W_q_packed,
                      void* scale, void* zero, void* zero_meta, void* workspace, size_t workspace_bytes,
                      int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32, void* stream) {
    return hqq::quantize_entry(W, rows, cols, dtype, nbits, group_size, axis, p, beta, kappa, iters, stop_mode,
                               zero_nbits, W_q_packed, scale, zero, zero_meta, workspace, workspace_bytes, false,
                               debug_best_iter, debug_best_err, debug_zero_f32, stream, true);
}

}  // extern "C"

namespace {

// hqq_dequantize and hqq_dequantize_s8: scale8 == true reads 8-bit scale codes
// and their per-run meta instead of fp16 scales.
int dequantize_entry(const void* W_q_packed, const void* scale, const void* scale_meta, int scale_group, bool scale8,
                     const void* zero, const void* zero_meta, int64_t rows, int64_t cols, int nbits, int group_size,
                     int axis, int zero_nbits, int out_dtype, void* W_out, void* stream) {
    if (out_dtype != HQQ_F16 && out_dtype != HQQ_BF16) return HQQ_ERR_DTYPE;
    if (!valid_nbits(nbits)) return HQQ_ERR_INVALID_ARG;
    const int sh = check_shape(rows, cols, group_size, axis);
    if (sh != HQQ_OK) return sh;
    if (zero_nbits != 8 && zero_nbits != 16) return HQQ_ERR_INVALID_ARG;
    if (scale8 && scale_group < 1) return HQQ_ERR_INVALID_ARG;
    if (rows * cols == 0) return HQQ_OK;
    if (!is_device_ptr(W_q_packed) || !is_device_ptr(scale) || !is_device_ptr(zero) || !is_device_ptr(W_out))
        return HQQ_ERR_INVALID_ARG;
    if (zero_nbits == 8 && !is_device_ptr(zero_meta)) return HQQ_ERR_INVALID_ARG;
    if (scale8 && !is_device_ptr(scale_meta)) return HQQ_ERR_INVALID_ARG;
    if (!aligned(W_q_packed, 16) || !aligned(W_out, 16)) return HQQ_ERR_ALIGN;
    if (!scale8 && !aligned(scale, 2)) return HQQ_ERR_ALIGN;
    if (scale8 && !aligned(scale_meta, 4)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 16 && !aligned(zero, 2)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 8 && !aligned(zero_meta, 4)) return HQQ_ERR_ALIGN;
    if (axis == 1 && cols % 8 != 0) return HQQ_ERR_SHAPE;  // implied by g | cols, kept explicit
    hqq::DequantArgs a{};
    a.packed = static_cast<const uint8_t*>(W_q_packed);
    a.scale = scale8 ? nullptr : static_cast<const uint16_t*>(scale);
    a.scale_q = scale8 ? static_cast<const uint8_t*>(scale) : nullptr;
    a.scale_meta = scale8 ? static_cast<const float*>(scale_meta) : nullptr;
    a.scale_group = scale8 ? scale_group : 1;
    a.zero = zero;
    a.zero_meta = static_cast<const float*>(zero_meta);
    a.rows = rows;
    a.cols = cols;
    a.nbits = nbits;
    a.g = group_size;
    a.axis = axis;
    a.zero_nbits = zero_nbits;
    a.out_dtype = out_dtype;
    a.out = W_out;
    if (hqq::launch_dequant(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

}  // namespace

extern "C" {

int hqq_dequantize(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta, int64_t rows,
                   int64_t cols, int nbits, int group_size, int axis, int zero_nbits, int out_dtype, void* W_out,
                   void* stream) {
    return dequantize_entry(W_q_packed, scale, nullptr, 0, false, zero, zero_meta, rows, cols, nbits, group_size, axis,
                            zero_nbits, out_dtype, W_out, stream);
}

int hqq_dequantize_s8(const void* W_q_packed, const void* scale_q, const void* scale_meta, int scale_group,
                      const void* zero, const void* zero_meta, int64_t rows, int64_t cols, int nbits, int group_size,
                      int axis, int zero_nbits, int out_dtype, void* W_out, void* stream) {
    return dequantize_entry(W_q_packed, scale_q, scale_meta, scale_group, true, zero, zero_meta, rows, cols, nbits,
                            group_size, axis, zero_nbits, out_dtype, W_out, stream);
}

int hqq_gemv(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta, int64_t rows,
             int64_t cols, int nbits, int group_size, int zero_nbits, const void* x, int x_dtype, int batch, float* y,
             void* stream) {
    if (x_dtype != HQQ_F16 && x_dtype != HQQ_BF16) return HQQ_ERR_DTYPE;
    if (!valid_nbits(nbits) || batch < 1 || batch > 8) return HQQ_ERR_INVALID_ARG;
    const int sh = check_shape(rows, cols, group_size, 1);
    if (sh != HQQ_OK) return sh;
    if (zero_nbits != 8 && zero_nbits != 16) return HQQ_ERR_INVALID_ARG;
    if (rows * cols == 0) return HQQ_OK;
    if (!is_device_ptr(W_q_packed) || !is_device_ptr(scale) || !is_device_ptr(zero) || !is_device_ptr(x) ||
        !is_device_ptr(y))
        return HQQ_ERR_INVALID_ARG;
    if (zero_nbits == 8 && !is_device_ptr(zero_meta)) return HQQ_ERR_INVALID_ARG;
    if (!aligned(W_q_packed, 16) || !aligned(scale, 2) || !aligned(x, 16) || !aligned(y, 4)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 16 && !aligned(zero, 2)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 8 && !aligned(zero_meta, 4)) return HQQ_ERR_ALIGN;
    hqq::GemvArgs a{};
    a.packed = static_cast<const uint8_t*>(W_q_packed);
    a.scale = static_cast<const uint16_t*>(scale);
    a.zero = zero;
    a.zero_meta = static_cast<const float*>(zero_meta);
    a.rows = rows;
    a.cols = cols;
    a.nbits = nbits;
    a.g = group_size;
    a.zero_nbits = zero_nbits;
    a.x = x;
    a.x_dtype = x_dtype;
    a.batch = batch;
    a.y = y;
    if (hqq::launch_gemv(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

size_t hqq_gemm_workspace_bytes(int64_t rows, int64_t cols, int batch) {
    if (rows < 1 || cols < 64 || cols % 64 != 0 || batch < 1 || batch > hqq::kGemmMaxBatch) return 0;
    if (cols > 0 && rows > (INT64_MAX / 16) / cols) return 0;
    return hqq::gemm_workspace_bytes(rows, cols, batch);
}

int hqq_gemm(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta, int64_t rows,
             int64_t cols, int nbits, int group_size, int zero_nbits, const void* x, int x_dtype, int batch, float* y,
             void* workspace, size_t workspace_bytes, void* stream) {
    if (x_dtype != HQQ_F16 && x_dtype != HQQ_BF16) return HQQ_ERR_DTYPE;
    if (!valid_nbits(nbits) || batch < 1 || batch > hqq::kGemmMaxBatch) return HQQ_ERR_INVALID_ARG;
    const int sh = check_shape(rows, cols, group_size, 1);
    if (sh != HQQ_OK) return sh;
    if (cols % 64 != 0) return HQQ_ERR_SHAPE;
    if (zero_nbits != 8 && zero_nbits != 16) return HQQ_ERR_INVALID_ARG;
    if (rows * cols == 0) return HQQ_OK;
    if (!is_device_ptr(W_q_packed) || !is_device_ptr(scale) || !is_device_ptr(zero) || !is_device_ptr(x) ||
        !is_device_ptr(y))
        return HQQ_ERR_INVALID_ARG;
    if (zero_nbits == 8 && !is_device_ptr(zero_meta)) return HQQ_ERR_INVALID_ARG;
    if (!aligned(W_q_packed, 16) || !aligned(scale, 2) || !aligned(x, 16) || !aligned(y, 4)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 16 && !aligned(zero, 2)) return HQQ_ERR_ALIGN;
    if (zero_nbits == 8 && !aligned(zero_meta, 4)) return HQQ_ERR_ALIGN;
    if (workspace != nullptr && (!is_device_ptr(workspace) || !aligned(workspace, 256))) return HQQ_ERR_INVALID_ARG;
    hqq::GemvArgs a{};
    a.packed = static_cast<const uint8_t*>(W_q_packed);
    a.scale = static_cast<const uint16_t*>(scale);
    a.zero = zero;
    a.zero_meta = static_cast<const float*>(zero_meta);
    a.rows = rows;
    a.cols = cols;
    a.nbits = nbits;
    a.g = group_size;
    a.zero_nbits = zero_nbits;
    a.x = x;
    a.x_dtype = x_dtype;
    a.batch = batch;
    a.y = y;
    a.workspace = workspace;
    a.workspace_bytes = workspace ? workspace_bytes : 0;
    if (hqq::launch_gemm(a, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

int hqq_gemm_get_status(void* stream) { return hqq::gemm_take_status(static_cast<cudaStream_t>(stream)); }

int hqq_gemm_wait_selftest(int64_t limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return HQQ_ERR_INVALID_ARG;
    if (hqq::launch_gemm_wait_selftest(static_cast<unsigned long long>(limit_us) * 1000ull,
                                       static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

int hqq_set_tensor_resident(int mode) {
    if (mode < 0 || mode > 2) return -1;
    const int prev = hqq::tensor_resident();
    hqq::set_tensor_resident(mode);
    return prev;
}

int hqq_tensor_resident(int64_t rows, int64_t cols, int dtype, int group_size, int axis, int iters) {
    if (hqq::check_args(rows, cols, dtype, 4, group_size, axis, 0.7f, 1.0f, 1.0f, iters, HQQ_STOP_TENSOR, 16) !=
        HQQ_OK)
        return 0;
    return hqq::tensor_uses_resident(rows, cols, dtype, group_size, axis, iters) ? 1 : 0;
}

int hqq_quantize_wait_selftest(void* workspace, size_t workspace_bytes, int64_t limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000 || workspace_bytes < 256) return HQQ_ERR_INVALID_ARG;
    if (!is_device_ptr(workspace) || !aligned(workspace, 256)) return HQQ_ERR_INVALID_ARG;
    if (hqq::launch_tensor_wait_selftest(static_cast<uint8_t*>(workspace), static_cast<unsigned long long>(limit_us) * 1000ull,
                                         static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

int hqq_quantize_scale8(const void* scale, int64_t num_groups, int scale_group, void* scale_q, void* scale_meta,
                        void* stream) {
    if (num_groups < 0 || scale_group < 1) return HQQ_ERR_INVALID_ARG;
    if (num_groups == 0) return HQQ_OK;
    if (!is_device_ptr(scale) || !is_device_ptr(scale_q) || !is_device_ptr(scale_meta)) return HQQ_ERR_INVALID_ARG;
    if (!aligned(scale, 2) || !aligned(scale_meta, 4)) return HQQ_ERR_ALIGN;
    if (hqq::launch_scale8(static_cast<const uint16_t*>(scale), num_groups, scale_group,
                           static_cast<uint8_t*>(scale_q), static_cast<float*>(scale_meta),
                           static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return HQQ_OK;
}

int hqq_get_status(const void* workspace, void* stream) {
    if (!is_device_ptr(workspace)) return HQQ_ERR_INVALID_ARG;
    uint32_t st = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    return static_cast<int>(st);
}

const char* hqq_status_string(int status) {
    switch (status) {
        case HQQ_OK: return "ok";
        case HQQ_ERR_INVALID_ARG: return "invalid argument";
        case HQQ_ERR_SHAPE: return "invalid shape or group size";
        case HQQ_ERR_DTYPE: return "unsupported dtype";
        case HQQ_ERR_ALIGN: return "misaligned buffer";
        case HQQ_ERR_CUDA: return "CUDA runtime error";
        case HQQ_ERR_TIMEOUT: return "a bounded device wait gave up";
        case HQQ_ERR_COOP_UNSUPPORTED: return "cooperative launch unsupported (reserved; not returned)";
        case HQQ_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

}  // extern "C"
