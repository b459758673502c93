// hqq_internal.h -- shared between the C-ABI front end (hqq_api.cu) and the
// kernels (hqq_kernels.cu).  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace hqq {

constexpr int kPiece = 8;            // elements per 16-byte piece of 16-bit data
constexpr int kMaxPartials = 4096;   // per-CTA partial slots in the workspace (tensor mode)
constexpr int64_t kMinSlice = 4096;  // smallest group-mode slice (entries) a workspace may be cut into
constexpr int kGemmMaxBatch = 65536;  // batch bound of hqq_gemm (argument check)
constexpr int kMaxIters = 1000;      // upper bound on iters (argument check)
constexpr float kScaleCap = 2.0e4f;  // cap on s (and on the 8-bit zero quantiser's scale)
constexpr uint32_t kStatusTimeout = 6;  // HQQ_ERR_TIMEOUT, as the device writes it to the status word

// Workspace layout (offsets 256-byte aligned):
//   header      256 B: status word, CTA ticket, kept-zero range, pass counts
//   zbest       float[G]               kept zeros (8-bit zero path)
//   group / no stop, per slice of S entries (a warp-tile slot each; S = all
//   entries, at most 2^31, unless the workspace is smaller):
//                state float4[2][S], state_it int[S], survivor lists u32[2][S]
//   tensor mode: tparts double[12][kMaxPartials], etot double[kMaxIters],
//                s f32[G], z0 f32[G], sum w*s f64[G], zeros of every iteration of
//                two chunks f32[2][slots][G] (slots = 6 for g <= 16, 12 above)
struct WorkspaceLayout {
    size_t header, zbest, state, state_it, list0, list1, tparts, etot, t_s, t_z0, t_sws, t_zs, total;
    int64_t slice;  // group mode: entries per slice
};
// slice <= 0: one slice holding every entry.
WorkspaceLayout workspace_layout(int64_t rows, int64_t cols, int g, int axis, int stop_mode, int zero_nbits,
                                 int64_t slice);
// Group mode: the largest slice whose layout fits in `bytes` (0 if none of at
// least kMinSlice entries does); every entry if the full layout fits.
int64_t fit_slice(int64_t rows, int64_t cols, int g, int axis, int stop_mode, int zero_nbits, size_t bytes);

struct Geometry {
    int g;     // group size
    int E;     // elements per lane: min(g, 32)
    int P;     // lanes per group: g / E
    int logP;
};
Geometry make_geometry(int g);
int64_t group_entries(int64_t rows, int64_t cols, int g, int axis);  // warp-tile slots over all groups

struct SolveArgs {
    const void* W;
    int64_t rows, cols, G;
    int dtype, nbits, g, axis, iters, stop_mode, zero_nbits;
    float p, beta, kappa;
    uint8_t* packed;
    uint16_t* scale;   // fp16 bits
    void* zero;        // fp16 bits or uint8
    float* zero_meta;  // fp32[2] or null
    uint8_t* ws;       // workspace base
    int64_t slice;     // group mode: entries per slice (from the workspace layout)
    int32_t* dbg_iter;
    float* dbg_err;
    float* dbg_zero;
    bool half = false;  // the half-precision solver variant (fp16 input, axis 1, group or no stop)
};

struct DequantArgs {
    const uint8_t* packed;
    const uint16_t* scale;      // fp16 scales (scale_meta == null), else
    const uint8_t* scale_q;     // 8-bit codes and
    const float* scale_meta;    // (1/sc, zc) per run of scale_group
    int scale_group;
    const void* zero;
    const float* zero_meta;
    int64_t rows, cols;
    int nbits, g, axis, zero_nbits, out_dtype;
    void* out;
};

struct GemvArgs {
    const uint8_t* packed;
    const uint16_t* scale;
    const void* zero;
    const float* zero_meta;
    int64_t rows, cols;
    int nbits, g, zero_nbits;
    const void* x;  // [batch][cols] fp16/bf16
    int x_dtype, batch;
    float* y;       // [batch][rows]
    void* workspace = nullptr;  // split tensor-core products: tickets and partial tiles
    size_t workspace_bytes = 0;
};
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t stream);
// The tensor-core product (batch >= 1, cols a multiple of 64, x 16-byte aligned).
cudaError_t launch_gemm(const GemvArgs& a, cudaStream_t stream);
// Batch tiles of launch_gemm: ntiles tiles of ntile (a multiple of 16, <= 256) rows.
void gemm_tiles(int batch, int* ntile, int* ntiles);
// K splits launch_gemm uses when its workspace allows, and the bytes that needs (0: unsplit).
int gemm_splits(int64_t rows, int64_t cols, int batch);
size_t gemm_workspace_bytes(int64_t rows, int64_t cols, int batch);
int sm_count();
// One bounded wait, as the product's, on a barrier nothing arrives on (diagnostic).
cudaError_t launch_gemm_wait_selftest(unsigned long long limit_ns, cudaStream_t stream);
// Synchronises the stream; 0, 6 (a wait of a product gave up; cleared) or 5 (CUDA error).
int gemm_take_status(cudaStream_t stream);

// Tensor stop on one cooperative launch with W kept on chip, or the chunked
// launches: mode 0 never the former, 1 (default) for g >= 32 where it fits, 2
// wherever it fits.
void set_tensor_resident(int mode);
int tensor_resident();
// Whether a tensor-stop call of this shape takes the resident kernel on the current device.
bool tensor_uses_resident(int64_t rows, int64_t cols, int dtype, int g, int axis, int iters);
// The resident kernel's bounded wait on a decision nothing publishes (diagnostic):
// zeroes the workspace header, then records HQQ_ERR_TIMEOUT in its status word.
cudaError_t launch_tensor_wait_selftest(uint8_t* ws, unsigned long long limit_ns, cudaStream_t stream);

// Launchers: return cudaSuccess or the launch error.
cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream);
cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream);
cudaError_t launch_scale8(const uint16_t* scale, int64_t G, int S, uint8_t* codes, float* meta, cudaStream_t stream);

// The host-side argument checks of hqq_quantize (dtype, bit width, shape,
// solver parameters, modes): HQQ_OK or the status hqq_quantize returns.
int check_args(int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis, float p, float beta,
               float kappa, int iters, int stop_mode, int zero_nbits);

// hqq_quantize with an option to cut group-mode work into slices that fit a
// smaller workspace (used by hqq_quantize_noalloc).
int quantize_entry(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis, float p,
                   float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* W_q_packed, void* scale,
                   void* zero, void* zero_meta, void* workspace, size_t workspace_bytes, bool allow_slices,
                   int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32, void* stream,
                   bool half = false);

}  // namespace hqq
