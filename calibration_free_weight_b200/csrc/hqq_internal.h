// hqq_internal.h -- shared between the C-ABI front end (hqq_api.cu) and the
// kernels (hqq_kernels.cu).  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace hqq {

constexpr int kPiece = 8;            // elements per 16-byte piece of 16-bit data
constexpr int kMaxPartials = 4096;   // per-CTA partial slots in the workspace
constexpr int kMaxIters = 1000;      // upper bound on iters (argument check)
constexpr float kScaleCap = 2.0e4f;  // cap on s (and on the 8-bit zero quantiser's scale)

// Workspace layout (offsets 256-byte aligned):
//   header      256 B: status word, CTA ticket, 64-bit work counter
//   minmax      float2[kMaxPartials]   per-CTA min/max of the kept zeros
//   zbest       float[G]               kept zeros (8-bit zero path)
//   tensor mode: tparts double[4][kMaxPartials], etot double[kMaxIters],
//                s f32[G], z0 f32[G], sum w*s f64[G], chunk-start zeros f32[3][G]
struct WorkspaceLayout {
    size_t header, minmax, zbest, tparts, etot, t_s, t_z0, t_sws, t_zs, total;
};
WorkspaceLayout workspace_layout(int64_t G, int stop_mode, int zero_nbits, int iters);

struct Geometry {
    int g;  // group size
    int E;  // elements per lane
    int P;  // lanes per group (g / E, <= 32)
};
Geometry make_geometry(int g);

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
    int32_t* dbg_iter;
    float* dbg_err;
    float* dbg_zero;
};

struct DequantArgs {
    const uint8_t* packed;
    const uint16_t* scale;
    const void* zero;
    const float* zero_meta;
    int64_t rows, cols;
    int nbits, g, axis, zero_nbits, out_dtype;
    void* out;
};

// Launchers: return cudaSuccess or the launch error.
cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream);
cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream);

}  // namespace hqq
