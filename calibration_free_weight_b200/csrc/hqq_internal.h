// hqq_internal.h -- shared between the C-ABI front end (hqq_api.cu) and the
// kernels (hqq_kernels.cu).  Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace hqq {

constexpr int kThreads = 256;         // threads per CTA of every solver kernel
constexpr int kPiece = 8;             // elements per 16-byte piece
constexpr int kMaxTileGroups = 512;   // groups per tile at most
constexpr int kMaxTileElems = 16384;  // elements per tile at most (32 KB of fp16/bf16)
constexpr int kMaxPartials = 4096;    // per-CTA partial slots in the workspace
constexpr float kScaleCap = 2.0e4f;   // cap on s (and on the 8-bit zero quantiser's scale)

// Device status word values (mirrors hqq_status).
constexpr uint32_t kStatusOk = 0;
constexpr uint32_t kStatusTimeout = 6;

// Workspace layout (all offsets 256-byte aligned):
//   [0, 256)                 header: status, barrier count, barrier generation
//   partial min/max          float2[kMaxPartials]
//   tensor error partials    double[2][kMaxPartials]
//   zbest                    float[G]            (zero_nbits == 8)
//   tensor state             s f32[G], 1/s f32[G], z0 f32[G], sws f64[G], Z f32[3][G], E f32[3][G]
struct WorkspaceLayout {
    size_t header, minmax, tparts, zbest, t_s, t_is, t_z0, t_sws, t_z, t_e, total;
};
WorkspaceLayout workspace_layout(int64_t G, int stop_mode, int zero_nbits);

struct Geometry {
    int g;            // group size
    int P;            // lanes per group (<= 32, power of two)
    int NP;           // 16-byte pieces per lane
    int tile_groups;  // groups per tile
    int tile_elems;   // tile_groups * g
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
    bool vec_ok;       // 16-byte vector loads allowed for the tile loader
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
cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream, int* coop_unsupported);
cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream);

// Test hook for the tensor-mode grid barrier.
void set_barrier_debug(int skip_block, uint64_t timeout_ns);

}  // namespace hqq
