// hqq_kernels.cu -- sm_100a kernels of the HQQ zero-point solver and their launchers.
//
// Method: techreport.ngo, "Weight-only quantization without the calibration
// tax" (Half-Quadratic Quantization of Large Machine Learning Models), sections
// "Outlier-aware optimization without gradients" (lp loss, half-quadratic
// split, generalised soft-thresholding, group-mean zero update, fixed scale)
// and "Benchmark results"/"Llama-2" (p, beta, kappa, 20 iterations, early
// stopping, 8-bit zero).  The per-step formulas are restated in include/hqq.h;
// the per-element evaluation is in hqq_device.cuh.
//
// The path has no dense contraction: no tensor cores.  Each element and
// evaluation costs 7 fp32 operations, six of them issued as packed pairs
// (add/sub/mul.rn.f32x2), and two MUFU ops (|r|^p through lg2/ex2), so the
// MUFU pipe, not HBM, bounds the solver.
//
// The solver kernels hold a warp tile of 32/P groups in registers, E = g/P
// elements per lane (E = min(g, 32)).  Only solve_tensor_resident_kernel has
// CTAs that wait for others (bounded waits, in a cooperative launch).
//
// solve_group_onepass_kernel (group / no stop, axis 1): reads W once; groups
//   that run past their first two evaluations wait in a per-warp pool in
//   shared memory (see the kernel's own comment).
// solve_group_kernel (group / no stop, axis 0): a sequence of passes.  Pass
//   0 initialises every group (min/max -> s, z0; fp32 w*s; sum of w*s) and runs
//   up to m_0 evaluations; a group that stops is packed and stored at once, a
//   group still running leaves its state (z, best error, kept zero, s, z0,
//   max w*s, sum of w*s) in the workspace and its index in a survivor list
//   (warp-aggregated atomic append).  Pass p runs the survivors of pass p-1
//   for m_p more evaluations.  Every group in a pass has done the same number
//   of iterations, so the iteration index and beta are warp-uniform, and the
//   lanes of a warp stay busy: a tile only runs as long as its slowest group
//   within one pass.
// solve_tensor_resident_kernel (tensor stop, axis 1, W within half the L2 and
//   the groups' state within shared memory): one cooperative launch runs every
//   iteration; W stays in L2, the state between rounds in shared memory, and
//   the tensor error of each iteration is reduced and the stop decided on the
//   device (see the kernel's own comment).
// solve_tensor_kernel (tensor stop, otherwise): runs iterations [k0, k1) of every group,
//   stores the zero-point of each of them, accumulates the per-iteration tensor
//   error per CTA, and the last CTA to finish (atomic ticket) sums the partials
//   in a fixed order, applies the stop rule to the errors so far and leaves
//   its outcome (first rise, kept iterate) in two workspace header words.  The
//   next launch reads those words and either runs the next chunk or returns.
//   The outputs: without debug outputs (axis 1) the last chunk writes those of
//   its last iterate (g >= 32), and tensor_output_kernel rewrites them from the
//   kept iterate's stored zero-point only when a tensor error rose; otherwise
//   the chunk kernel's own output launch writes them.

#include <atomic>
#include <type_traits>

#include "hqq_device.cuh"

namespace hqq {

namespace {

using namespace dev;

constexpr int kRegThreads = 256;
constexpr int kRegWarps = kRegThreads / 32;
constexpr int kChunkMax = 12;  // most iterations of one tensor-mode launch

// Iterations per tensor-mode launch: 8 for tiles of 32 elements per lane (the
// per-tile reload and set-up amortised over more iterations), 4 for smaller
// tiles (their iteration loop is unrolled and their partials held in registers).
__host__ __device__ constexpr int chunk_len(int E) { return E <= 16 ? 4 : 8; }
// Longest chunk: with C >= 8 a short last chunk is merged into the one before.
__host__ __device__ constexpr int chunk_max(int C) { return C >= 8 ? C + C / 2 - 1 : C; }
// Whether the last chunk writes the outputs of its last iterate when the
// outputs are streamed (32-element tiles; the smaller tiles have no spare
// registers for it).
__host__ __device__ constexpr bool last_chunk_outputs(int E) { return E > 16; }

// Header words of the workspace (uint32 index); word 0 is the status word.
constexpr int kWordTicket = 1;
constexpr int kWordZmin = 2;   // ~key(min kept zero), by atomicMax
constexpr int kWordZmax = 3;   // key(max kept zero), by atomicMax
constexpr int kWordSpecZmin = 4;  // the same two keys for the zeros of the last tensor-mode iterate
constexpr int kWordSpecZmax = 5;
constexpr int kWordStopAt = 6;  // tensor stop rule over the iterations run so far: first rise + 1 (0: none)
constexpr int kWordBestIt = 7;  // and the kept iterate + 1 (0: none), written by each chunk's last CTA
constexpr int kWordPass = 8;   // survivor count of group pass p at kWordPass + p
constexpr int kMaxPasses = 16;
constexpr int kWordChunk = 24;  // words 24-25: next chunk of the one-pass group solver (64-bit counter)
constexpr int kWordArrive = 26;  // words 26-29: warps of the resident tensor solver that posted the error
                                 // partial of an iteration, by iteration mod 4 (cumulative over the call)
constexpr int kWordDec = 32;     // words 32-63: its published stop decisions, 4 entries of 8 words

// ------------------------------------------------------- group outputs ----

__device__ __forceinline__ void store_group(const KParams& k, int64_t j, float s, float zb, int bi, float err_mean,
                                            float* zmin, float* zmax) {
    k.scale[j] = half_bits(__fdiv_rn(1.0f, s));
    if (k.zero_nbits == 16) {
        reinterpret_cast<uint16_t*>(k.zero)[j] = half_bits(zb);
    } else {
        k.zbest_ws[j] = zb;
        *zmin = fminf(*zmin, zb);
        *zmax = fmaxf(*zmax, zb);
    }
    if (k.dbg_iter) k.dbg_iter[j] = bi;
    if (k.dbg_err) k.dbg_err[j] = err_mean;
    if (k.dbg_zero) k.dbg_zero[j] = zb;
}

// Order-preserving key of a float (x < y <=> key(x) < key(y) as unsigned).
__device__ __forceinline__ uint32_t order_key(float x) {
    const uint32_t b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Block-wide min/max of the kept zeros, merged into the workspace header by
// two atomics per CTA (exact and order-independent, so launches and slices
// can all contribute).  The header starts at zero: the neutral element of both.
// The keys go to header words `word` (min) and `word` + 1 (max).
template <int NW>
__device__ __forceinline__ void merge_zero_range(const KParams& k, float zmin, float zmax, float2* sred,
                                                 int word = kWordZmin) {
    for (int o = 16; o > 0; o >>= 1) {
        zmin = fminf(zmin, __shfl_xor_sync(kFull, zmin, o));
        zmax = fmaxf(zmax, __shfl_xor_sync(kFull, zmax, o));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sred[warp] = make_float2(zmin, zmax);
    __syncthreads();
    if (threadIdx.x == 0) {
        float2 r = sred[0];
        for (int w = 1; w < NW; ++w) {
            r.x = fminf(r.x, sred[w].x);
            r.y = fmaxf(r.y, sred[w].y);
        }
        if (r.x <= r.y) {  // this CTA stored at least one zero
            atomicMax(k.counters + word, ~order_key(r.x));
            atomicMax(k.counters + word + 1, order_key(r.y));
        }
    }
}

// ====================================================== register tiles ==

// Chunk schedule of tensor mode with chunk length C: chunk 0 = iterations
// [0, 2), chunk c >= 1 = [C(c-1) + 2, Cc + 2), clipped to iters; with C >= 8
// a last chunk shorter than C/2 is merged into the one before it.
__host__ __device__ inline int num_chunks(int iters, int C) {
    if (iters <= 0) return 0;
    if (iters <= 2) return 1;
    int n = 1 + (iters - 2 + C - 1) / C;
    const int last = (iters - 2) - (n - 2) * C;
    if (C >= 8 && n > 2 && last < C / 2) --n;
    return n;
}
// First iteration of chunk c (iters for c >= num_chunks: the end of the last chunk).
__host__ __device__ inline int chunk_begin(int c, int iters, int C) {
    if (c == 0) return 0;
    if (c >= num_chunks(iters, C)) return iters;
    const int b = C * (c - 1) + 2;
    return b < iters ? b : iters;
}
__host__ __device__ inline int chunk_of(int k, int C, int iters) {
    if (k < 2) return 0;
    const int c = (k - 2) / C + 1, n = num_chunks(iters, C);
    return c < n ? c : n - 1;
}

struct WarpTile {
    bool valid;  // this lane's group exists
    int64_t j;   // group index
    int part;    // lane within the group
};

template <int AXIS>
__device__ __forceinline__ int64_t num_warp_tiles(const KParams& k) {
    const int gpw = 32 >> k.logP;  // groups per warp tile
    if (AXIS == 1) return (k.G + gpw - 1) / gpw;
    return (k.rows / k.g) * ((k.cols + gpw - 1) / gpw);
}

template <int AXIS>
__device__ __forceinline__ WarpTile warp_tile(const KParams& k, int64_t t) {
    const int lane = threadIdx.x & 31;
    const int gpw = 32 >> k.logP;
    WarpTile w;
    w.part = lane & (k.P - 1);
    const int tg = lane >> k.logP;
    if (AXIS == 1) {
        w.j = t * gpw + tg;
        w.valid = w.j < k.G;
    } else {
        const int64_t ncb = (k.cols + gpw - 1) / gpw;
        const int64_t rb = t / ncb, c = (t % ncb) * gpw + tg;
        w.valid = c < k.cols;
        w.j = rb * k.cols + c;
    }
    return w;
}

// This lane's E elements: element part*E + i of its group.
template <int DT, int AXIS, int E>
__device__ __forceinline__ void load_lane(const KParams& k, const WarpTile& w, float* x) {
    if (!w.valid) {
#pragma unroll
        for (int i = 0; i < E; ++i) x[i] = 0.0f;
        return;
    }
    if (AXIS == 1) {
        const uint4* src = reinterpret_cast<const uint4*>(k.W + w.j * k.g + w.part * E);
#pragma unroll
        for (int t = 0; t < E / kPiece; ++t) unpack8<DT>(__ldg(src + t), x + t * kPiece);
    } else {
        const int64_t rb = w.j / k.cols, c = w.j % k.cols;
        const uint16_t* src = k.W + (rb * k.g + w.part * E) * k.cols + c;
#pragma unroll
        for (int i = 0; i < E; ++i) x[i] = bits_to_float<DT>(__ldg(src + i * k.cols));
    }
}

// Eight codes, LSB first, NBITS each, as the NBITS bytes of one piece.
template <int NBITS>
__device__ __forceinline__ uint64_t pack8_t(const uint32_t* c) {
    if (NBITS == 8) {
        const uint32_t lo = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
        const uint32_t hi = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
        return static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32);
    }
    uint32_t v = 0;  // 8 * NBITS <= 32
#pragma unroll
    for (int i = 0; i < 8; ++i) v |= c[i] << (i * NBITS);
    return v;
}

template <int AXIS, int E, int NBITS>
__device__ __forceinline__ void store_lane_codes_t(const KParams& k, const WarpTile& w, const float* ws, float z) {
    constexpr float Lf = static_cast<float>((1 << NBITS) - 1);
#pragma unroll
    for (int t = 0; t < E / kPiece; ++t) {
        uint32_t code[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) round_clamp(__fadd_rn(ws[t * 8 + i], z), Lf, &code[i]);
        const uint64_t v = pack8_t<NBITS>(code);
        const int pc = (w.part * E) / kPiece + t;  // piece index within the group
        if (AXIS == 1) {
            uint8_t* dst = k.packed + (w.j * (k.g / kPiece) + pc) * NBITS;
            if (NBITS == 8) *reinterpret_cast<uint64_t*>(dst) = v;
            else if (NBITS == 4) *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(v);
            else if (NBITS == 2) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(v);
            else if (NBITS == 1) *dst = static_cast<uint8_t>(v);
            else {
                dst[0] = static_cast<uint8_t>(v);
                dst[1] = static_cast<uint8_t>(v >> 8);
                dst[2] = static_cast<uint8_t>(v >> 16);
            }
        } else {
            const int64_t rb = w.j / k.cols, c = w.j % k.cols;
            uint8_t* dst = k.packed + ((rb * k.g) / kPiece * NBITS + static_cast<int64_t>(pc) * NBITS) * k.cols + c;
#pragma unroll
            for (int b = 0; b < NBITS; ++b) dst[b * k.cols] = static_cast<uint8_t>(v >> (8 * b));
        }
    }
}

// Packed codes of this lane's E elements with zero-point z (bit width chosen
// by a warp-uniform switch, so the packing is compiled per width).
template <int AXIS, int E>
__device__ __forceinline__ void store_lane_codes(const KParams& k, const WarpTile& w, const float* ws, float z) {
    if (!w.valid) return;
    switch (k.nbits) {
        case 1: store_lane_codes_t<AXIS, E, 1>(k, w, ws, z); break;
        case 2: store_lane_codes_t<AXIS, E, 2>(k, w, ws, z); break;
        case 3: store_lane_codes_t<AXIS, E, 3>(k, w, ws, z); break;
        case 4: store_lane_codes_t<AXIS, E, 4>(k, w, ws, z); break;
        default: store_lane_codes_t<AXIS, E, 8>(k, w, ws, z); break;
    }
}

// min/max -> s, z0; fp32 w*s; fp64 sum of w*s (over the group's P lanes).
// Also returns this lane's range of w*s (for the clamp-free test).
template <int E, bool SUM = true>
__device__ __forceinline__ void init_lane(const KParams& k, const WarpTile& w, const float* x, float* ws, float* s_out,
                                          float* z0_out, double* sws_out, float* lmin_out, float* lmax_out) {
    float lmn = FLT_MAX, lmx = -FLT_MAX;
    if (w.valid) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            lmn = fminf(lmn, x[i]);
            lmx = fmaxf(lmx, x[i]);
        }
    }
    const float mn = seg_min(lmn, k.P);
    const float mx = seg_max(lmx, k.P);
    float s = kScaleCap;
    if (mx > mn) s = fminf(__fdiv_rn(k.Lf, __fsub_rn(mx, mn)), kScaleCap);
    // the sum of fp32 w*s in fp64, as the oracle accumulates it (up to the order)
    double accd = 0.0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        ws[i] = __fmul_rn(x[i], s);
        if (SUM) accd += static_cast<double>(ws[i]);
    }
    const double acc = (SUM && w.valid) ? accd : 0.0;
    *s_out = s;
    *z0_out = __fmul_rn(-mn, s);
    *sws_out = SUM ? seg_sum_d(acc, k.P) : 0.0;
    *lmin_out = w.valid ? __fmul_rn(lmn, s) : 0.0f;
    *lmax_out = w.valid ? __fmul_rn(lmx, s) : 0.0f;
}

// One evaluation of zero-point z: group sums of |r|^p and W_q, and (only when
// the proximal step may be active, warp-uniform branch) of fl((w - W_e)*s).
template <int E>
__device__ __forceinline__ void eval_lane(const KParams& k, bool active, const float* x, const float* ws, float s,
                                          float z, float z0, float beta, float thr, float* err_out, float* sq_out,
                                          bool* sp_out, double* swe_out) {
    float err = 0.0f, sq = 0.0f;
    const bool sp = active && shrink_possible(s, z, z0, thr, k.Lf);
    if (active) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const ElemEval ee = eval_elem(ws[i], z, k.Lf);
            err += pow_pos(fabsf(ee.r), k.p);
            sq += ee.q;
        }
    }
    *err_out = seg_sum(err, k.P);
    *sq_out = seg_sum(sq, k.P);
    double swe = 0.0;
    if (__any_sync(kFull, sp)) {
        if (sp) {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const ElemEval ee = eval_elem(ws[i], z, k.Lf);
                const float we = shrink_elem(ee.r, s, k.p, beta);
                swe += static_cast<double>(__fmul_rn(__fsub_rn(x[i], we), s));
            }
        }
        swe = seg_sum_d(swe, k.P);
    }
    *sp_out = sp;
    *swe_out = swe;
}

// beta_k = kappa^k * beta as the sequential fp32 product.
__device__ __forceinline__ float beta_at(const KParams& k, int it) {
    float b = k.beta;
    for (int i = 0; i < it; ++i) b = __fmul_rn(b, k.kappa);
    return b;
}

// Slow path of one evaluation for one lane: a group that needs the clamp or
// may have a non-zero proximal step (rare).  The lane's raw values are reloaded and ws = fl(w*s) recomputed (the
// same product as at init); returns the lane's partial sums of |r|^p, W_q and
// (when sp) fl((w - W_e)*s).
template <int DT, int AXIS, int E>
__device__ __forceinline__ float3 eval_lane_slow(const KParams k, const WarpTile w, float s, float z, int it, bool sp,
                                                 double* swe_out) {
    float err = 0.0f, sq = 0.0f;
    double swe = 0.0;
    const float beta = beta_at(k, it);
    const int64_t rb = AXIS == 1 ? 0 : w.j / k.cols, c = AXIS == 1 ? 0 : w.j % k.cols;
#pragma unroll 1
    for (int t = 0; t < E / kPiece; ++t) {  // one 8-element piece at a time: few live registers
        float x[kPiece];
        if (AXIS == 1) {
            unpack8<DT>(__ldg(reinterpret_cast<const uint4*>(k.W + w.j * k.g + w.part * E) + t), x);
        } else {
            const uint16_t* src = k.W + (rb * k.g + w.part * E + t * kPiece) * k.cols + c;
#pragma unroll
            for (int i = 0; i < kPiece; ++i) x[i] = bits_to_float<DT>(__ldg(src + i * k.cols));
        }
#pragma unroll
        for (int i = 0; i < kPiece; ++i) {
            const ElemEval ee = eval_elem(__fmul_rn(x[i], s), z, k.Lf);
            err += pow_pos(fabsf(ee.r), k.p);
            sq += ee.q;
            if (sp) {
                const float we = shrink_elem(ee.r, s, k.p, beta);
                swe += static_cast<double>(__fmul_rn(__fsub_rn(x[i], we), s));
            }
        }
    }
    *swe_out = swe;
    return make_float3(err, sq, 0.0f);
}

// One evaluation of zero-point z for a warp tile whose raw values are not kept
// in registers.  Fast path (warp-uniform): every group clamp-free and no
// proximal step possible -- then only v, round, r, |r|^p and W_q per element.
template <int DT, int AXIS, int E>
__device__ __forceinline__ void eval_lane_reload(const KParams& k, const WarpTile& w, const float* ws, float lmin,
                                                 float lmax, float s, float z, float z0, int it, float thr,
                                                 float* err_out, float* sq_out, bool* sp_out, double* swe_out) {
    const bool sp = w.valid && shrink_possible(s, z, z0, thr, k.Lf);
    const bool fast = __all_sync(kFull, !w.valid || (!sp && clamp_free(lmin, lmax, z, k.Lf)));
    float err = 0.0f, sq = 0.0f;
    double swe = 0.0;
    if (fast) {
        if (w.valid) fast_sums<E>(ws, z, k.p, &err, &sq);
    } else if (w.valid) {
        const float3 r = eval_lane_slow<DT, AXIS, E>(k, w, s, z, it, sp, &swe);
        err = r.x;
        sq = r.y;
    }
    *err_out = seg_sum(err, k.P);
    *sq_out = seg_sum(sq, k.P);
    if (__any_sync(kFull, sp)) swe = seg_sum_d(swe, k.P);
    *sp_out = sp;
    *swe_out = swe;
}

// Raw 16-bit data of this lane (axis 1): E/8 16-byte pieces, for prefetching.
template <int E>
__device__ __forceinline__ void load_raw1(const KParams& k, const WarpTile& w, uint4* raw) {
    const uint4* src = reinterpret_cast<const uint4*>(k.W + w.j * k.g + w.part * E);
#pragma unroll
    for (int t = 0; t < E / kPiece; ++t) raw[t] = w.valid ? __ldg(src + t) : make_uint4(0, 0, 0, 0);
}

// One tensor-mode iteration of a warp tile: evaluate z, add this lane's share
// of the group's error to its per-thread partial (tensor mode needs only the
// sum over all groups, so the error is not reduced over the group's lanes),
// step z.  Fast path: one vote, one reduction (of the sum of W_q).
template <int DT, int AXIS, int E, typename Acc>
__device__ __forceinline__ void tensor_iteration(const KParams& k, const WarpTile& w, const float* ws, float lmin,
                                                 float lmax, float s, float z0, int it, float thr, float spow,
                                                 F2 sws2, float inv_g, Acc& acc, float& z) {
    const bool sp = w.valid && shrink_possible(s, z, z0, thr, k.Lf);
    float err = 0.0f, sq = 0.0f;
    if (__all_sync(kFull, !w.valid || (!sp && clamp_free(lmin, lmax, z, k.Lf)))) {
        if (w.valid) fast_sums<E>(ws, z, k.p, &err, &sq);
        sq = seg_sum(sq, k.P);
        z = zero_from_sums_f2(sq, sws2, inv_g);
    } else {
        double swe = 0.0;
        if (w.valid) {
            const float3 r = eval_lane_slow<DT, AXIS, E>(k, w, s, z, it, sp, &swe);
            err = r.x;
            sq = r.y;
        }
        sq = seg_sum(sq, k.P);
        if (__any_sync(kFull, sp)) swe = seg_sum_d(swe, k.P);
        z = sp ? zero_from_sums(sq, swe, k.g) : zero_from_sums_f2(sq, sws2, inv_g);
    }
    if (w.valid) acc += static_cast<Acc>(err * spow);
}

// tensor_iteration that also stores the packed codes of the evaluated
// iterate (axis 1).  On the fast path the codes are the ones the evaluation
// rounds to (every v is clamp-free, so round-half-even is already in [0, L]),
// packed as they come: element e of the lane at bit e * NBITS of the lane's
// E * NBITS / 8 bytes, which start on a multiple of 4 * NBITS bytes (the
// packed buffer is 16-byte aligned, g >= 32).  Otherwise the codes are
// recomputed with the clamp after the step.
template <int DT, int E, int NBITS, typename Acc>
__device__ __forceinline__ void tensor_iteration_codes(const KParams& k, const WarpTile& w, const float* ws,
                                                       float lmin, float lmax, float s, float z0, int it, float thr,
                                                       float spow, F2 sws2, float inv_g, Acc& acc, float& z) {
    static_assert(E == 32, "one lane holds 32 elements");
    const bool sp = w.valid && shrink_possible(s, z, z0, thr, k.Lf);
    if (__all_sync(kFull, !w.valid || (!sp && clamp_free(lmin, lmax, z, k.Lf)))) {
        float err = 0.0f, sq = 0.0f;
        uint32_t pk[NBITS] = {};
        if (w.valid) {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const ElemEval e = eval_elem_nc(ws[i], z);
                err += pow_pos(fabsf(e.r), k.p);
                sq += e.q;
                const int b = i * NBITS;
                pk[b / 32] |= e.code << (b % 32);
                if (b % 32 + NBITS > 32) pk[b / 32 + 1] |= e.code >> (32 - b % 32);
            }
            uint8_t* dst = k.packed + (w.j * (k.g / kPiece) + w.part * (E / kPiece)) * NBITS;
            if (NBITS == 1) {
                *reinterpret_cast<uint32_t*>(dst) = pk[0];
            } else if (NBITS == 2) {
                *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1 % NBITS]);
            } else if (NBITS == 3) {
#pragma unroll
                for (int m = 0; m < NBITS; ++m) reinterpret_cast<uint32_t*>(dst)[m] = pk[m];
            } else {
#pragma unroll
                for (int m = 0; m < NBITS; m += 4)
                    reinterpret_cast<uint4*>(dst)[m / 4] =
                        make_uint4(pk[m], pk[(m + 1) % NBITS], pk[(m + 2) % NBITS], pk[(m + 3) % NBITS]);
            }
        }
        sq = seg_sum(sq, k.P);
        z = zero_from_sums_f2(sq, sws2, inv_g);
        if (w.valid) acc += static_cast<Acc>(err * spow);
    } else {
        const float ze = z;
        tensor_iteration<DT, 1, E>(k, w, ws, lmin, lmax, s, z0, it, thr, spow, sws2, inv_g, acc, z);
        if (w.valid) store_lane_codes_t<1, E, NBITS>(k, w, ws, ze);
    }
}

// tensor_iteration_codes with the bit width chosen by a warp-uniform switch.
template <int DT, int E, typename... Args>
__device__ __forceinline__ void tensor_iteration_codes_n(int nbits, Args&&... args) {
    switch (nbits) {
        case 1: tensor_iteration_codes<DT, E, 1>(args...); break;
        case 2: tensor_iteration_codes<DT, E, 2>(args...); break;
        case 3: tensor_iteration_codes<DT, E, 3>(args...); break;
        case 4: tensor_iteration_codes<DT, E, 4>(args...); break;
        default: tensor_iteration_codes<DT, E, 8>(args...); break;
    }
}

__device__ __forceinline__ double warp_sum_d(double x) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}

// ============================================================ tensor stop ==

// Resident CTAs per SM: 2 for 32 elements per lane (128 registers), 4 below
// (64 registers; the few spilled bytes cost less than the lost occupancy).
template <int DT, int AXIS, int E>
__global__ void __launch_bounds__(kRegThreads, E <= 16 ? 4 : 2)
    solve_tensor_kernel(const KParams k, int chunk, int write_outputs) {
    __shared__ float2 sred[kRegWarps];
    __shared__ double sacc[kChunkMax][kRegThreads];  // per-thread tensor error partials
    __shared__ float saccf[E <= 16 ? 1 : kChunkMax][kRegThreads];  // fp32 running partials (32-element tiles)
    __shared__ float sthr[kChunkMax];                 // shrink threshold of each iteration of the chunk
    __shared__ int sflag;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ntiles = num_warp_tiles<AXIS>(k);
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * kRegWarps;
    const int64_t G = k.G;
    const float inv_g = 1.0f / static_cast<float>(k.g);
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    const int iters = k.iters_eff;
    constexpr int C = chunk_len(E);
    const int nch = num_chunks(iters, C);
    // Stop rule on the tensor errors of iterations [0, k0) (same decision in
    // every CTA), as summarised by the last CTA of the last chunk that ran.
    const int k0 = chunk_begin(chunk, iters, C);
    int best_it = -1, stop_at = -1;
    if (k0 > 0) {
        stop_at = static_cast<int>(__ldcg(k.counters + kWordStopAt)) - 1;
        best_it = static_cast<int>(__ldcg(k.counters + kWordBestIt)) - 1;
    }
    const int prev_begin = chunk > 0 ? chunk_begin(chunk - 1, iters, C) : 0;
    bool finalize;
    if (stop_at >= 0) {
        if (stop_at < prev_begin || !write_outputs) return;  // outputs written elsewhere
        finalize = true;
    } else {
        finalize = chunk >= nch;
        if (finalize) best_it = iters - 1;
    }
    // z of every iteration of a chunk, two slots by chunk parity:
    // slot(c)[q][j] = z of iteration chunk_begin(c) + q, q = nk: the next chunk's start
    constexpr int kSlots = chunk_max(C) + 1;
    auto zslot = [&](int c, int q) { return k.t_zs + (static_cast<int64_t>(c & 1) * kSlots + q) * G; };

    if (finalize) {
        // the kept iterate lies in the last chunk run or the one before it: both slots intact
        const int kb = best_it < 0 ? 0 : best_it;  // iters == 0: z* = z0
        const int cb = chunk_of(kb, C, iters), b0 = chunk_begin(cb, iters, C);
        const float* Zc = zslot(cb, kb - b0);
        for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp; t < ntiles; t += wstride) {
            const WarpTile w = warp_tile<AXIS>(k, t);
            float x[E], ws[E];
            load_lane<DT, AXIS, E>(k, w, x);
            float s, z0, z;
            if (nch > 0) {  // s, z0 and the kept zero-point were stored by the chunks
                s = w.valid ? k.t_s[w.j] : 1.0f;
                z0 = w.valid ? k.t_z0[w.j] : 0.0f;
                z = w.valid ? Zc[w.j] : 0.0f;
#pragma unroll
                for (int i = 0; i < E; ++i) ws[i] = __fmul_rn(x[i], s);
            } else {  // iters == 0: z* = z0 from min/max
                float lmin, lmax;
                double sws;
                init_lane<E, false>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
                z = z0;
            }
            store_lane_codes<AXIS, E>(k, w, ws, z);
            float err_mean = 0.0f;
            if (k.dbg_err) {
                float err, sq;
                bool sp;
                double swe;
                const float beta = beta_at(k, kb);
                eval_lane<E>(k, w.valid, x, ws, s, z, z0, beta, shrink_threshold(beta, k.p), &err, &sq, &sp, &swe);
                err_mean = err * pow_pos(s, -k.p) / static_cast<float>(k.g);
            }
            if (w.valid && w.part == 0) store_group(k, w.j, s, z, kb, err_mean, &zmin, &zmax);
        }
        if (k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred);
        return;
    }

    // run iterations [k0, k1)
    const int k1 = chunk_begin(chunk + 1, iters, C);
    const int nk = k1 - k0;
    const float* const Zin = chunk > 0 ? zslot(chunk - 1, k0 - prev_begin) : nullptr;
    float* const Zcur = zslot(chunk, 0);
    // Streamed outputs: the last chunk also writes the outputs of its last
    // iterate.  They are the call's outputs whenever no tensor error rose
    // (the kept iterate is then the last one); otherwise the output kernel
    // overwrites every one of them.
    const bool spec = AXIS == 1 && last_chunk_outputs(E) && !write_outputs && k1 == iters;
    // per-thread tensor error partials: registers for small tiles, else shared
    constexpr int CM = chunk_max(C);
    double accr[CM] = {};
    for (int q = 0; q < CM; ++q) sacc[q][threadIdx.x] = 0.0;
    if constexpr (E > 16)
        for (int q = 0; q < CM; ++q) saccf[q][threadIdx.x] = 0.0f;
    if (threadIdx.x < CM) sthr[threadIdx.x] = shrink_threshold(beta_at(k, k0 + threadIdx.x), k.p);
    __syncthreads();
    constexpr bool kPrefetch = AXIS == 1 && E <= 16;
    int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp;
    uint4 raw[kPrefetch ? E / kPiece : 1];
    if (kPrefetch && t < ntiles) load_raw1<E>(k, warp_tile<AXIS>(k, t), raw);
    for (; t < ntiles; t += wstride) {
        const WarpTile w = warp_tile<AXIS>(k, t);
        float x[E], ws[E];
        if (kPrefetch) {
#pragma unroll
            for (int q = 0; q < E / kPiece; ++q) unpack8<DT>(raw[q], x + q * kPiece);
            if (t + wstride < ntiles) load_raw1<E>(k, warp_tile<AXIS>(k, t + wstride), raw);  // prefetch
            if (!w.valid) {
#pragma unroll
                for (int i = 0; i < E; ++i) x[i] = 0.0f;
            }
        } else {
            load_lane<DT, AXIS, E>(k, w, x);
        }
        float s, z0, z, lmin, lmax;
        double sws;
        if (k0 == 0) {
            init_lane<E>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
            if (w.valid && w.part == 0) {
                k.t_s[w.j] = s;
                k.t_z0[w.j] = z0;
                k.t_sws[w.j] = sws;
            }
            z = z0;
        } else {
            s = w.valid ? k.t_s[w.j] : 1.0f;
            z0 = w.valid ? k.t_z0[w.j] : 0.0f;
            sws = w.valid ? k.t_sws[w.j] : 0.0;
            z = w.valid ? Zin[w.j] : 0.0f;
            float xmn = FLT_MAX, xmx = -FLT_MAX;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                ws[i] = __fmul_rn(x[i], s);
                xmn = fminf(xmn, x[i]);
                xmx = fmaxf(xmx, x[i]);
            }
            lmin = w.valid ? __fmul_rn(xmn, s) : 0.0f;
            lmax = w.valid ? __fmul_rn(xmx, s) : 0.0f;
        }
        const float spow = pow_pos(s, -k.p);
        const F2 sws2 = split_f2(sws);
        // small tiles: unrolled over the chunk's iterations (more independent
        // work in flight); large tiles: a loop, to keep the code cache-resident
        float* const zrow = (w.valid && w.part == 0) ? Zcur + w.j : nullptr;
        if constexpr (E <= 16) {
#pragma unroll
            for (int q = 0; q < CM; ++q)
                if (q < nk) {
                    if (zrow) zrow[q * G] = z;
                    tensor_iteration<DT, AXIS, E>(k, w, ws, lmin, lmax, s, z0, k0 + q, sthr[q], spow, sws2, inv_g,
                                                  accr[q], z);
                }
        } else {
            const int nrun = spec ? nk - 1 : nk;  // with streamed outputs the last iteration also stores codes
#pragma unroll 1
            for (int q = 0; q < nrun; ++q) {
                if (zrow) zrow[q * G] = z;
                tensor_iteration<DT, AXIS, E>(k, w, ws, lmin, lmax, s, z0, k0 + q, sthr[q], spow, sws2, inv_g,
                                              saccf[q][threadIdx.x], z);
            }
            if constexpr (AXIS == 1 && last_chunk_outputs(E)) {
                if (spec) {
                    const int q = nk - 1;
                    const float zl = z;
                    if (zrow) zrow[q * G] = z;
                    tensor_iteration_codes_n<DT, E>(k.nbits, k, w, ws, lmin, lmax, s, z0, k0 + q, sthr[q], spow,
                                                    sws2, inv_g, saccf[q][threadIdx.x], z);
                    if (w.valid && w.part == 0) store_group(k, w.j, s, zl, iters - 1, 0.0f, &zmin, &zmax);
                }
            }
        }
        if (zrow) zrow[nk * G] = z;  // the next chunk's first zero-point
    }
    if (spec && k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred, kWordSpecZmin);
    // per-CTA partials (fixed order), then the last CTA sums them in a fixed order
    if constexpr (E <= 16) {
#pragma unroll
        for (int q = 0; q < CM; ++q) sacc[q][threadIdx.x] = accr[q];
    } else {
        // fp32 running sums of at most ~20 tiles per thread (relative error ~1e-6), then fp64
        for (int q = 0; q < CM; ++q) sacc[q][threadIdx.x] = static_cast<double>(saccf[q][threadIdx.x]);
    }
    __syncthreads();
    for (int q = warp; q < nk; q += kRegWarps) {
        double v = 0.0;
        for (int i = lane; i < kRegThreads; i += 32) v += sacc[q][i];
        v = warp_sum_d(v);
        if (lane == 0) k.tparts[static_cast<size_t>(q) * kMaxPartials + blockIdx.x] = v;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(k.counters + kWordTicket, 1u);
        sflag = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!sflag) return;
    __threadfence();
    // the tensor errors of iterations [0, k1): earlier ones from memory, this chunk's from the partials
    static_assert(kChunkMax * kRegThreads >= kMaxIters, "the error history fits in the partials' buffer");
    double* const serr = &sacc[0][0];  // free once the partials are written
    for (int it = threadIdx.x; it < k0; it += kRegThreads) serr[it] = __ldcg(k.etot + it);
    for (int q = warp; q < nk; q += kRegWarps) {
        double v = 0.0;
        for (unsigned b = lane; b < gridDim.x; b += 32)
            v += __ldcg(k.tparts + static_cast<size_t>(q) * kMaxPartials + b);
        v = warp_sum_d(v);
        if (lane == 0) {
            const double e = v / static_cast<double>(k.n);
            k.etot[k0 + q] = e;
            serr[k0 + q] = e;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // stop at the first iteration whose error is not below the best so far
        int bi = -1, sa = -1;
        double best = INFINITY;
        for (int it = 0; it < k1; ++it) {
            if (serr[it] < best) {
                best = serr[it];
                bi = it;
            } else {
                sa = it;
                break;
            }
        }
        k.counters[kWordStopAt] = static_cast<uint32_t>(sa + 1);
        k.counters[kWordBestIt] = static_cast<uint32_t>(bi + 1);
        k.counters[kWordTicket] = 0;
    }
}

// The outputs of a tensor-stop call, axis 1, no debug outputs.  The kept
// iterate (the stop rule's outcome) is in the workspace header.  When no error rose
// it is the last iterate, whose outputs the last chunk already wrote, and
// there is nothing left to do.  Otherwise a streaming pass over W (persistent
// CTAs, 8-element pieces, kOutPieces per thread with their loads issued
// together): the kept iterate's stored zero-point and the stored scale give
// the codes; the first piece of a group writes the group's scale and zero.
constexpr int kOutPieces = 4;  // pieces per thread of tensor_output_kernel, loads issued together

// Codes of one 8-element piece at (s, z), packed LSB first.  As in
// round_clamp, t = fl(clamp(fl(fl(w*s) + z), 0, L) + 1.5*2^23) holds the code
// in its low mantissa bits: bits(t) = bits(1.5*2^23) + code.  So the packed
// value is the sum of bits(t_i) << (i * NBITS) less the magic's share of that
// sum, all mod 2^32 (one multiply-add per element).
template <int DT, int NBITS>
__device__ __forceinline__ uint64_t piece_codes(const uint4 raw, float s, float z) {
    constexpr float Lf = static_cast<float>((1 << NBITS) - 1);
    constexpr int kPer = NBITS == 8 ? 4 : 8;  // codes per 32-bit word
    constexpr uint32_t kOnes = NBITS == 8 ? 0x01010101u
                               : NBITS == 4 ? 0x11111111u
                               : NBITS == 3 ? 0x00249249u
                               : NBITS == 2 ? 0x00005555u
                                            : 0x000000ffu;  // sum of 1 << (i * NBITS) over a word's codes
    constexpr uint32_t kMagicShare = kMagicBits * kOnes;     // mod 2^32
    float x[kPiece];
    unpack8<DT>(raw, x);
    uint32_t word[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < kPiece; ++i) {
        const float t = __fadd_rn(fminf(fmaxf(__fadd_rn(__fmul_rn(x[i], s), z), 0.0f), Lf), kMagic);
        word[i / kPer] += __float_as_uint(t) << ((i % kPer) * NBITS);
    }
    if (NBITS == 8)
        return static_cast<uint64_t>(word[0] - kMagicShare) | (static_cast<uint64_t>(word[1] - kMagicShare) << 32);
    return word[0] - kMagicShare;
}

template <int DT, int NBITS>
__global__ void __launch_bounds__(256) tensor_output_kernel(const KParams k) {
    __shared__ float2 sred[8];
    const int iters = k.iters_eff;
    // kept iterate: the stop rule's outcome, written by the last chunk that ran
    const int bi = static_cast<int>(__ldcg(k.counters + kWordBestIt)) - 1;
    const int kb = bi < 0 ? 0 : bi;
    if (kb == iters - 1 && last_chunk_outputs(k.E)) {  // no error rose: the last chunk wrote these outputs
        if (k.zero_nbits == 8 && blockIdx.x == 0 && threadIdx.x == 0) {
            k.counters[kWordZmin] = __ldcg(k.counters + kWordSpecZmin);
            k.counters[kWordZmax] = __ldcg(k.counters + kWordSpecZmax);
        }
        return;
    }
    const int C = chunk_len(k.E);
    const int cb = chunk_of(kb, C, iters), b0 = chunk_begin(cb, iters, C);
    const int64_t slots = chunk_max(C) + 1;
    const float* Zc = k.t_zs + ((cb & 1) * slots + (kb - b0)) * k.G;
    int log_ppg = 0;
    while ((kPiece << log_ppg) < k.g) ++log_ppg;  // pieces per group: g / 8, a power of two
    float zmin = FLT_MAX, zmax = -FLT_MAX;
    const int64_t npieces = k.n / kPiece;
    const int64_t nblk = (npieces + 256 * kOutPieces - 1) / (256 * kOutPieces);
    for (int64_t blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
        const int64_t pc0 = blk * 256 * kOutPieces + threadIdx.x;
        uint4 raw[kOutPieces];
        float sv[kOutPieces], zv[kOutPieces];
#pragma unroll
        for (int u = 0; u < kOutPieces; ++u) {
            const int64_t pc = pc0 + u * 256;
            if (pc < npieces) {
                const int64_t j = pc >> log_ppg;
                raw[u] = __ldg(reinterpret_cast<const uint4*>(k.W) + pc);
                sv[u] = __ldg(k.t_s + j);
                zv[u] = __ldcg(Zc + j);
            }
        }
#pragma unroll
        for (int u = 0; u < kOutPieces; ++u) {
            const int64_t pc = pc0 + u * 256;
            if (pc >= npieces) break;
            const uint64_t v = piece_codes<DT, NBITS>(raw[u], sv[u], zv[u]);
            uint8_t* dst = k.packed + pc * NBITS;
            if (NBITS == 8) *reinterpret_cast<uint64_t*>(dst) = v;
            else if (NBITS == 4) *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(v);
            else if (NBITS == 2) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(v);
            else if (NBITS == 1) *dst = static_cast<uint8_t>(v);
            else {
                dst[0] = static_cast<uint8_t>(v);
                dst[1] = static_cast<uint8_t>(v >> 8);
                dst[2] = static_cast<uint8_t>(v >> 16);
            }
            if ((pc & ((int64_t{1} << log_ppg) - 1)) == 0)
                store_group(k, pc >> log_ppg, sv[u], zv[u], kb, 0.0f, &zmin, &zmax);
        }
    }
    if (k.zero_nbits == 8) merge_zero_range<8>(k, zmin, zmax, sred);
}

// 16-byte copies global -> shared that bypass the registers (and L1).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ============================================ tensor stop, W kept on chip ==
//
// solve_tensor_resident_kernel (tensor stop, axis 1): one cooperative launch
// runs every iteration of every group.  Each warp owns a fixed run of T warp
// tiles.  The iterations go in rounds of C: in a round the warp visits
// each of its tiles once, copies its raw values from W (cp.async, two buffers
// per warp), forms fl(w*s) once and runs the round's iterations on it in
// registers.  The launcher only takes this path when W fits in half the L2, so
// after the first round those copies are L2 hits, and when each group's state
// between rounds -- float4 (s, z0, the group's largest w*s, s^-p), float2 (the
// sum of w*s split into two floats) and the zero-point to continue from --
// fits in the warp's shared memory.  The zero-point of every iteration goes to
// a ring of 2*C + 2 slots per group in the workspace, from which the kept one
// is read at the end.
//
// The tensor error of iteration m is the sum over all groups: one grid-wide
// reduction per iteration, and no grid barrier.  At the end of a round every
// warp adds its fp64 partials to its CTA's shared memory; the CTA's last warp
// to arrive sums the CTA's eight in warp order and posts them to the workspace
// with a global arrival counter; the warp that brings the counter to the grid
// size sums all CTAs' partials of each of the round's iterations in CTA order
// (the same on every run with the same grid), applies the stop rule to the
// state published for the previous round, and publishes (best error so far,
// first rise) for the round.  A warp starts round r only after round r-2 is
// published, so the wait is normally already satisfied, and leaves the loop
// when a rise is reported: the kept iterate, the one before the first rise,
// then lies in the last 2*C + 1 iterations run, all still in the ring.
// Iterations past the rise run speculatively and are discarded.  Every wait
// is bounded by the global timer: after the limit the warp records
// HQQ_ERR_TIMEOUT in the workspace's status word, the other warps see it in
// their next wait and give up too, and no outputs are written.
// Iterations per round: 10 for tiles of 32 elements per lane (measured 2-5 %
// faster than 8: one reload of the tiles fewer in 20 iterations), 4 below
// (the workspace's zero-point slots, 24 and 10, hold the ring of 2*C + 2).
__host__ __device__ constexpr int res_c(int E) { return E >= 32 ? 10 : 4; }
__host__ __device__ constexpr int res_slots(int E) { return 2 * res_c(E) + 2; }
constexpr unsigned long long kResWaitNs = 1000000000ull;

__device__ __forceinline__ unsigned long long res_now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Published decision of round r: words kWordDec + 8*(r mod 4) + (0-1: tensor
// error of the round's last iteration, 2-3: best error so far, 4: first rise
// + 1 or 0, 5: r + 1 once published).
__device__ __forceinline__ uint32_t* res_dec(const KParams& k, int r) { return k.counters + kWordDec + 8 * (r & 3); }

// Lane-0 wait until round r is published; false after the limit (recording
// the timeout) or when another warp already gave up.
__device__ __forceinline__ bool res_wait_dec(const KParams& k, int r, unsigned long long limit_ns) {
    volatile uint32_t* tag = res_dec(k, r) + 5;
    volatile uint32_t* status = k.counters;
    if (*tag == static_cast<uint32_t>(r + 1)) {
        __threadfence();
        return true;
    }
    const unsigned long long t0 = res_now_ns();
    while (*tag != static_cast<uint32_t>(r + 1)) {
        if (*status != 0u) return false;
        if (res_now_ns() - t0 > limit_ns) {
            atomicCAS(k.counters, 0u, kStatusTimeout);
            return false;
        }
        __nanosleep(128);
    }
    __threadfence();
    return true;
}

// Lane-0 wait of a warp for the first rise (or -1) reported by round r,
// through its CTA's copy in shared memory: the CTA knows the rounds < *pub, the
// rises in rise[r mod 4]; one warp at a time (*poll) reads the workspace for
// the CTA and copies what was published, the others wait on shared memory, so
// the published words see one reader per CTA.  False after the limit
// (recording the timeout) or when another warp already gave up.
__device__ __forceinline__ bool res_cta_dec(const KParams& k, int r, volatile int* pub, volatile int* rise,
                                            int* poll, unsigned long long limit_ns, int* rise_out) {
    volatile uint32_t* status = k.counters;
    unsigned long long t0 = 0;
    unsigned spins = 0;
    for (;;) {
        if (*pub > r) {
            *rise_out = rise[r & 3];
            return true;
        }
        if (t0 == 0) t0 = res_now_ns();
        if (atomicCAS(poll, 0, 1) == 0) {  // this warp reads the workspace for the CTA
            bool ok = true;
            while (*pub <= r) {
                const int rr = *pub;
                const uint32_t* d = res_dec(k, rr);
                if (*reinterpret_cast<volatile const uint32_t*>(d + 5) == static_cast<uint32_t>(rr + 1)) {
                    __threadfence();
                    rise[rr & 3] = static_cast<int>(__ldcg(d + 4)) - 1;
                    __threadfence_block();
                    *pub = rr + 1;
                    continue;
                }
                if ((++spins & 15u) == 0u && *status != 0u) {
                    ok = false;
                    break;
                }
                if (res_now_ns() - t0 > limit_ns) {
                    atomicCAS(k.counters, 0u, kStatusTimeout);
                    ok = false;
                    break;
                }
                __nanosleep(128);
            }
            atomicExch(poll, 0);
            if (!ok) return false;
            continue;
        }
        if ((++spins & 63u) == 0u && *status != 0u) return false;
        if (res_now_ns() - t0 > limit_ns) {
            atomicCAS(k.counters, 0u, kStatusTimeout);
            return false;
        }
        __nanosleep(64);
    }
}

__device__ __forceinline__ double res_load_d(const uint32_t* w) {
    const uint32_t lo = __ldcg(w), hi = __ldcg(w + 1);
    return __hiloint2double(static_cast<int>(hi), static_cast<int>(lo));
}

// Called by the whole warp after its CTA posted the partials of round r
// (iterations k0 .. k0+nk-1, row c of `parts` for iteration k0+c) as the last
// of nc CTAs: sum each iteration's partials in CTA order (a lane's loads for
// the nk iterations are issued together), apply the stop rule in iteration
// order, publish.
template <int C>
__device__ __forceinline__ bool res_publish(const KParams& k, int r, int k0, int nk, const double* parts, int nc,
                                            unsigned long long limit_ns) {
    const int lane = threadIdx.x & 31;
    double v[C] = {};
    for (int b = lane; b < nc; b += 32) {
        double t[C];
#pragma unroll
        for (int c = 0; c < C; ++c) t[c] = c < nk ? __ldcg(parts + static_cast<size_t>(c) * nc + b) : 0.0;
#pragma unroll
        for (int c = 0; c < C; ++c) v[c] += t[c];
    }
#pragma unroll
    for (int c = 0; c < C; ++c) v[c] = warp_sum_d(v[c]);
    bool ok = true;
    if (lane == 0) {
        double best = INFINITY, e = 0.0;
        int rise = -1;
        if (r > 0) {
            ok = res_wait_dec(k, r - 1, limit_ns);
            if (ok) {
                const uint32_t* d = res_dec(k, r - 1);
                best = res_load_d(d + 2);
                rise = static_cast<int>(__ldcg(d + 4)) - 1;
            }
        }
        if (ok) {
#pragma unroll
            for (int c = 0; c < C; ++c) {
                if (c >= nk) break;
                e = v[c] / static_cast<double>(k.n);
                if (rise < 0) {  // first iteration whose error is not below the best so far
                    if (e < best) best = e;
                    else rise = k0 + c;
                }
            }
            uint32_t* d = res_dec(k, r);
            d[0] = static_cast<uint32_t>(__double2loint(e));
            d[1] = static_cast<uint32_t>(__double2hiint(e));
            d[2] = static_cast<uint32_t>(__double2loint(best));
            d[3] = static_cast<uint32_t>(__double2hiint(best));
            d[4] = static_cast<uint32_t>(rise + 1);
            __threadfence();
            atomicExch(d + 5, static_cast<uint32_t>(r + 1));
        }
    }
    return __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
}

// Shared memory of one warp, in bytes: two copy buffers of a tile (64*E bytes
// each), then per group of its T tiles a float4, a float2 and a float (the
// state between rounds); rounded up to 16 bytes so that every warp's region
// starts 16-byte aligned.
__host__ __device__ constexpr size_t res_warp_bytes(int E, int T, int gpw) {
    return (static_cast<size_t>(128 * E) + static_cast<size_t>(T) * gpw * (16 + 8 + 4) + 15) & ~static_cast<size_t>(15);
}

template <int DT, int E>
__global__ void __launch_bounds__(kRegThreads, E <= 16 ? 4 : 2)
    solve_tensor_resident_kernel(const KParams k, int T, unsigned long long limit_ns) {
    constexpr int C = res_c(E);
    constexpr int kSlots = res_slots(E);
    extern __shared__ uint4 dyn_smem[];
    __shared__ float2 sred[kRegWarps];
    __shared__ double sacc[C][kRegThreads];      // this round's error partial of each thread
    __shared__ double cpart[4][C][kRegWarps];    // warps' partials, by round mod 4
    __shared__ unsigned ccount[4];                   // warps that posted them (cumulative)
    __shared__ int dpub, dpoll, drise[4];            // the CTA's copy of the published rounds
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < 4) ccount[threadIdx.x] = 0u;
    if (threadIdx.x == 0) dpub = dpoll = 0;
    __syncthreads();
    const int gpw = 32 >> k.logP;
    const int slot = lane >> k.logP;
    const int nst = T * gpw;  // state entries of this warp
    unsigned char* const base = reinterpret_cast<unsigned char*>(dyn_smem) + res_warp_bytes(E, T, gpw) * warp;
    uint4* const buf = reinterpret_cast<uint4*>(base);              // [2][E/8][32]
    float4* const stA = reinterpret_cast<float4*>(base + 128 * E);  // [nst]
    float2* const stB = reinterpret_cast<float2*>(stA + nst);       // [nst]
    float* const stZ = reinterpret_cast<float*>(stB + nst);         // [nst]
    const int nc = static_cast<int>(gridDim.x);
    const int gw = static_cast<int>(blockIdx.x) * kRegWarps + warp;
    const int64_t ntiles = num_warp_tiles<1>(k);
    const int64_t t0 = static_cast<int64_t>(gw) * T;
    const int nt = t0 >= ntiles ? 0 : static_cast<int>(ntiles - t0 < T ? ntiles - t0 : T);
    const float inv_g = 1.0f / static_cast<float>(k.g);
    const int iters = k.iters_eff;
    const int64_t G = k.G;
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    // The copies of this warp's tiles form one cyclic stream (tile q of copy
    // number c = q + nt * round).  Copy c goes to buffer c mod 2, as the
    // tile's 16-byte pieces in order, piece p of the tile by lane p mod 32 (so
    // each instruction copies 512 contiguous bytes), stored where its owner
    // lane reads it: piece p belongs to lane p / (E/8), as that lane's piece
    // p mod (E/8), at buf[(c&1)][p mod (E/8)][p / (E/8)].
    int issued = 0, qi = 0, used = 0;
    auto issue = [&]() {
        if (nt > 0) {
            const int64_t e0 = (t0 + qi) * 32 * E;  // first element of the tile
            const int64_t n_el = k.n - e0;          // elements left in W (the last tile may be partial)
#pragma unroll
            for (int u = 0; u < E / kPiece; ++u) {
                const int p = u * 32 + lane;
                if (static_cast<int64_t>(p) * kPiece < n_el)
                    cp_async16(buf + ((issued & 1) * (E / kPiece) + p % (E / kPiece)) * 32 + p / (E / kPiece),
                               k.W + e0 + static_cast<int64_t>(p) * kPiece);
            }
            if (++qi == nt) qi = 0;
        }
        cp_async_commit();
        ++issued;
    };
    // the next tile of the stream as fp32 (zeros for lanes past the last group)
    auto next_tile = [&](int q, float* x, WarpTile& w) {
        __syncwarp();  // every lane has read the buffer the next copy overwrites
        issue();
        cp_async_wait<1>();
        __syncwarp();  // every lane's share of this copy has landed
        w = warp_tile<1>(k, t0 + q);
        if (w.valid) {
#pragma unroll
            for (int u = 0; u < E / kPiece; ++u) unpack8<DT>(buf[((used & 1) * (E / kPiece) + u) * 32 + lane], x + u * kPiece);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) x[i] = 0.0f;
        }
        ++used;
    };

    issue();
    bool ok = true;
    int kept = -1;  // kept iterate once a rise is known
    float beta = k.beta;  // beta of the round's first iteration (sequential fp32 products)
    const int nrounds = (iters + C - 1) / C;
    int r = 0;
    for (; r < nrounds; ++r) {
        const int k0 = r * C;
        const int nk = iters - k0 < C ? iters - k0 : C;
        if (r >= 2) {
            int rise = -1;
            if (lane == 0) ok = res_cta_dec(k, r - 2, &dpub, drise, &dpoll, limit_ns, &rise);
            ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
            rise = __shfl_sync(kFull, rise, 0);
            if (!ok) break;
            if (rise >= 0) {
                kept = rise > 0 ? rise - 1 : 0;
                break;
            }
        }
        float thr[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            thr[c] = shrink_threshold(beta, k.p);
            if (c < nk) beta = __fmul_rn(beta, k.kappa);
        }
#pragma unroll
        for (int c = 0; c < C; ++c) sacc[c][threadIdx.x] = 0.0;
        for (int q = 0; q < nt; ++q) {
            float x[E], ws[E];
            WarpTile w;
            next_tile(q, x, w);
            const int i = q * gpw + slot;
            const bool writer = w.valid && w.part == 0;
            float s, z0, z, lmin, lmax, spow;
            F2 sws2;
            if (r == 0) {
                double sws;
                init_lane<E>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
                spow = pow_pos(s, -k.p);
                sws2 = split_f2(sws);
                z = z0;
                const float gmax = seg_max(lmax, k.P);
                if (writer) {
                    stA[i] = make_float4(s, z0, gmax, spow);
                    stB[i] = make_float2(sws2.hi, sws2.lo);
                }
            } else {
                const float4 a = w.valid ? stA[i] : make_float4(1.0f, 0.0f, 0.0f, 1.0f);
                const float2 b = w.valid ? stB[i] : make_float2(0.0f, 0.0f);
                s = a.x;
                z0 = a.y;
                lmin = -z0;  // fl(min w * s), exactly: rounding is symmetric
                lmax = a.z;  // the group's; the warp-wide clamp test is the same as with the lanes' own
                spow = a.w;
                sws2 = F2{b.x, b.y};
                z = w.valid ? stZ[i] : 0.0f;
                const uint64_t s2 = f2_pack(s, s);
#pragma unroll
                for (int e = 0; e < E; e += 2) f2_unpack(f2_mul(f2_pack(x[e], x[e + 1]), s2), ws[e], ws[e + 1]);
            }
            float* const zring = writer ? k.t_zs + w.j : nullptr;
#pragma unroll 1
            for (int c = 0; c < nk; ++c) {
                if (zring) zring[static_cast<int64_t>((k0 + c) % kSlots) * G] = z;
                tensor_iteration<DT, 1, E>(k, w, ws, lmin, lmax, s, z0, k0 + c, thr[c], spow, sws2, inv_g,
                                           sacc[c][threadIdx.x], z);
            }
            if (writer) stZ[i] = z;
        }
        // post this warp's partials; the CTA's last warp posts the CTA's, and
        // the grid's last CTA publishes the round
        double v[C];
#pragma unroll
        for (int c = 0; c < C; ++c) v[c] = warp_sum_d(sacc[c][threadIdx.x]);
        double* const parts = k.tparts + static_cast<size_t>(r & 3) * C * nc;
        unsigned last = 0;
        if (lane == 0) {
#pragma unroll
            for (int c = 0; c < C; ++c) cpart[r & 3][c][warp] = v[c];
            __threadfence_block();
            const unsigned ctarget = static_cast<unsigned>(r / 4 + 1) * kRegWarps;
            if (atomicAdd(&ccount[r & 3], 1u) + 1u == ctarget) {
                __threadfence_block();
                for (int c = 0; c < nk; ++c) {
                    double cv = 0.0;
                    for (int w = 0; w < kRegWarps; ++w) cv += cpart[r & 3][c][w];
                    parts[static_cast<size_t>(c) * nc + blockIdx.x] = cv;
                }
                __threadfence();
                const uint32_t target = static_cast<uint32_t>(r / 4 + 1) * static_cast<uint32_t>(nc);
                last = atomicAdd(k.counters + kWordArrive + (r & 3), 1u) + 1u == target;
                if (last) __threadfence();
            }
        }
        if (__shfl_sync(kFull, last, 0)) {
            ok = res_publish<C>(k, r, k0, nk, parts, nc, limit_ns);
            if (!ok) break;
        }
    }
    if (ok && kept < 0) {  // every round ran: the rule over all of them
        int rise = -1;
        if (lane == 0) ok = res_cta_dec(k, nrounds - 1, &dpub, drise, &dpoll, limit_ns, &rise);
        ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
        rise = __shfl_sync(kFull, rise, 0);
        kept = rise >= 0 ? (rise > 0 ? rise - 1 : 0) : iters - 1;
    }
    if (ok) {  // outputs of the kept iterate
        __threadfence();  // the ring's zero-points, written by this warp's lanes, are read back below
        __syncwarp();
        const float* const zk = k.t_zs + static_cast<int64_t>(kept % kSlots) * G;
        float bk = k.beta;
        for (int i = 0; i < kept; ++i) bk = __fmul_rn(bk, k.kappa);
        for (int q = 0; q < nt; ++q) {
            float x[E], ws[E];
            WarpTile w;
            next_tile(q, x, w);
            const int i = q * gpw + slot;
            const float4 a = w.valid ? stA[i] : make_float4(1.0f, 0.0f, 0.0f, 1.0f);
            const float s = a.x, z0 = a.y;
            const float z = w.valid ? __ldcg(zk + w.j) : 0.0f;
            const uint64_t s2 = f2_pack(s, s);
#pragma unroll
            for (int e = 0; e < E; e += 2) f2_unpack(f2_mul(f2_pack(x[e], x[e + 1]), s2), ws[e], ws[e + 1]);
            store_lane_codes<1, E>(k, w, ws, z);
            float err_mean = 0.0f;
            if (k.dbg_err) {
                float err, sq;
                bool sp;
                double swe;
                eval_lane<E>(k, w.valid, x, ws, s, z, z0, bk, shrink_threshold(bk, k.p), &err, &sq, &sp, &swe);
                err_mean = err * a.w * inv_g;
            }
            if (w.valid && w.part == 0) store_group(k, w.j, s, z, kept, err_mean, &zmin, &zmax);
        }
    }
    cp_async_wait<0>();
    if (k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred);
}

// Diagnostic: the resident solver's bounded wait on a decision that nothing
// publishes, with a short limit; it gives up and records the timeout in the
// workspace's status word exactly as the solver does.
__global__ void res_wait_selftest_kernel(KParams k, unsigned long long limit_ns) {
    if (threadIdx.x == 0) res_wait_dec(k, 0, limit_ns);
}

// ============================================================= group stop ==

// One pass of the group-stop solver (see the file comment).  Entries are warp
// tile slots: axis 1, entry e is group e; axis 0, entry e is lane group
// e % gpw of warp tile e / gpw (32/P neighbouring columns of one row block).
// State and survivor lists are indexed by the entry's offset in the slice.
struct PassArgs {
    const uint32_t* in;         // entries of this pass (nullptr: every entry of the slice, in order)
    const uint32_t* in_count;   // number of entries in `in`
    uint32_t* out;              // entries still running after the pass (nullptr: the last pass)
    uint32_t* out_count;
    float4* state;              // [2 * slice]: (z, best error, kept zero, s), (z0, max w*s, sum w*s hi, lo)
    int* state_it;              // [slice]: iteration of the kept zero
    int64_t e0;                 // first entry of the slice
    int64_t n;                  // entries in the slice
    int k0;                     // iterations every group of this pass has done
    int evals;                  // evaluations in this pass
};

template <int AXIS>
__device__ __forceinline__ bool entry_group(const KParams& k, int64_t e, int64_t* j) {
    if (AXIS == 1) {
        *j = e;
        return e < k.G;
    }
    const int gpw = 32 >> k.logP;
    const int64_t t = e >> (5 - k.logP);
    const int64_t ncb = (k.cols + gpw - 1) / gpw;
    const int64_t rb = t / ncb, c = (t % ncb) * gpw + (e & (gpw - 1));
    *j = rb * k.cols + c;
    return c < k.cols;
}

__host__ __device__ inline int64_t num_entries(int64_t rows, int64_t cols, int64_t G, int g, int axis, int logP) {
    const int gpw = 32 >> logP;
    if (axis == 1) return G;
    return (rows / g) * ((cols + gpw - 1) / gpw) * gpw;
}

// Three CTAs per SM (80 registers) for 32 elements per lane, four (64) below:
// occupancy beats the few spilled bytes.
template <int DT, int AXIS, int E>
__global__ void __launch_bounds__(kRegThreads, E <= 16 ? 4 : 3) solve_group_kernel(const KParams k, const PassArgs pa) {
    __shared__ float2 sred[kRegWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gpw = 32 >> k.logP;
    const int part = lane & (k.P - 1);
    const int64_t count = pa.in ? static_cast<int64_t>(__ldcg(pa.in_count)) : pa.n;
    const int64_t ntiles = (count + gpw - 1) / gpw;
    const bool stop_group = k.stop_mode == 0;
    const float inv_g = 1.0f / static_cast<float>(k.g);
    // smallest shrink threshold of the run (beta only grows): a conservative gate
    const float thr = shrink_threshold(k.beta_last, k.p);
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp; t < ntiles;
         t += static_cast<int64_t>(gridDim.x) * kRegWarps) {
        const int64_t slot = t * gpw + (lane >> k.logP);
        int64_t el = -1;  // entry offset in the slice
        if (slot < count) el = pa.in ? static_cast<int64_t>(pa.in[slot]) : slot;
        WarpTile w;
        w.part = part;
        w.j = 0;
        w.valid = el >= 0 && entry_group<AXIS>(k, pa.e0 + el, &w.j);
        float x[E], ws[E];
        load_lane<DT, AXIS, E>(k, w, x);
        float s, z0, z, be, zb, lmin, lmax, wsmax;
        F2 sws2;
        int bi;
        if (pa.k0 == 0) {
            double sws;
            init_lane<E>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
            sws2 = split_f2(sws);
            wsmax = seg_max(w.valid ? lmax : -FLT_MAX, k.P);
            z = zb = z0;
            be = INFINITY;
            bi = 0;
        } else {
            float4 a = make_float4(0.0f, INFINITY, 0.0f, 1.0f), b = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            bi = 0;
            if (w.valid) {
                a = __ldcg(pa.state + 2 * el);
                b = __ldcg(pa.state + 2 * el + 1);
                bi = __ldcg(pa.state_it + el);
            }
            z = a.x;
            be = a.y;
            zb = a.z;
            s = a.w;
            z0 = b.x;
            wsmax = b.y;
            sws2 = F2{b.z, b.w};
#pragma unroll
            for (int i = 0; i < E; ++i) ws[i] = __fmul_rn(x[i], s);
            lmin = -z0;  // fl(min w * s) = -fl(-min w * s) = -z0
            lmax = wsmax;
        }
        bool active = w.valid && pa.k0 < k.iters_eff;
        for (int e = 0; e < pa.evals && __any_sync(kFull, active); ++e) {
            const int it = pa.k0 + e;
            WarpTile wa = w;
            wa.valid = active;
            float err, sq;
            bool sp;
            double swe;
            eval_lane_reload<DT, AXIS, E>(k, wa, ws, lmin, lmax, s, z, z0, it, thr, &err, &sq, &sp, &swe);
            if (active) {
                const bool improved = err < be;
                if (improved) {
                    be = err;
                    zb = z;
                    bi = it;
                }
                bool stop = (stop_group && !improved) || it >= k.iters_eff - 1;
                if (!stop) {
                    const float zn = sp ? zero_from_sums(sq, swe, k.g) : zero_from_sums_f2(sq, sws2, inv_g);
                    if (stop_group && zn == z) stop = true;  // fixed point: the next error equals this one
                    else z = zn;
                }
                if (stop) active = false;
            }
        }
        if (!pa.out) active = false;  // the last pass: evals reach iters_eff - 1, every group has stopped
        if (active) {
            // still running: leave the state for the next pass
            if (part == 0) {
                pa.state[2 * el] = make_float4(z, be, zb, s);
                pa.state[2 * el + 1] = make_float4(z0, wsmax, sws2.hi, sws2.lo);
                pa.state_it[el] = bi;
            }
        } else if (w.valid) {
            store_lane_codes<AXIS, E>(k, w, ws, zb);
            if (part == 0) {
                const float err_mean = k.dbg_err ? be * pow_pos(s, -k.p) / static_cast<float>(k.g) : 0.0f;
                store_group(k, w.j, s, zb, bi, err_mean, &zmin, &zmax);
            }
        }
        const unsigned run = __ballot_sync(kFull, active && part == 0);
        if (run) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(pa.out_count, static_cast<uint32_t>(__popc(run)));
            base = __shfl_sync(kFull, base, 0);
            if (active && part == 0) pa.out[base + __popc(run & ((1u << lane) - 1u))] = static_cast<uint32_t>(el);
        }
    }
    if (k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred);
}

// ====================================================== one-pass group stop ==
//
// solve_group_onepass_kernel (axis 1, group or no stop): every group is read
// from HBM once and stays on chip from its first evaluation to its packed
// codes.  A warp owns S = 32/P group slots (a slot is the P lanes of one
// group) and works in rounds:
//   fresh round: the next chunk of S consecutive groups (32*E contiguous
//     16-bit elements, staged in shared memory by cp.async, the chunk after it
//     already in flight) fills every slot; each is initialised and evaluated
//     twice -- most groups stop there (group stop needs at least two
//     evaluations) -- or, without early stopping, to the end;
//   survivor round: when the warp's pool of running groups in shared memory
//     holds S of them (or nothing else is left), S of them are restored to the
//     slots and evaluated until fewer than S/2 (3S/4 for 32 elements per lane)
//     still run (or, at the end, all have stopped).
// After a round the stopped groups are packed and stored, and the running
// ones go to the pool (raw values, scale, state: the codes of a group are
// never recomputed from a second read of W).  Slots run at different
// iteration indices; beta only matters on the rare proximal path, which takes
// each slot's own.

// Packed min/max of eight 16-bit values held in a uint4 (fp16 or bf16; the
// order of 16-bit values equals the order of their fp32 conversions).
template <int DT>
__device__ __forceinline__ void minmax8(const uint4 u, uint32_t& mn2, uint32_t& mx2) {
    const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (DT == 0) {
            asm("min.f16x2 %0, %0, %1;" : "+r"(mn2) : "r"(x[i]));
            asm("max.f16x2 %0, %0, %1;" : "+r"(mx2) : "r"(x[i]));
        } else {
            asm("min.bf16x2 %0, %0, %1;" : "+r"(mn2) : "r"(x[i]));
            asm("max.bf16x2 %0, %0, %1;" : "+r"(mx2) : "r"(x[i]));
        }
    }
}

// Error-free sum of two floats (Knuth's TwoSum): s + e == a + b exactly.
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bp = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bp)), __fsub_rn(b, bp));
}

// A fresh group for this lane's slot (fresh) from its raw 16-bit values:
// min/max -> s, z0; fp32 w*s into ws; the sum of w*s as an unevaluated pair
// hi + lo (hi = fl(hi + lo)) over the group's P lanes, accumulated by pairwise
// TwoSum (no fp64 conversions: those issue on the pipe the solver is bound
// by); and this lane's range of w*s.  Executed by every lane of the warp
// (shuffles); lanes without a fresh group keep ws and the outputs unchanged.
template <int DT, int E>
__device__ __forceinline__ void init_fresh(const KParams& k, bool fresh, const uint4* raw, float* ws, float& s,
                                           float& z0, F2& sws2, float& lmin, float& lmax) {
    uint32_t mn2 = raw[0].x, mx2 = raw[0].x;
#pragma unroll
    for (int t = 0; t < E / kPiece; ++t) minmax8<DT>(raw[t], mn2, mx2);
    const float lmn = fminf(bits_to_float<DT>(mn2 & 0xffffu), bits_to_float<DT>(mn2 >> 16));
    const float lmx = fmaxf(bits_to_float<DT>(mx2 & 0xffffu), bits_to_float<DT>(mx2 >> 16));
    const float mn = seg_min(lmn, k.P), mx = seg_max(lmx, k.P);
    float sn = kScaleCap;
    if (mx > mn) sn = fminf(__fdiv_rn(k.Lf, __fsub_rn(mx, mn)), kScaleCap);
    float hi = 0.0f, lo = 0.0f;
    if (fresh) {
        s = sn;
        z0 = __fmul_rn(-mn, sn);
        lmin = __fmul_rn(lmn, sn);
        lmax = __fmul_rn(lmx, sn);
        const uint64_t s2 = f2_pack(sn, sn);
        uint64_t acc[2] = {f2_pack(0.0f, 0.0f), f2_pack(0.0f, 0.0f)};
        uint64_t cmp[2] = {f2_pack(0.0f, 0.0f), f2_pack(0.0f, 0.0f)};
#pragma unroll
        for (int t = 0; t < E / kPiece; ++t) {
            float x[kPiece];
            unpack8<DT>(raw[t], x);
#pragma unroll
            for (int i = 0; i < kPiece; i += 2) {
                const int c = (i >> 1) & 1;  // two independent chains of packed pairs
                const uint64_t w2 = f2_mul(f2_pack(x[i], x[i + 1]), s2);
                f2_unpack(w2, ws[t * kPiece + i], ws[t * kPiece + i + 1]);
                // TwoSum of the running pair and the two new products
                const uint64_t sum = f2_add(acc[c], w2);
                const uint64_t bp = f2_sub(sum, acc[c]);
                cmp[c] = f2_add(cmp[c], f2_add(f2_sub(acc[c], f2_sub(sum, bp)), f2_sub(w2, bp)));
                acc[c] = sum;
            }
        }
        float a0, a1, a2, a3, c0, c1, h0, h1, e0, e1, a, e2;
        f2_unpack(acc[0], a0, a1);
        f2_unpack(acc[1], a2, a3);
        f2_unpack(f2_add(cmp[0], cmp[1]), c0, c1);
        two_sum(a0, a1, h0, e0);
        two_sum(a2, a3, h1, e1);
        two_sum(h0, h1, a, e2);
        const float c = __fadd_rn(__fadd_rn(c0, c1), __fadd_rn(__fadd_rn(e0, e1), e2));
        hi = __fadd_rn(a, c);  // Fast2Sum (|a| >= |c|)
        lo = __fsub_rn(c, __fsub_rn(hi, a));
    }
    for (int o = 1; o < k.P; o <<= 1) {
        const float h2 = __shfl_xor_sync(kFull, hi, o), l2 = __shfl_xor_sync(kFull, lo, o);
        float h, e;
        two_sum(hi, h2, h, e);
        const float l = __fadd_rn(__fadd_rn(lo, l2), e);
        hi = __fadd_rn(h, l);
        lo = __fsub_rn(l, __fsub_rn(hi, h));
    }
    if (fresh) sws2 = F2{hi, lo};
}

// Packed codes of this lane's E elements at zero-point z (axis 1); cf: every
// v = fl(fl(w*s) + z) of the lane is clamp-free, so the code is read from the
// rounding sum's low mantissa bits without the clamp.
template <int E, int NBITS>
__device__ __forceinline__ void store_codes_lane(const KParams& k, int64_t j, int part, const float* ws, float z,
                                                 bool cf) {
    constexpr float Lf = static_cast<float>((1 << NBITS) - 1);
    constexpr int kWords = (E * NBITS + 31) / 32;
    uint32_t wd[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) wd[w] = 0u;
    const uint64_t z2 = f2_pack(z, z), m2 = f2_pack(kMagic, kMagic);
    if (cf && NBITS != 3) {
        // t = fl(fl(w*s + z) + 1.5*2^23) holds its code in the low mantissa bits,
        // bits(t) = bits(1.5*2^23) + code: a word is the sum of bits(t_i) << (i*NBITS)
        // less the magic's share (mod 2^32) -- one shifted add per code
#pragma unroll
        for (int i = 0; i < E; i += 2) {
            float t0, t1;
            f2_unpack(f2_add(f2_add(f2_pack(ws[i], ws[i + 1]), z2), m2), t0, t1);
            wd[(i * NBITS) / 32] += __float_as_uint(t0) << ((i * NBITS) % 32);
            wd[((i + 1) * NBITS) / 32] += __float_as_uint(t1) << (((i + 1) * NBITS) % 32);
        }
        constexpr uint32_t kOnes = NBITS == 8 ? 0x01010101u
                                   : NBITS == 4 ? 0x11111111u
                                   : NBITS == 2 ? 0x55555555u
                                                : 0xffffffffu;  // sum of 1 << (i*NBITS % 32) over a full word
        constexpr int kPerWord = 32 / NBITS;
#pragma unroll
        for (int w = 0; w < kWords; ++w) {
            const int n_in = E - w * kPerWord < kPerWord ? E - w * kPerWord : kPerWord;  // codes in this word
            const uint32_t ones = n_in == kPerWord ? kOnes : (kOnes & ((1u << (n_in * NBITS)) - 1u));
            wd[w] -= kMagicBits * ones;
        }
    } else {
#pragma unroll
        for (int i = 0; i < E; i += 2) {
            uint32_t c2[2];
            if (cf) {
                float t0, t1;
                f2_unpack(f2_add(f2_add(f2_pack(ws[i], ws[i + 1]), z2), m2), t0, t1);
                c2[0] = __float_as_uint(t0) - kMagicBits;
                c2[1] = __float_as_uint(t1) - kMagicBits;
            } else {
                round_clamp(__fadd_rn(ws[i], z), Lf, &c2[0]);
                round_clamp(__fadd_rn(ws[i + 1], z), Lf, &c2[1]);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int b = (i + h) * NBITS;
                wd[b / 32] |= c2[h] << (b % 32);
                if (b % 32 + NBITS > 32) wd[b / 32 + 1] |= c2[h] >> (32 - b % 32);
            }
        }
    }
    constexpr int kBytes = E * NBITS / 8;
    uint8_t* dst = k.packed + (j * (k.g / E) + part) * kBytes;
    if (kBytes % 16 == 0) {
#pragma unroll
        for (int q = 0; q < kBytes / 16; ++q)
            reinterpret_cast<uint4*>(dst)[q] = make_uint4(wd[4 * q], wd[4 * q + 1], wd[4 * q + 2], wd[4 * q + 3]);
    } else if (kBytes == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[kWords > 1 ? 1 : 0]);
    } else if (kBytes == 4) {
        *reinterpret_cast<uint32_t*>(dst) = wd[0];
    } else if (kBytes == 2) {
        *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(wd[0]);
    } else if (kBytes == 1) {
        *dst = static_cast<uint8_t>(wd[0]);
    } else if (kBytes == 12) {  // 3-bit, E = 32: 4-byte aligned
#pragma unroll
        for (int q = 0; q < 3; ++q) reinterpret_cast<uint32_t*>(dst)[q] = wd[q];
    } else if (kBytes == 6) {  // 3-bit, E = 16: 2-byte aligned
#pragma unroll
        for (int q = 0; q < 3; ++q) reinterpret_cast<uint16_t*>(dst)[q] = static_cast<uint16_t>(wd[q / 2] >> (16 * (q & 1)));
    } else {  // 3-bit, E = 8: 3 bytes
#pragma unroll
        for (int q = 0; q < kBytes; ++q) dst[q] = static_cast<uint8_t>(wd[0] >> (8 * q));
    }
}

template <int E>
__device__ __forceinline__ void store_codes_lane_n(const KParams& k, int64_t j, int part, const float* ws, float z,
                                                   bool cf) {
    switch (k.nbits) {
        case 1: store_codes_lane<E, 1>(k, j, part, ws, z, cf); break;
        case 2: store_codes_lane<E, 2>(k, j, part, ws, z, cf); break;
        case 3: store_codes_lane<E, 3>(k, j, part, ws, z, cf); break;
        case 4: store_codes_lane<E, 4>(k, j, part, ws, z, cf); break;
        default: store_codes_lane<E, 8>(k, j, part, ws, z, cf); break;
    }
}

// Shared memory of one warp of the one-pass kernel, in uint4 units: two chunk
// buffers of 32*E 16-bit values, and a pool of 2S running groups stored as 64
// lane records (a group's P lanes), structure of arrays: record field f of
// record r at pool[f * 64 + r], fields 0 .. E/8-1 the lane's raw values, then
// (s, z, z0, best error), (kept zero, sum hi, sum lo, lane min w*s),
// (lane max w*s, kept iterate, iteration, group lo), (group hi, -, -, -).
__host__ __device__ constexpr int onepass_fields(int E) { return E / kPiece + 4; }
__host__ __device__ constexpr int onepass_warp_uint4(int E) { return 8 * E + 64 * onepass_fields(E); }
constexpr int kPoolRecords = 64;
__host__ __device__ constexpr int onepass_ctas(int E) { return E >= 32 ? 2 : (E == 16 ? 3 : 4); }

template <int DT, int E>
__global__ void __launch_bounds__(kRegThreads, onepass_ctas(E))
    solve_group_onepass_kernel(const KParams k, int64_t nchunks) {
    extern __shared__ uint4 dyn_smem[];
    __shared__ float2 sred[kRegWarps];
    constexpr int F = onepass_fields(E);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4* const cbuf = dyn_smem + warp * onepass_warp_uint4(E);  // [2][4E]
    uint4* const pool = cbuf + 8 * E;                              // [F][64]
    const int logP = k.logP;
    const int part = lane & (k.P - 1);
    const int slot = lane >> logP;
    const int S = 32 >> logP;  // group slots per warp
    const bool stop_group = k.stop_mode == 0;
    const int m_fresh = stop_group ? 2 : k.iters_eff;  // evaluations of a fresh round
    const float inv_g = 1.0f / static_cast<float>(k.g);
    const float thr = shrink_threshold(k.beta_last, k.p);  // smallest threshold of the run: a conservative gate
    unsigned long long* const counter = reinterpret_cast<unsigned long long*>(k.counters + kWordChunk);
    const unsigned leader = lane & ~(k.P - 1);  // first lane of this lane's slot
    const unsigned below = (1u << leader) - 1u;
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    // take the next chunk and start copying it into buffer b; returns its group count
    auto fetch = [&](int b, int64_t& c_out) -> int {
        unsigned long long c = 0;
        if (lane == 0) c = atomicAdd(counter, 1ull);
        c = __shfl_sync(kFull, c, 0);
        int cnt = 0;
        if (static_cast<int64_t>(c) < nchunks) {
            const int64_t g0 = static_cast<int64_t>(c) * S;
            cnt = static_cast<int>(k.G - g0 < S ? k.G - g0 : S);
            if (lane * E < cnt * k.g) {
                const uint4* src = reinterpret_cast<const uint4*>(k.W + g0 * k.g + lane * E);
#pragma unroll
                for (int t = 0; t < E / kPiece; ++t) cp_async16(cbuf + b * 4 * E + lane * (E / kPiece) + t, src + t);
            }
        }
        cp_async_commit();
        c_out = static_cast<int64_t>(c);
        return cnt;
    };

    int cur = 0;
    int64_t cur_c, nxt_c;
    int cur_cnt = fetch(0, cur_c);
    int nxt_cnt = fetch(1, nxt_c);
    int pool_n = 0;  // running groups in the pool

    float ws[E];
    float s = 1.0f, z = 0.0f, z0 = 0.0f, be = INFINITY, zb = 0.0f, lmin = 0.0f, lmax = 0.0f;
    F2 sws2{0.0f, 0.0f};
    int bi = 0, it = 0;
    int64_t j = 0;

    for (;;) {
        const bool survivor = pool_n >= S || (cur_cnt == 0 && pool_n > 0);
        if (!survivor && cur_cnt == 0) break;  // nothing left
        bool has = false;  // this slot holds a group this round
        uint4 raw[E / kPiece];
        if (survivor) {
            const int n = pool_n < S ? pool_n : S;
            has = slot < n;
            if (has) {
                const int r = (pool_n - n + slot) * k.P + part;
#pragma unroll
                for (int t = 0; t < E / kPiece; ++t) raw[t] = pool[t * kPoolRecords + r];
                const uint4 f0 = pool[(E / kPiece) * kPoolRecords + r];
                const uint4 f1 = pool[(E / kPiece + 1) * kPoolRecords + r];
                const uint4 f2 = pool[(E / kPiece + 2) * kPoolRecords + r];
                const uint4 f3 = pool[(E / kPiece + 3) * kPoolRecords + r];
                s = __uint_as_float(f0.x);
                z = __uint_as_float(f0.y);
                z0 = __uint_as_float(f0.z);
                be = __uint_as_float(f0.w);
                zb = __uint_as_float(f1.x);
                sws2 = F2{__uint_as_float(f1.y), __uint_as_float(f1.z)};
                lmin = __uint_as_float(f1.w);
                lmax = __uint_as_float(f2.x);
                bi = static_cast<int>(f2.y);
                it = static_cast<int>(f2.z);
                j = static_cast<int64_t>((static_cast<uint64_t>(f3.x) << 32) | f2.w);
                const uint64_t s2 = f2_pack(s, s);
#pragma unroll
                for (int t = 0; t < E / kPiece; ++t) {  // fl(w*s), as at initialisation
                    float x[kPiece];
                    unpack8<DT>(raw[t], x);
#pragma unroll
                    for (int i = 0; i < kPiece; i += 2)
                        f2_unpack(f2_mul(f2_pack(x[i], x[i + 1]), s2), ws[t * kPiece + i], ws[t * kPiece + i + 1]);
                }
            }
            pool_n -= n;
            __syncwarp();  // every lane has read its record before records are rewritten at the end of the round
        } else {
            cp_async_wait<1>();
            __syncwarp();  // this chunk has landed in every lane's copy
            has = slot < cur_cnt;
            const uint4* src = cbuf + cur * 4 * E + lane * (E / kPiece);
#pragma unroll
            for (int t = 0; t < E / kPiece; ++t) raw[t] = has ? src[t] : make_uint4(0, 0, 0, 0);
            j = cur_c * S + slot;
            __syncwarp();  // every lane has read the buffer: refill it with the chunk after next
            int64_t c_new;
            const int cnt_new = fetch(cur, c_new);
            cur ^= 1;
            cur_c = nxt_c;
            cur_cnt = nxt_cnt;
            nxt_c = c_new;
            nxt_cnt = cnt_new;
            init_fresh<DT, E>(k, has, raw, ws, s, z0, sws2, lmin, lmax);
            if (has) {
                z = zb = z0;
                be = INFINITY;
                bi = 0;
                it = 0;
            }
        }
        bool alive = has && it < k.iters_eff;
        // ---------------------------------------------- evaluations -------
        const bool more = pool_n > 0 || cur_cnt > 0;  // work beyond this round
        for (int e = 0;; ++e) {
            const int n_alive = __popc(__ballot_sync(kFull, part == 0 && alive));
            if (n_alive == 0) break;
            if (!survivor && e >= m_fresh) break;
            // a survivor round ends when too few of its slots still run (tiles of 32 elements per
            // lane return them to the pool sooner: measured 2.5% faster at g128, 2% slower at g16)
            if (survivor && more && (E >= 32 ? 4 * n_alive < 3 * S : 2 * n_alive < S)) break;
            WarpTile wt;
            wt.valid = alive;
            wt.j = j;
            wt.part = part;
            float err, sq;
            bool sp;
            double swe;
            eval_lane_reload<DT, 1, E>(k, wt, ws, lmin, lmax, s, z, z0, it, thr, &err, &sq, &sp, &swe);
            if (alive) {
                const bool improved = err < be;
                if (improved) {
                    be = err;
                    zb = z;
                    bi = it;
                }
                bool stop = (stop_group && !improved) || it >= k.iters_eff - 1;
                if (!stop) {
                    const float zn = sp ? zero_from_sums(sq, swe, k.g) : zero_from_sums_f2(sq, sws2, inv_g);
                    if (stop_group && zn == z) stop = true;  // fixed point: the next error equals this one
                    else z = zn;
                }
                if (stop) alive = false;
                else ++it;
            }
        }
        // ------------------------------------------ stopped: outputs -------
        if (has && !alive) {
            store_codes_lane_n<E>(k, j, part, ws, zb, clamp_free(lmin, lmax, zb, k.Lf));
            if (part == 0) {
                const float err_mean = k.dbg_err ? be * pow_pos(s, -k.p) * inv_g : 0.0f;
                store_group(k, j, s, zb, bi, err_mean, &zmin, &zmax);
            }
        }
        // ------------------------------------------ running: to the pool ---
        const unsigned run = __ballot_sync(kFull, part == 0 && alive);
        if (alive) {
            const int r = (pool_n + __popc(run & below)) * k.P + part;
#pragma unroll
            for (int t = 0; t < E / kPiece; ++t) pool[t * kPoolRecords + r] = raw[t];
            pool[(E / kPiece) * kPoolRecords + r] =
                make_uint4(__float_as_uint(s), __float_as_uint(z), __float_as_uint(z0), __float_as_uint(be));
            pool[(E / kPiece + 1) * kPoolRecords + r] = make_uint4(__float_as_uint(zb), __float_as_uint(sws2.hi),
                                                                   __float_as_uint(sws2.lo), __float_as_uint(lmin));
            pool[(E / kPiece + 2) * kPoolRecords + r] =
                make_uint4(__float_as_uint(lmax), static_cast<uint32_t>(bi), static_cast<uint32_t>(it),
                           static_cast<uint32_t>(static_cast<uint64_t>(j)));
            pool[(E / kPiece + 3) * kPoolRecords + r] =
                make_uint4(static_cast<uint32_t>(static_cast<uint64_t>(j) >> 32), 0u, 0u, 0u);
        }
        pool_n += __popc(run);
        __syncwarp();  // pool writes visible to the whole warp before the next round reads them
    }
    cp_async_wait<0>();
    if (k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred);
}

// ============================================= half-precision variant ==
//
// solve_half_kernel (group / no stop, axis 1, fp16 input): the solver in half
// precision, as the pages run it on the GPU ("Speed: from hours to minutes"),
// with the steps of "Outlier-aware optimization without gradients".  Reading
// H: every element-wise value is rounded to fp16 (to nearest, ties to even):
// s = h(min(L/(max-min), 2e4)), z0 = h(-min*s), ws = h(w*s), v = h(ws + z)
// (add.rn.f16x2), W_q = clamp(round(v), 0, L), r = h(v - W_q); the error of z
// is the sum of h(|r|^p) (|r|^p through the hardware base-2 log and
// exponential in fp32, then rounded to fp16); each z update rounds an exact
// mean to fp16 once; the rare proximal step rounds d = h(fl32(r/s)),
// W_e = h(shrink(d)) and h(h(w - W_e)*s).  A warp holds a tile of 32/P groups
// in registers (ws as packed f16x2 pairs) and runs it until every group has
// stopped; W is read once (again only on the rare proximal path).
__device__ __forceinline__ uint32_t h2_add(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ float h_lo(uint32_t x) { return __half2float(__ushort_as_half(static_cast<unsigned short>(x))); }
__device__ __forceinline__ float h_hi(uint32_t x) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(x >> 16)));
}
__device__ __forceinline__ float h_round(float x) { return __half2float(__float2half_rn(x)); }
__device__ __forceinline__ uint32_t h2_splat(float x) {
    const uint32_t b = __half_as_ushort(__float2half_rn(x));
    return b | (b << 16);
}
constexpr uint32_t kHalfMagic2 = 0x66006600u;  // 1536 in both halves: adding it rounds |v| < 512 to an integer

// Slow path of one evaluation for one lane (a clamp is needed or the proximal
// step may be non-zero): W re-read one 16-byte piece at a time; err, sq and
// (sp) the exact sum of h(h(w - W_e)*s) accumulate.
template <int E>
__device__ __forceinline__ void half_eval_slow(const KParams& k, int64_t j, int part, float s, float z, float beta,
                                               bool sp, float* err, float* sq, double* swe) {
    const __half zh = __float2half_rn(z);
    const uint4* src = reinterpret_cast<const uint4*>(k.W + j * k.g + part * E);
#pragma unroll 1
    for (int t = 0; t < E / kPiece; ++t) {
        float x[kPiece];
        unpack8<0>(__ldg(src + t), x);
#pragma unroll
        for (int i = 0; i < kPiece; ++i) {
            const float wsv = h_round(__fmul_rn(x[i], s));  // the fp16 product is exact in fp32: one rounding
            const float v = __half2float(__hadd(__float2half_rn(wsv), zh));
            const float q = fminf(fmaxf(rintf(v), 0.0f), k.Lf);
            const float r = h_round(__fsub_rn(v, q));  // v - q is exact in fp32
            *err = __fadd_rn(*err, h_round(pow_pos(fabsf(r), k.p)));
            *sq = __fadd_rn(*sq, q);
            if (sp) {
                const float d = h_round(__fdiv_rn(r, s));
                const float we = h_round(shrink_elem(d, 1.0f, k.p, beta));
                const float a = __half2float(__double2half(static_cast<double>(x[i]) - static_cast<double>(we)));
                *swe += static_cast<double>(h_round(__fmul_rn(a, s)));
            }
        }
    }
}

// Packed codes of this lane's E elements at zero-point z: clamp(round(h(ws + z))).
template <int E, int NBITS>
__device__ __forceinline__ void store_codes_half(const KParams& k, int64_t j, int part, const uint32_t* ws2,
                                                 float z) {
    constexpr float Lf = static_cast<float>((1 << NBITS) - 1);
    constexpr int kWords = (E * NBITS + 31) / 32;
    uint32_t wd[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) wd[w] = 0u;
    const uint32_t z2 = h2_splat(z);
#pragma unroll
    for (int i = 0; i < E; i += 2) {
        const uint32_t v = h2_add(ws2[i / 2], z2);
        const uint32_t c2[2] = {static_cast<uint32_t>(fminf(fmaxf(rintf(h_lo(v)), 0.0f), Lf)),
                                static_cast<uint32_t>(fminf(fmaxf(rintf(h_hi(v)), 0.0f), Lf))};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int b = (i + h) * NBITS;
            wd[b / 32] |= c2[h] << (b % 32);
            if (b % 32 + NBITS > 32) wd[b / 32 + 1] |= c2[h] >> (32 - b % 32);
        }
    }
    constexpr int kBytes = E * NBITS / 8;
    uint8_t* dst = k.packed + (j * (k.g / E) + part) * kBytes;
#pragma unroll
    for (int q = 0; q < kBytes; ++q) dst[q] = static_cast<uint8_t>(wd[q / 4] >> (8 * (q % 4)));
}

template <int E>
__device__ __forceinline__ void store_codes_half_n(const KParams& k, int64_t j, int part, const uint32_t* ws2,
                                                   float z) {
    switch (k.nbits) {
        case 1: store_codes_half<E, 1>(k, j, part, ws2, z); break;
        case 2: store_codes_half<E, 2>(k, j, part, ws2, z); break;
        case 3: store_codes_half<E, 3>(k, j, part, ws2, z); break;
        case 4: store_codes_half<E, 4>(k, j, part, ws2, z); break;
        default: store_codes_half<E, 8>(k, j, part, ws2, z); break;
    }
}

template <int E>
__global__ void __launch_bounds__(kRegThreads, 3) solve_half_kernel(const KParams k) {
    __shared__ float2 sred[kRegWarps];
    const int warp = threadIdx.x >> 5;
    const bool stop_group = k.stop_mode == 0;
    const float thr = shrink_threshold(k.beta_last, k.p);  // smallest threshold of the run: a conservative gate
    const int64_t ntiles = num_warp_tiles<1>(k);
    float zmin = FLT_MAX, zmax = -FLT_MAX;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp; t < ntiles;
         t += static_cast<int64_t>(gridDim.x) * kRegWarps) {
        const WarpTile w = warp_tile<1>(k, t);
        uint4 raw[E / kPiece];
        const uint4* src = reinterpret_cast<const uint4*>(k.W + w.j * k.g + w.part * E);
#pragma unroll
        for (int q = 0; q < E / kPiece; ++q) raw[q] = w.valid ? __ldg(src + q) : make_uint4(0, 0, 0, 0);
        // initialisation: s, z0, ws = h(w*s) as f16x2 pairs, the exact sum of ws, this lane's ws range
        uint32_t mn2 = raw[0].x, mx2 = raw[0].x;
#pragma unroll
        for (int q = 0; q < E / kPiece; ++q) minmax8<0>(raw[q], mn2, mx2);
        const float lmn = fminf(h_lo(mn2), h_hi(mn2)), lmx = fmaxf(h_lo(mx2), h_hi(mx2));
        const float mn = seg_min(lmn, k.P), mx = seg_max(lmx, k.P);
        float s = kScaleCap;
        if (mx > mn) s = fminf(__fdiv_rn(k.Lf, __fsub_rn(mx, mn)), kScaleCap);
        s = h_round(s);
        const float z0 = h_round(__fmul_rn(-mn, s));
        uint32_t ws2[E / 2];
        double acc = 0.0;
#pragma unroll
        for (int q = 0; q < E / kPiece; ++q) {
            float x[kPiece];
            unpack8<0>(raw[q], x);
#pragma unroll
            for (int i = 0; i < kPiece; i += 2) {
                const __half2 h2 = __floats2half2_rn(__fmul_rn(x[i], s), __fmul_rn(x[i + 1], s));
                ws2[(q * kPiece + i) / 2] = *reinterpret_cast<const uint32_t*>(&h2);
                acc += static_cast<double>(__low2float(h2)) + static_cast<double>(__high2float(h2));
            }
        }
        const double sws = seg_sum_d(w.valid ? acc : 0.0, k.P);
        const float wsmin = h_round(__fmul_rn(lmn, s)), wsmax = h_round(__fmul_rn(lmx, s));
        float z = z0, zb = z0, be = INFINITY;
        int bi = 0;
        bool active = w.valid && k.iters_eff > 0;
        for (int it = 0; __any_sync(kFull, active); ++it) {
            const float beta = beta_at(k, it);
            const bool sp = active && shrink_possible(s, z, z0, thr, k.Lf);
            const __half zh = __float2half_rn(z);
            const bool cf = __half2float(__hadd(__float2half_rn(wsmin), zh)) >= -0.5f &&
                            __half2float(__hadd(__float2half_rn(wsmax), zh)) < k.Lf + 0.5f;
            float err = 0.0f, sq = 0.0f;
            double swe = 0.0;
            if (__all_sync(kFull, !active || (!sp && cf))) {
                if (active) {
                    const uint32_t z2 = h2_splat(z);
#pragma unroll
                    for (int i = 0; i < E / 2; ++i) {
                        const uint32_t v = h2_add(ws2[i], z2);
                        const uint32_t qv = h2_sub(h2_add(v, kHalfMagic2), kHalfMagic2);
                        const uint32_t r = h2_sub(v, qv) & 0x7fff7fffu;  // |r|, exact
                        err = __fadd_rn(err, h_round(pow_pos(h_lo(r), k.p)));
                        err = __fadd_rn(err, h_round(pow_pos(h_hi(r), k.p)));
                        sq = __fadd_rn(sq, __fadd_rn(h_lo(qv), h_hi(qv)));
                    }
                }
            } else if (active) {
                half_eval_slow<E>(k, w.j, w.part, s, z, beta, sp, &err, &sq, &swe);
            }
            err = seg_sum(err, k.P);
            sq = seg_sum(sq, k.P);
            if (__any_sync(kFull, sp)) swe = seg_sum_d(swe, k.P);
            if (active) {
                const bool improved = err < be;
                if (improved) {
                    be = err;
                    zb = z;
                    bi = it;
                }
                bool stop = (stop_group && !improved) || it >= k.iters_eff - 1;
                if (!stop) {
                    const double m = (static_cast<double>(sq) - (sp ? swe : sws)) / static_cast<double>(k.g);
                    const float zn = __half2float(__double2half(m));
                    if (stop_group && zn == z) stop = true;  // fixed point: the next error equals this one
                    else z = zn;
                }
                if (stop) active = false;
            }
        }
        if (w.valid) {
            store_codes_half_n<E>(k, w.j, w.part, ws2, zb);
            if (w.part == 0) {
                const float err_mean = k.dbg_err ? be * pow_pos(s, -k.p) / static_cast<float>(k.g) : 0.0f;
                store_group(k, w.j, s, zb, bi, err_mean, &zmin, &zmax);
            }
        }
    }
    if (k.zero_nbits == 8) merge_zero_range<kRegWarps>(k, zmin, zmax, sred);
}

// ------------------------------------------------------- 8-bit zero ------

// One RTN quantiser for all kept zeros of the tensor, from their min/max
// (merged into the workspace header by the solver kernels).
__global__ void __launch_bounds__(256) zero_q8_kernel(const float* zbest, int64_t G, const uint32_t* counters,
                                                       uint8_t* zq, float* meta) {
    float mn = 0.0f, mx = 0.0f;
    if (G > 0) {
        mn = key_value(~__ldcg(counters + kWordZmin));
        mx = key_value(__ldcg(counters + kWordZmax));
    }
    float sz = kScaleCap;
    if (mx > mn) sz = fminf(__fdiv_rn(255.0f, __fsub_rn(mx, mn)), kScaleCap);
    const float zz = __fmul_rn(-mn, sz);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        meta[0] = __fdiv_rn(1.0f, sz);
        meta[1] = zz;
    }
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; j < G;
         j += static_cast<int64_t>(gridDim.x) * 256) {
        uint32_t code;
        round_clamp(__fadd_rn(__fmul_rn(zbest[j], sz), zz), 255.0f, &code);
        zq[j] = static_cast<uint8_t>(code);
    }
}

// ------------------------------------------------------ 8-bit scales -----

// The "_s*" variant (table footnote of "Benchmark results"/"Llama-2"): one
// round-to-nearest 8-bit quantiser per run of S consecutive fp16 scales, from
// the run's min and max (sc = 255/(max-min), 1 for a constant run; zc =
// -min*sc; meta (1/sc, zc)).  HBM-bound: 2 bytes read, 1 written per scale.
__device__ __forceinline__ float2 scale8_pair(float mn, float mx) {
    const float sc = mx > mn ? __fdiv_rn(255.0f, __fsub_rn(mx, mn)) : 1.0f;
    return make_float2(sc, __fmul_rn(-mn, sc));
}

__device__ __forceinline__ uint32_t scale8_code(float v, float2 p) {
    uint32_t code;
    round_clamp(__fadd_rn(__fmul_rn(v, p.x), p.y), 255.0f, &code);
    return code;
}

// Any S: one warp per run, lanes stride over the run.
__device__ __forceinline__ void scale8_run(const uint16_t* scale, int64_t G, int S, int64_t r, uint8_t* codes,
                                           float* meta) {
    const int lane = threadIdx.x & 31;
    const int64_t k0 = r * S;
    const int len = static_cast<int>(G - k0 < S ? G - k0 : S);
    float mn = FLT_MAX, mx = -FLT_MAX;
    for (int i = lane; i < len; i += 32) {
        const float v = __half2float(__ushort_as_half(__ldg(scale + k0 + i)));
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
    mn = seg_min(mn, 32);
    mx = seg_max(mx, 32);
    const float2 p = scale8_pair(mn, mx);
    for (int i = lane; i < len; i += 32)
        codes[k0 + i] = static_cast<uint8_t>(scale8_code(__half2float(__ushort_as_half(__ldg(scale + k0 + i))), p));
    if (lane == 0) {
        meta[2 * r] = __fdiv_rn(1.0f, p.x);
        meta[2 * r + 1] = p.y;
    }
}

__global__ void __launch_bounds__(256) scale8_kernel(const uint16_t* scale, int64_t G, int S, uint8_t* codes,
                                                      float* meta) {
    const int64_t nruns = (G + S - 1) / S;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); r < nruns;
         r += static_cast<int64_t>(gridDim.x) * 8)
        scale8_run(scale, G, S, r, codes, meta);
}

// S == 128, 16-byte aligned scales and codes: a warp takes 4 runs, 8 lanes
// per run, 16 consecutive scales per lane (two 16-byte loads, one 16-byte
// store of codes); a warp whose runs are not all full uses scale8_run.
__global__ void __launch_bounds__(256) scale8_kernel_128(const uint16_t* scale, int64_t G, uint8_t* codes,
                                                          float* meta) {
    const int lane = threadIdx.x & 31, part = lane & 7;
    const int64_t nruns = (G + 127) / 128;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); w * 4 < nruns;
         w += static_cast<int64_t>(gridDim.x) * 8) {
        if ((w + 1) * 4 * 128 > G) {  // the tail: a partial run or fewer than 4 runs
            for (int64_t r = w * 4; r < nruns && r < (w + 1) * 4; ++r) scale8_run(scale, G, 128, r, codes, meta);
            continue;
        }
        const int64_t r = w * 4 + (lane >> 3);
        const int64_t e0 = r * 128 + part * 16;
        const uint4* src = reinterpret_cast<const uint4*>(scale + e0);
        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
        float v[16];
        unpack8<0>(u0, v);
        unpack8<0>(u1, v + 8);
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int i = 1; i < 16; ++i) {
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
        mn = seg_min(mn, 8);
        mx = seg_max(mx, 8);
        const float2 p = scale8_pair(mn, mx);
        uint32_t c[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            c[t] = scale8_code(v[4 * t], p) | (scale8_code(v[4 * t + 1], p) << 8) |
                   (scale8_code(v[4 * t + 2], p) << 16) | (scale8_code(v[4 * t + 3], p) << 24);
        *reinterpret_cast<uint4*>(codes + e0) = make_uint4(c[0], c[1], c[2], c[3]);
        if (part == 0) {
            meta[2 * r] = __fdiv_rn(1.0f, p.x);
            meta[2 * r + 1] = p.y;
        }
    }
}

// -------------------------------------------------------- dequantise -----

template <int OUT_DT>
__device__ __forceinline__ uint16_t float_to_out(float x) {
    if (OUT_DT == 0) return __half_as_ushort(__float2half_rn(x));
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint64_t load_piece(const uint8_t* src, int nbits) {
    switch (nbits) {
        case 1: return *src;
        case 2: return *reinterpret_cast<const uint16_t*>(src);
        case 4: return *reinterpret_cast<const uint32_t*>(src);
        case 8: return *reinterpret_cast<const uint64_t*>(src);
        default:
            return static_cast<uint64_t>(src[0]) | (static_cast<uint64_t>(src[1]) << 8) |
                   (static_cast<uint64_t>(src[2]) << 16);
    }
}

struct DqParams {
    const uint8_t* packed;
    const uint16_t* scale;     // fp16 scales, or
    const uint8_t* scale_q;    // 8-bit scale codes with
    const float* scale_meta;   // (1/sc, zc) per run of scale_group (null: fp16 scales)
    int scale_group;
    const void* zero;
    const float* meta;
    int64_t rows, cols;
    int nbits, g, zero_nbits;
    uint16_t* out;
};

__device__ __forceinline__ float dq_scale(const DqParams& d, int64_t j) {
    if (!d.scale_meta) return __half2float(__ushort_as_half(d.scale[j]));
    const float* m = d.scale_meta + 2 * (j / d.scale_group);
    return __fmul_rn(__fsub_rn(static_cast<float>(d.scale_q[j]), m[1]), m[0]);
}

__device__ __forceinline__ float dq_zero(const DqParams& d, int64_t j) {
    if (d.zero_nbits == 16) return __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(d.zero)[j]));
    const float zq = static_cast<float>(reinterpret_cast<const uint8_t*>(d.zero)[j]);
    return __fmul_rn(__fsub_rn(zq, d.meta[1]), d.meta[0]);
}

template <int OUT_DT, int AXIS>
__global__ void __launch_bounds__(256) dequant_kernel(const DqParams d) {
    const uint32_t mask = (1u << d.nbits) - 1u;
    if (AXIS == 1) {
        const int64_t npieces = d.rows * d.cols / kPiece;
        for (int64_t pc = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; pc < npieces;
             pc += static_cast<int64_t>(gridDim.x) * 256) {
            const uint64_t v = load_piece(d.packed + pc * d.nbits, d.nbits);
            const int64_t j = pc * kPiece / d.g;
            const float z = dq_zero(d, j);
            const float sc = dq_scale(d, j);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float q0 = static_cast<float>(static_cast<uint32_t>(v >> ((2 * i) * d.nbits)) & mask);
                const float q1 = static_cast<float>(static_cast<uint32_t>(v >> ((2 * i + 1) * d.nbits)) & mask);
                o[i] = static_cast<uint32_t>(float_to_out<OUT_DT>(__fmul_rn(__fsub_rn(q0, z), sc))) |
                       (static_cast<uint32_t>(float_to_out<OUT_DT>(__fmul_rn(__fsub_rn(q1, z), sc))) << 16);
            }
            reinterpret_cast<uint4*>(d.out)[pc] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
        const int64_t n = (d.rows / kPiece) * d.cols;
        for (int64_t u = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; u < n;
             u += static_cast<int64_t>(gridDim.x) * 256) {
            const int64_t m = u / d.cols, c = u % d.cols;
            uint64_t v = 0;
            for (int b = 0; b < d.nbits; ++b)
                v |= static_cast<uint64_t>(d.packed[(m * d.nbits + b) * d.cols + c]) << (8 * b);
            const int64_t j = (m * kPiece / d.g) * d.cols + c;
            const float z = dq_zero(d, j);
            const float sc = dq_scale(d, j);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float q = static_cast<float>(static_cast<uint32_t>(v >> (i * d.nbits)) & mask);
                d.out[(m * kPiece + i) * d.cols + c] = float_to_out<OUT_DT>(__fmul_rn(__fsub_rn(q, z), sc));
            }
        }
    }
}

// ------------------------------------------------------- host side -------

struct DevInfo {
    int sms = 0;
    int l2_bytes = 0;
    int coop = 0;        // cooperative launches supported
    int smem_optin = 0;  // largest dynamic shared memory per CTA after opting in
};

DevInfo device_info() {
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!have[dev]) {
        DevInfo d;
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&d.l2_bytes, cudaDevAttrL2CacheSize, dev);
        cudaDeviceGetAttribute(&d.coop, cudaDevAttrCooperativeLaunch, dev);
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (d.sms < 1) d.sms = 1;
        cache[dev] = d;
        have[dev] = true;
    }
    return cache[dev];
}

std::atomic<int> g_tensor_resident{1};

template <typename K>
cudaError_t persistent_grid(K kernel, int threads, size_t smem, int64_t work_units, int* grid) {
    if (smem > 47 * 1024) {  // with the kernel's static shared memory, beyond the default 48 KB
        const cudaError_t e =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t cap = static_cast<int64_t>(device_info().sms) * per_sm;
    if (cap > kMaxPartials) cap = kMaxPartials;
    if (work_units < 1) work_units = 1;
    *grid = static_cast<int>(work_units < cap ? work_units : cap);
    return cudaSuccess;
}

// Evaluations per group-mode pass: short passes first (most groups stop after
// two or three evaluations), longer ones for the tail, then the rest.
int pass_schedule(int iters_eff, int stop_mode, int* m) {
    if (stop_mode != 0 || iters_eff <= 2) {  // no early stop: one pass runs everything
        m[0] = iters_eff;
        return 1;
    }
    static const int sched[] = {2, 3};
    int n = 0, done = 0;
    for (int v : sched) {
        if (done + v >= iters_eff) break;
        m[n++] = v;
        done += v;
    }
    m[n++] = iters_eff - done;
    return n;
}

template <int DT, int AXIS, int E>
cudaError_t launch_group(KParams& k, const WorkspaceLayout& L, uint8_t* ws, cudaStream_t stream) {
    auto kern = solve_group_kernel<DT, AXIS, E>;
    const int64_t n_all = num_entries(k.rows, k.cols, k.G, k.g, AXIS, k.logP);
    const int64_t slice = L.slice < n_all ? L.slice : n_all;
    const int gpw = 32 >> k.logP;
    int grid = 0;
    cudaError_t err = persistent_grid(kern, kRegThreads, 0, ((slice + gpw - 1) / gpw + kRegWarps - 1) / kRegWarps, &grid);
    if (err != cudaSuccess) return err;
    int m[kMaxPasses];
    const int np = pass_schedule(k.iters_eff, k.stop_mode, m);
    uint32_t* const list[2] = {reinterpret_cast<uint32_t*>(ws + L.list0), reinterpret_cast<uint32_t*>(ws + L.list1)};
    for (int64_t e0 = 0; e0 < n_all; e0 += slice) {
        if (e0 > 0) {  // pass counts of the previous slice
            err = cudaMemsetAsync(k.counters + kWordPass, 0, sizeof(uint32_t) * kMaxPasses, stream);
            if (err != cudaSuccess) return err;
        }
        PassArgs pa{};
        pa.state = reinterpret_cast<float4*>(ws + L.state);
        pa.state_it = reinterpret_cast<int*>(ws + L.state_it);
        pa.e0 = e0;
        pa.n = n_all - e0 < slice ? n_all - e0 : slice;
        int k0 = 0;
        for (int q = 0; q < np; ++q) {
            pa.in = q == 0 ? nullptr : list[(q - 1) & 1];
            pa.in_count = q == 0 ? nullptr : k.counters + kWordPass + q - 1;
            pa.out = q + 1 < np ? list[q & 1] : nullptr;
            pa.out_count = k.counters + kWordPass + q;
            pa.k0 = k0;
            pa.evals = m[q];
            kern<<<grid, kRegThreads, 0, stream>>>(k, pa);
            err = cudaGetLastError();
            if (err != cudaSuccess) return err;
            k0 += m[q];
        }
    }
    return cudaSuccess;
}

template <int DT, int E>
cudaError_t launch_group_onepass(KParams& k, cudaStream_t stream) {
    auto kern = solve_group_onepass_kernel<DT, E>;
    const int S = 32 >> k.logP;
    const int64_t nchunks = (k.G + S - 1) / S;
    const size_t smem = sizeof(uint4) * static_cast<size_t>(onepass_warp_uint4(E)) * kRegWarps;
    int grid = 0;
    cudaError_t err = persistent_grid(kern, kRegThreads, smem, (nchunks + kRegWarps - 1) / kRegWarps, &grid);
    if (err != cudaSuccess) return err;
    kern<<<grid, kRegThreads, smem, stream>>>(k, nchunks);
    return cudaGetLastError();
}

// Launch shape of the resident tensor-stop kernel, or false when this problem
// does not take it: the mode allows it (0 never; 1, the default, for tiles of
// 32 elements per lane, g >= 32; 2 for every g); axis 1 and at least one
// iteration; a device with
// cooperative launches; W within half the L2 (so its copies at every
// iteration hit); the per-group state of every warp's tiles within the shared
// memory of the CTAs one SM holds.  Two (32-element tiles) or four CTAs per
// SM, fewer when the state needs more shared memory per CTA.
template <int DT, int E>
bool plan_resident(const KParams& k, int* grid_out, int* T_out, size_t* smem_out) {
    if (!g_tensor_resident.load() || k.axis != 1 || k.iters_eff < 1) return false;
    if (E < 32 && g_tensor_resident.load() != 2) return false;  // measured slower than the chunks below g = 32
                                                                  // (mode 2 takes it wherever it fits)
    const DevInfo d = device_info();
    if (!d.coop || static_cast<double>(k.n) * 2.0 > 0.5 * static_cast<double>(d.l2_bytes)) return false;
    auto kern = solve_tensor_resident_kernel<DT, E>;
    const int gpw = 32 >> k.logP;
    const int64_t ntiles = (k.G + gpw - 1) / gpw;
    static_assert(res_slots(E) <= 2 * (chunk_max(chunk_len(E)) + 1), "the zero-point ring fits the workspace's slots");
    for (int cps = E <= 16 ? 4 : 2; cps >= 2; --cps) {  // at least 16 warps per SM
        int64_t grid = static_cast<int64_t>(d.sms) * cps;
        const int64_t enough = (ntiles + kRegWarps - 1) / kRegWarps;  // a tile per warp
        if (grid > enough) grid = enough;
        const int64_t nw = grid * kRegWarps;
        if (4 * res_c(E) * grid > static_cast<int64_t>(kChunkMax) * kMaxPartials) continue;  // partial rows
        const int64_t T = (ntiles + nw - 1) / nw;
        const size_t smem = res_warp_bytes(E, static_cast<int>(T), gpw) * kRegWarps;
        if (smem + 26 * 1024 > static_cast<size_t>(d.smem_optin)) continue;  // with the kernel's static shared memory
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
            cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRegThreads, smem) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        if (per_sm < cps) continue;
        *grid_out = static_cast<int>(grid);
        *T_out = static_cast<int>(T);
        *smem_out = smem;
        return true;
    }
    return false;
}

template <int DT, int E>
cudaError_t launch_resident(KParams& k, int grid, int T, size_t smem, cudaStream_t stream) {
    unsigned long long limit = kResWaitNs;
    void* args[] = {&k, &T, &limit};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(solve_tensor_resident_kernel<DT, E>), dim3(grid),
                                       dim3(kRegThreads), args, smem, stream);
}

template <int DT, int AXIS, int E>
cudaError_t launch_tensor(KParams& k, cudaStream_t stream) {
    if constexpr (AXIS == 1) {
        int rg = 0, rt = 0;
        size_t rs = 0;
        if (plan_resident<DT, E>(k, &rg, &rt, &rs)) return launch_resident<DT, E>(k, rg, rt, rs, stream);
    }
    const int gpw = 32 >> k.logP;
    const int64_t tiles = AXIS == 1 ? (k.G + gpw - 1) / gpw : (k.rows / k.g) * ((k.cols + gpw - 1) / gpw);
    auto kern = solve_tensor_kernel<DT, AXIS, E>;
    int grid = 0;
    cudaError_t err = persistent_grid(kern, kRegThreads, 0, (tiles + kRegWarps - 1) / kRegWarps, &grid);
    if (err != cudaSuccess) return err;
    const int nch = num_chunks(k.iters_eff, chunk_len(E));
    // axis 1 without debug outputs: the outputs come from a streaming kernel
    const bool stream_out = AXIS == 1 && nch > 0 && !k.dbg_iter && !k.dbg_err && !k.dbg_zero;
    for (int c = 0; c < nch; ++c) {
        kern<<<grid, kRegThreads, 0, stream>>>(k, c, stream_out ? 0 : 1);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    if (!stream_out) {  // the chunk kernel's own output launch
        kern<<<grid, kRegThreads, 0, stream>>>(k, nch, 1);
        return cudaGetLastError();
    }
    const int64_t pieces = k.n / kPiece;
    const int64_t blocks = (pieces + 256 * kOutPieces - 1) / (256 * kOutPieces);
    auto launch_out = [&](auto kernel) {
        int og = 0;
        cudaError_t e = persistent_grid(kernel, 256, 0, blocks, &og);
        if (e != cudaSuccess) return e;
        kernel<<<og, 256, 0, stream>>>(k);
        return cudaGetLastError();
    };
    switch (k.nbits) {
        case 1: return launch_out(tensor_output_kernel<DT, 1>);
        case 2: return launch_out(tensor_output_kernel<DT, 2>);
        case 3: return launch_out(tensor_output_kernel<DT, 3>);
        case 4: return launch_out(tensor_output_kernel<DT, 4>);
        default: return launch_out(tensor_output_kernel<DT, 8>);
    }
}

template <int DT, int AXIS, int E>
cudaError_t launch_solver(KParams& k, const WorkspaceLayout& L, uint8_t* ws, cudaStream_t stream) {
    if (k.stop_mode == 1) return launch_tensor<DT, AXIS, E>(k, stream);
    if (AXIS == 1) return launch_group_onepass<DT, E>(k, stream);
    return launch_group<DT, AXIS, E>(k, L, ws, stream);
}

template <int E>
cudaError_t launch_half(KParams& k, cudaStream_t stream) {
    auto kern = solve_half_kernel<E>;
    int grid = 0;
    const int gpw = 32 >> k.logP;
    const int64_t tiles = (k.G + gpw - 1) / gpw;
    cudaError_t err = persistent_grid(kern, kRegThreads, 0, (tiles + kRegWarps - 1) / kRegWarps, &grid);
    if (err != cudaSuccess) return err;
    kern<<<grid, kRegThreads, 0, stream>>>(k);
    return cudaGetLastError();
}

template <int DT, int AXIS>
cudaError_t launch_solver_e(KParams& k, const WorkspaceLayout& L, uint8_t* ws, cudaStream_t stream) {
    if (k.E == 8) return launch_solver<DT, AXIS, 8>(k, L, ws, stream);
    if (k.E == 16) return launch_solver<DT, AXIS, 16>(k, L, ws, stream);
    return launch_solver<DT, AXIS, 32>(k, L, ws, stream);
}

}  // namespace

// A whole group per lane up to g = 32 (E = g, P = 1): every lane has E
// independent elements per evaluation and the group sums need no shuffles;
// larger groups spread over P = g/32 lanes.
Geometry make_geometry(int g) {
    Geometry geo;
    geo.g = g;
    geo.E = g < 32 ? g : 32;
    geo.P = g / geo.E;
    geo.logP = 0;
    while ((1 << geo.logP) < geo.P) ++geo.logP;
    return geo;
}

int64_t group_entries(int64_t rows, int64_t cols, int g, int axis) {
    return num_entries(rows, cols, rows * cols / g, g, axis, make_geometry(g).logP);
}

WorkspaceLayout workspace_layout(int64_t rows, int64_t cols, int g, int axis, int stop_mode, int zero_nbits,
                                 int64_t slice) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const int64_t G = rows * cols / g;
    const size_t Gs = static_cast<size_t>(G > 0 ? G : 0);
    WorkspaceLayout l{};
    size_t off = 0;
    l.header = off;
    off += 256;
    l.zbest = off;
    if (zero_nbits == 8) off = up(off + 4 * Gs);
    l.state = l.state_it = l.list0 = l.list1 = off;
    l.tparts = l.etot = l.t_s = l.t_z0 = l.t_sws = l.t_zs = off;
    if (stop_mode == 1) {
        l.tparts = off;
        off = up(off + sizeof(double) * kChunkMax * kMaxPartials);
        l.etot = off;
        off = up(off + sizeof(double) * kMaxIters);
        l.t_s = off;
        off = up(off + 4 * Gs);
        l.t_z0 = off;
        off = up(off + 4 * Gs);
        l.t_sws = off;
        off = up(off + 8 * Gs);
        l.t_zs = off;  // z of every iteration of two chunks
        const size_t slots = static_cast<size_t>(chunk_max(chunk_len(g < 32 ? g : 32)) + 1);
        off = up(off + 4 * 2 * slots * Gs);
    } else if (axis == 1) {
        l.slice = group_entries(rows, cols, g, axis);  // one pass over every group: no per-group state
    } else {
        const int64_t n = group_entries(rows, cols, g, axis);
        constexpr int64_t kMaxSlice = int64_t{1} << 31;  // survivor lists hold 32-bit entry offsets
        l.slice = (slice > 0 && slice < n) ? slice : n;
        if (l.slice > kMaxSlice) l.slice = kMaxSlice;
        const size_t S = static_cast<size_t>(l.slice > 0 ? l.slice : 0);
        l.state = off;
        off = up(off + 32 * S);
        l.state_it = off;
        off = up(off + 4 * S);
        l.list0 = off;
        off = up(off + 4 * S);
        l.list1 = off;
        off = up(off + 4 * S);
    }
    l.total = off;
    return l;
}

int64_t fit_slice(int64_t rows, int64_t cols, int g, int axis, int stop_mode, int zero_nbits, size_t bytes) {
    const WorkspaceLayout full = workspace_layout(rows, cols, g, axis, stop_mode, zero_nbits, 0);
    if (full.total <= bytes) return full.slice > 0 ? full.slice : 1;
    if (stop_mode == 1 || axis == 1) return 0;  // nothing to cut into slices
    const WorkspaceLayout base = workspace_layout(rows, cols, g, axis, stop_mode, zero_nbits, 1);
    const size_t fixed = base.state;  // header and kept zeros
    const size_t per = 44;            // bytes per entry of a slice, before each part's rounding to 256
    if (bytes < fixed) return 0;
    // the largest multiple of 32 entries whose parts, each rounded up to 256 bytes, fit
    int64_t s = static_cast<int64_t>((bytes - fixed) / per) & ~static_cast<int64_t>(31);
    while (s >= kMinSlice && workspace_layout(rows, cols, g, axis, stop_mode, zero_nbits, s).total > bytes) s -= 32;
    return s >= kMinSlice ? s : 0;
}

cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream) {
    const Geometry geo = make_geometry(a.g);
    const WorkspaceLayout L = workspace_layout(a.rows, a.cols, a.g, a.axis, a.stop_mode, a.zero_nbits, a.slice);
    KParams k{};
    k.W = static_cast<const uint16_t*>(a.W);
    k.rows = a.rows;
    k.cols = a.cols;
    k.G = a.G;
    k.n = a.rows * a.cols;
    k.g = a.g;
    k.E = geo.E;
    k.P = geo.P;
    k.logP = geo.logP;
    k.nbits = a.nbits;
    k.iters = a.iters;
    k.iters_eff = a.iters > 0 ? a.iters : (a.dbg_err ? 1 : 0);  // iters 0 == 1: z* = z0 either way
    k.stop_mode = a.stop_mode;
    k.zero_nbits = a.zero_nbits;
    k.axis = a.axis;
    k.p = a.p;
    k.beta = a.beta;
    k.kappa = a.kappa;
    float bl = a.beta;
    for (int i = 1; i < k.iters_eff; ++i) bl *= a.kappa;  // the same sequential fp32 products as the device
    k.beta_last = bl;
    k.Lf = static_cast<float>((1 << a.nbits) - 1);
    k.packed = a.packed;
    k.scale = a.scale;
    k.zero = a.zero;
    k.dbg_iter = a.dbg_iter;
    k.dbg_err = a.dbg_err;
    k.dbg_zero = a.dbg_zero;
    k.counters = reinterpret_cast<uint32_t*>(a.ws + L.header);
    k.zbest_ws = a.zero_nbits == 8 ? reinterpret_cast<float*>(a.ws + L.zbest) : nullptr;
    if (a.stop_mode == 1) {
        k.tparts = reinterpret_cast<double*>(a.ws + L.tparts);
        k.etot = reinterpret_cast<double*>(a.ws + L.etot);
        k.t_s = reinterpret_cast<float*>(a.ws + L.t_s);
        k.t_z0 = reinterpret_cast<float*>(a.ws + L.t_z0);
        k.t_sws = reinterpret_cast<double*>(a.ws + L.t_sws);
        k.t_zs = reinterpret_cast<float*>(a.ws + L.t_zs);
    }

    cudaError_t err = cudaMemsetAsync(a.ws + L.header, 0, 256, stream);
    if (err != cudaSuccess) return err;
    if (a.G > 0 && a.half) {  // the half-precision variant: fp16 input, axis 1, group or no stop
        if (k.E == 8) err = launch_half<8>(k, stream);
        else if (k.E == 16) err = launch_half<16>(k, stream);
        else err = launch_half<32>(k, stream);
        if (err != cudaSuccess) return err;
    } else if (a.G > 0) {
        if (a.dtype == 0 && a.axis == 1) err = launch_solver_e<0, 1>(k, L, a.ws, stream);
        else if (a.dtype == 0) err = launch_solver_e<0, 0>(k, L, a.ws, stream);
        else if (a.axis == 1) err = launch_solver_e<1, 1>(k, L, a.ws, stream);
        else err = launch_solver_e<1, 0>(k, L, a.ws, stream);
        if (err != cudaSuccess) return err;
    }
    if (a.zero_nbits == 8) {
        int64_t blocks = (a.G + 255) / 256;
        const int64_t cap = static_cast<int64_t>(device_info().sms) * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        zero_q8_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(k.zbest_ws, a.G, k.counters,
                                                                    static_cast<uint8_t*>(a.zero), a.zero_meta);
        err = cudaGetLastError();
    }
    return err;
}

void set_tensor_resident(int mode) { g_tensor_resident.store(mode < 0 ? 0 : (mode > 2 ? 2 : mode)); }
int tensor_resident() { return g_tensor_resident.load(); }

bool tensor_uses_resident(int64_t rows, int64_t cols, int dtype, int g, int axis, int iters) {
    if (axis != 1 || iters < 1 || rows * cols <= 0) return false;
    const Geometry geo = make_geometry(g);
    KParams k{};
    k.rows = rows;
    k.cols = cols;
    k.n = rows * cols;
    k.G = k.n / g;
    k.g = g;
    k.E = geo.E;
    k.P = geo.P;
    k.logP = geo.logP;
    k.axis = axis;
    k.iters_eff = iters;
    int grid = 0, T = 0;
    size_t smem = 0;
    auto plan = [&](auto dt) {
        constexpr int DT = decltype(dt)::value;
        if (k.E == 8) return plan_resident<DT, 8>(k, &grid, &T, &smem);
        if (k.E == 16) return plan_resident<DT, 16>(k, &grid, &T, &smem);
        return plan_resident<DT, 32>(k, &grid, &T, &smem);
    };
    return dtype == 0 ? plan(std::integral_constant<int, 0>{}) : plan(std::integral_constant<int, 1>{});
}

cudaError_t launch_tensor_wait_selftest(uint8_t* ws, unsigned long long limit_ns, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(ws, 0, 256, stream);
    if (err != cudaSuccess) return err;
    KParams k{};
    k.counters = reinterpret_cast<uint32_t*>(ws);
    res_wait_selftest_kernel<<<1, 32, 0, stream>>>(k, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_scale8(const uint16_t* scale, int64_t G, int S, uint8_t* codes, float* meta,
                          cudaStream_t stream) {
    const int64_t runs = (G + S - 1) / S;
    if (runs == 0) return cudaSuccess;
    const bool vec = S == 128 && (reinterpret_cast<uintptr_t>(scale) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
    const int64_t warps = vec ? (runs + 3) / 4 : runs;
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = static_cast<int64_t>(device_info().sms) * 64;
    if (blocks > cap) blocks = cap;
    if (vec) scale8_kernel_128<<<static_cast<int>(blocks), 256, 0, stream>>>(scale, G, codes, meta);
    else scale8_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(scale, G, S, codes, meta);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream) {
    DqParams d;
    d.packed = a.packed;
    d.scale = a.scale;
    d.scale_q = a.scale_q;
    d.scale_meta = a.scale_meta;
    d.scale_group = a.scale_group;
    d.zero = a.zero;
    d.meta = a.zero_meta;
    d.rows = a.rows;
    d.cols = a.cols;
    d.nbits = a.nbits;
    d.g = a.g;
    d.zero_nbits = a.zero_nbits;
    d.out = static_cast<uint16_t*>(a.out);
    const int64_t units = a.rows * a.cols / kPiece;
    if (units == 0) return cudaSuccess;
    int64_t blocks = (units + 255) / 256;
    const int64_t cap = static_cast<int64_t>(device_info().sms) * 16;
    if (blocks > cap) blocks = cap;
    const int nb = static_cast<int>(blocks);
    if (a.out_dtype == 0 && a.axis == 1) dequant_kernel<0, 1><<<nb, 256, 0, stream>>>(d);
    else if (a.out_dtype == 0) dequant_kernel<0, 0><<<nb, 256, 0, stream>>>(d);
    else if (a.axis == 1) dequant_kernel<1, 1><<<nb, 256, 0, stream>>>(d);
    else dequant_kernel<1, 0><<<nb, 256, 0, stream>>>(d);
    return cudaGetLastError();
}

}  // namespace hqq
