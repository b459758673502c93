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
// iteration costs ~8 FP32-pipe instructions and two MUFU ops (|r|^p through
// lg2/ex2), so the MUFU pipe, not HBM, bounds the solver.
//
// solve_pool_kernel (group / no stop, axis 1): every warp owns a pool of
//   "cells" in shared memory, one group each.  Per round it (A) packs and
//   stores the groups that finished, (B) refills free cells with the next
//   groups of a global work counter by cp.async (16-byte copies straight into
//   shared memory), (C) waits for the copies issued one round earlier,
//   (D) initialises those groups (min/max -> s, z0; w*s stored as fp32; sum
//   of w*s in fp64) and (E) evaluates every active group once, mapping each
//   onto P = g/E consecutive lanes after a ballot compaction.  Early-stopped
//   groups free their lanes at once; warps never wait on each other.
// solve_reg_kernel: a warp holds 32/P whole groups in registers.
//   MODE_LOCAL (group / no stop, any axis): iterates until every group of the
//   warp tile has stopped (used for axis 0).
//   MODE_TENSOR: runs iterations [k0, k1) of every group, accumulates the
//   per-iteration tensor error in fp64 per CTA, and the last CTA to finish
//   (atomic ticket) sums the partials in a fixed order.  The next launch
//   reads those sums, applies the stop rule, and either runs the next chunk
//   or writes the final codes with the kept iterate (recomputed from the
//   stored chunk-start zero with the cheap part of the iteration).  No CTA
//   ever waits for another.

#include "hqq_device.cuh"

namespace hqq {

namespace {

using namespace dev;

constexpr int kPoolWarps = 4;
constexpr int kPoolThreads = kPoolWarps * 32;
constexpr int kRegThreads = 256;
constexpr int kRegWarps = kRegThreads / 32;
constexpr int kChunkMax = 4;  // iterations per tensor-mode launch (after the first, which has 2)

enum : uint8_t { kEmpty = 0, kLoading = 1, kActive = 2, kDone = 3 };

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

// Block-wide min/max of the kept zeros -> one partial per CTA.
template <int NW>
__device__ __forceinline__ void write_minmax(const KParams& k, float zmin, float zmax, float2* sred) {
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
        k.minmax[blockIdx.x] = r;
    }
}

// ============================================================ pool kernel ==

// Per-warp pool layout (NC cells).  A cell holds one group: CS = g + 4 floats
// (the 16-byte pad staggers consecutive cells across shared-memory banks).
// Before initialisation the raw 16-bit group is staged in the top 2g bytes of
// the cell by cp.async; initialisation overwrites the cell with fp32 w*s.
struct Pool {
    float* data;
    float4* zs4;  // (z, s, z0, flags): what every lane of a group reads per evaluation
    float2* sws;  // sum of w*s as a float pair (hi, lo)
    int64_t* gidx;
    float *be, *zb, *beta, *wsmax;
    int *kk, *bi, *issued;
    uint8_t *st, *list;
};

__host__ __device__ inline int pool_cell_floats(int g) { return g + 4; }

__host__ __device__ inline int pool_warp_bytes(int NC, int g) {
    const int b = NC * (4 * pool_cell_floats(g) + 16 + 8 + 8 + 4 * 4 + 3 * 4 + 2);
    return (b + 15) & ~15;
}

__device__ __forceinline__ Pool carve_pool(unsigned char* base, int NC, int g) {
    Pool m;
    size_t off = 0;
    m.data = reinterpret_cast<float*>(base + off);
    off += static_cast<size_t>(NC) * pool_cell_floats(g) * 4;
    m.zs4 = reinterpret_cast<float4*>(base + off);
    off += NC * 16;
    m.sws = reinterpret_cast<float2*>(base + off);
    off += NC * 8;
    m.gidx = reinterpret_cast<int64_t*>(base + off);
    off += NC * 8;
    float* f = reinterpret_cast<float*>(base + off);
    m.be = f;
    m.zb = f + NC;
    m.beta = f + 2 * NC;
    m.wsmax = f + 3 * NC;
    off += NC * 4 * 4;
    int* iv = reinterpret_cast<int*>(base + off);
    m.kk = iv;
    m.bi = iv + NC;
    m.issued = iv + 2 * NC;
    off += NC * 3 * 4;
    m.st = base + off;
    m.list = base + off + NC;
    return m;
}

// Ordered list of the cells whose predicate holds (a: cell lane, b: cell lane+32).
__device__ __forceinline__ int make_list(bool a, bool b, uint8_t* list) {
    const int lane = threadIdx.x & 31;
    const unsigned lo = __ballot_sync(kFull, a), hi = __ballot_sync(kFull, b);
    const unsigned below = (1u << lane) - 1u;
    const int nlo = __popc(lo);
    if (a) list[__popc(lo & below)] = static_cast<uint8_t>(lane);
    if (b) list[nlo + __popc(hi & below)] = static_cast<uint8_t>(lane + 32);
    __syncwarp();
    return nlo + __popc(hi);
}

__device__ __forceinline__ float* cell_ptr(const Pool& m, int c, int g) {
    return m.data + static_cast<size_t>(c) * pool_cell_floats(g);
}

// The 8 fp32 values of piece pc of cell c.
__device__ __forceinline__ void load_ws8(const float* cell, int pc, float* ws) {
    const float4* p = reinterpret_cast<const float4*>(cell + pc * kPiece);
    const float4 a = p[0], b = p[1];
    ws[0] = a.x;
    ws[1] = a.y;
    ws[2] = a.z;
    ws[3] = a.w;
    ws[4] = b.x;
    ws[5] = b.y;
    ws[6] = b.z;
    ws[7] = b.w;
}

// Eight codes, LSB first, NBITS each (32-bit arithmetic when they fit).
template <int NBITS>
__device__ __forceinline__ void store_piece_t(uint8_t* dst, const uint32_t* c) {
    if (NBITS == 8) {
        uint2 v;
        v.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
        v.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
        *reinterpret_cast<uint2*>(dst) = v;
    } else {
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) v |= c[i] << (i * NBITS);
        if (NBITS == 4) *reinterpret_cast<uint32_t*>(dst) = v;
        else if (NBITS == 2) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(v);
        else if (NBITS == 1) *dst = static_cast<uint8_t>(v);
        else {
            dst[0] = static_cast<uint8_t>(v);
            dst[1] = static_cast<uint8_t>(v >> 8);
            dst[2] = static_cast<uint8_t>(v >> 16);
        }
    }
}

constexpr unsigned kFlagShrink = 1u;  // the proximal step may be non-zero
constexpr unsigned kFlagClamp = 2u;   // some v may leave [-0.5, L + 0.5)

// Flags of the next evaluation of a group at zero-point z (v = fl(ws + z) with
// ws in [-z0, wsmax]: fl(min w * s) = -z0 exactly).
__device__ __forceinline__ float eval_flags(float s, float z, float z0, float wsmax, float thr, float Lf) {
    unsigned f = 0;
    if (shrink_possible(s, z, z0, thr, Lf)) f |= kFlagShrink;
    if (!clamp_free(-z0, wsmax, z, Lf)) f |= kFlagClamp;
    return __uint_as_float(f);
}

// Group-level decision after evaluating zero-point z (one lane per group):
// keep the best iterate, apply the stop rule, compute the next zero-point and
// the flags of its evaluation.
__device__ __forceinline__ void decide(const KParams& k, const Pool& m, int c, bool stop_group, float err, float sq,
                                       bool sp, double swe, float z, float s, float z0, float beta, int kk) {
    const bool improved = err < m.be[c];
    if (improved) {
        m.be[c] = err;
        m.zb[c] = z;
        m.bi[c] = kk;
    }
    bool stop = (stop_group && !improved) || kk >= k.iters_eff - 1;
    if (!stop) {
        const float2 f = m.sws[c];
        const float zn = sp ? zero_from_sums(sq, swe, k.g)
                            : zero_from_sums_f2(sq, F2{f.x, f.y}, 1.0f / static_cast<float>(k.g));
        if (stop_group && zn == z) {
            stop = true;  // fixed point: the next error would equal this one
        } else {
            const float nbeta = __fmul_rn(beta, k.kappa);
            m.zs4[c] = make_float4(zn, s, z0, eval_flags(s, zn, z0, m.wsmax[c], shrink_threshold(nbeta, k.p), k.Lf));
            m.kk[c] = kk + 1;
            m.beta[c] = nbeta;
        }
    }
    m.st[c] = stop ? kDone : kActive;
}

template <int DT, int E, int NBITS>
__global__ void __launch_bounds__(kPoolThreads, 6) solve_pool_kernel(const KParams k) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ float2 sred[kPoolWarps];
    constexpr int NPL = E / kPiece;  // pieces per lane
    constexpr float Lf = static_cast<float>((1 << NBITS) - 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NC = k.NC, g = k.g, P = k.P, logP = k.logP;
    const int ppg = g / kPiece;  // pieces (16-byte raw copies) per group
    const Pool m = carve_pool(smem_raw + static_cast<size_t>(warp) * k.pool_warp_bytes, NC, g);
    const bool stop_group = k.stop_mode == 0;
    const float thr0 = shrink_threshold(k.beta, k.p);
    unsigned long long* work = reinterpret_cast<unsigned long long*>(k.counters + 2);
    float zmin = FLT_MAX, zmax = -FLT_MAX;
    int64_t qn = 0, qe = 0;
    bool exhausted = false;

    if (lane < NC) m.st[lane] = kEmpty;
    if (lane + 32 < NC) m.st[lane + 32] = kEmpty;
    __syncwarp();

    for (int round = 0;; ++round) {
        // (A) pack and store the groups that finished
        {
            const bool a = lane < NC && m.st[lane] == kDone;
            const bool b = lane + 32 < NC && m.st[lane + 32] == kDone;
            const int items = make_list(a, b, m.list) << logP;
            for (int it = lane; it < items; it += 32) {
                const int c = m.list[it >> logP], part = it & (P - 1);
                const int64_t j = m.gidx[c];
                const float zb = m.zb[c];
                const float* cell = cell_ptr(m, c, g);
#pragma unroll
                for (int t = 0; t < NPL; ++t) {
                    const int pc = part + t * P;
                    float ws[8];
                    uint32_t code[8];
                    load_ws8(cell, pc, ws);
#pragma unroll
                    for (int i = 0; i < 8; ++i) round_clamp(__fadd_rn(ws[i], zb), Lf, &code[i]);
                    store_piece_t<NBITS>(k.packed + (j * ppg + pc) * NBITS, code);
                }
                if (part == 0) {
                    const float s = m.zs4[c].y;
                    const float err = m.be[c] * pow_pos(s, -k.p) / static_cast<float>(g);
                    store_group(k, j, s, zb, m.bi[c], err, &zmin, &zmax);
                }
            }
            __syncwarp();
            if (a) m.st[lane] = kEmpty;
            if (b) m.st[lane + 32] = kEmpty;
            __syncwarp();
        }
        // (B) refill free cells from the work counter and start their copies
        {
            const bool a = lane < NC && m.st[lane] == kEmpty;
            const bool b = lane + 32 < NC && m.st[lane + 32] == kEmpty;
            const unsigned lo = __ballot_sync(kFull, a), hi = __ballot_sync(kFull, b);
            const int nf = __popc(lo) + __popc(hi);
            const int avail = static_cast<int>(qe - qn);
            int64_t q2 = 0;
            int avail2 = 0;
            if (nf > avail && !exhausted) {
                unsigned long long base = 0;
                if (lane == 0) base = atomicAdd(work, static_cast<unsigned long long>(NC));
                base = __shfl_sync(kFull, base, 0);
                if (static_cast<int64_t>(base) >= k.G) {
                    exhausted = true;
                } else {
                    q2 = static_cast<int64_t>(base);
                    const int64_t left = k.G - q2;
                    avail2 = left < NC ? static_cast<int>(left) : NC;
                }
            }
            const unsigned below = (1u << lane) - 1u;
            const int ra = __popc(lo & below), rb = __popc(lo) + __popc(hi & below);
            bool la = false, lb = false;
            if (a && ra < avail + avail2) {
                m.gidx[lane] = ra < avail ? qn + ra : q2 + (ra - avail);
                m.st[lane] = kLoading;
                m.issued[lane] = round;
                la = true;
            }
            if (b && rb < avail + avail2) {
                m.gidx[lane + 32] = rb < avail ? qn + rb : q2 + (rb - avail);
                m.st[lane + 32] = kLoading;
                m.issued[lane + 32] = round;
                lb = true;
            }
            const int used = nf < avail + avail2 ? nf : avail + avail2;
            if (used <= avail) {
                qn += used;
            } else {
                qn = q2 + (used - avail);
                qe = q2 + avail2;
            }
            const int copies = make_list(la, lb, m.list) * ppg;
            for (int it = lane; it < copies; it += 32) {
                const int c = m.list[it / ppg], pc = it % ppg;
                const uint16_t* src = k.W + m.gidx[c] * g + pc * kPiece;
                unsigned char* dst = reinterpret_cast<unsigned char*>(cell_ptr(m, c, g)) + 2 * g + 16 + pc * 16;
                cp_async16(dst, src);
            }
        }
        cp_async_commit();
        // (C) copies issued one round earlier have landed
        cp_async_wait_prev();
        __syncwarp();
        // (D) initialise those groups and evaluate their first zero-point z0
        {
            const bool a = lane < NC && m.st[lane] == kLoading && m.issued[lane] < round;
            const bool b = lane + 32 < NC && m.st[lane + 32] == kLoading && m.issued[lane + 32] < round;
            const int items = make_list(a, b, m.list) << logP;
            for (int base = 0; base < items; base += 32) {
                const int it = base + lane;
                const bool valid = it < items;
                const int c = valid ? m.list[it >> logP] : 0;
                const int part = it & (P - 1);
                float* cell = cell_ptr(m, c, g);
                const unsigned char* stage = reinterpret_cast<const unsigned char*>(cell) + 2 * g + 16;
                float w[E];
                float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
                for (int i = 0; i < E; ++i) w[i] = 0.0f;
                if (valid) {
#pragma unroll
                    for (int t = 0; t < NPL; ++t)
                        unpack8<DT>(*reinterpret_cast<const uint4*>(stage + (part + t * P) * 16), w + t * kPiece);
#pragma unroll
                    for (int i = 0; i < E; ++i) {
                        mn = fminf(mn, w[i]);
                        mx = fmaxf(mx, w[i]);
                    }
                }
                mn = seg_min(mn, P);
                mx = seg_max(mx, P);
                float s = kScaleCap;
                if (mx > mn) s = fminf(__fdiv_rn(Lf, __fsub_rn(mx, mn)), kScaleCap);
                const float z0 = __fmul_rn(-mn, s);
                float hi = 0.0f, lo = 0.0f;
                float ws[E];
                float err = 0.0f, sq = 0.0f;
#pragma unroll
                for (int i = 0; i < E; ++i) {
                    ws[i] = __fmul_rn(w[i], s);
                    two_sum_acc(hi, lo, ws[i]);
                    // at z0 every v lies in [0, L]: fl(min w * s) + z0 = 0, fl(max w * s) + z0 <= L
                    const ElemEval ee = eval_elem_nc(ws[i], z0);
                    err += pow_pos(fabsf(ee.r), k.p);
                    sq += ee.q;
                }
                double acc = static_cast<double>(hi) + static_cast<double>(lo);
                if (!valid) err = sq = 0.0f, acc = 0.0;
                acc = seg_sum_d(acc, P);
                err = seg_sum(err, P);
                sq = seg_sum(sq, P);
                const bool sp = valid && k.iters_eff > 1 && shrink_possible(s, z0, z0, thr0, Lf);
                double swe = 0.0;
                if (__any_sync(kFull, sp)) {  // rare: re-read the staged raw values (still intact here)
                    if (sp) {
#pragma unroll
                        for (int t = 0; t < NPL; ++t) {
                            float x[8];
                            unpack8<DT>(*reinterpret_cast<const uint4*>(stage + (part + t * P) * 16), x);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const ElemEval ee = eval_elem(ws[t * 8 + i], z0, Lf);
                                const float we = shrink_elem(ee.r, s, k.p, k.beta);
                                swe += static_cast<double>(__fmul_rn(__fsub_rn(x[i], we), s));
                            }
                        }
                    }
                    swe = seg_sum_d(swe, P);
                }
                __syncwarp();  // every lane has read its raw data before any fp32 write below
                if (valid) {
#pragma unroll
                    for (int t = 0; t < NPL; ++t) {
                        float4* dst = reinterpret_cast<float4*>(cell + (part + t * P) * kPiece);
                        dst[0] = make_float4(ws[t * 8 + 0], ws[t * 8 + 1], ws[t * 8 + 2], ws[t * 8 + 3]);
                        dst[1] = make_float4(ws[t * 8 + 4], ws[t * 8 + 5], ws[t * 8 + 6], ws[t * 8 + 7]);
                    }
                    if (part == 0) {
                        const F2 f = split_f2(acc);
                        m.sws[c] = make_float2(f.hi, f.lo);
                        m.zb[c] = z0;
                        m.bi[c] = 0;
                        m.wsmax[c] = __fmul_rn(mx, s);
                        m.zs4[c] = make_float4(z0, s, z0, 0.0f);
                        if (k.iters_eff == 0) {
                            m.be[c] = INFINITY;
                            m.st[c] = kDone;
                        } else {
                            m.be[c] = INFINITY;
                            decide(k, m, c, stop_group, err, sq, sp, swe, z0, s, z0, k.beta, 0);
                        }
                    }
                }
                __syncwarp();
            }
        }
        // (E) one evaluation of every active group
        {
            const bool a = lane < NC && m.st[lane] == kActive;
            const bool b = lane + 32 < NC && m.st[lane + 32] == kActive;
            const int items = make_list(a, b, m.list) << logP;
            for (int base = 0; base < items; base += 32) {
                const int it = base + lane;
                const bool valid = it < items;
                const int c = valid ? m.list[it >> logP] : 0;
                const int part = it & (P - 1);
                const float4 st4 = m.zs4[c];
                const float z = st4.x, s = st4.y, z0 = st4.z;
                const unsigned flags = valid ? __float_as_uint(st4.w) : 0u;
                const bool sp = (flags & kFlagShrink) != 0;
                const float* cell = cell_ptr(m, c, g);
                float err = 0.0f, sq = 0.0f;
                if (__all_sync(kFull, (flags & kFlagClamp) == 0)) {
                    if (valid) {
#pragma unroll
                        for (int t = 0; t < NPL; ++t) {
                            float ws[8];
                            load_ws8(cell, part + t * P, ws);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const ElemEval ee = eval_elem_nc(ws[i], z);
                                err += pow_pos(fabsf(ee.r), k.p);
                                sq += ee.q;
                            }
                        }
                    }
                } else if (valid) {
#pragma unroll
                    for (int t = 0; t < NPL; ++t) {
                        float ws[8];
                        load_ws8(cell, part + t * P, ws);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const ElemEval ee = eval_elem(ws[i], z, Lf);
                            err += pow_pos(fabsf(ee.r), k.p);
                            sq += ee.q;
                        }
                    }
                }
                err = seg_sum(err, P);
                sq = seg_sum(sq, P);
                double swe = 0.0;
                float beta = 0.0f;
                if (__any_sync(kFull, sp)) {  // rare: the proximal step may be non-zero
                    beta = m.beta[c];
                    if (sp) {
                        const int64_t j = m.gidx[c];
#pragma unroll
                        for (int t = 0; t < NPL; ++t) {
                            const int pc = part + t * P;
                            float ws[8], w[8];
                            load_ws8(cell, pc, ws);
                            unpack8<DT>(__ldg(reinterpret_cast<const uint4*>(k.W + j * g + pc * kPiece)), w);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const ElemEval ee = eval_elem(ws[i], z, Lf);
                                const float we = shrink_elem(ee.r, s, k.p, beta);
                                swe += static_cast<double>(__fmul_rn(__fsub_rn(w[i], we), s));
                            }
                        }
                    }
                    swe = seg_sum_d(swe, P);
                }
                if (valid && part == 0) decide(k, m, c, stop_group, err, sq, sp, swe, z, s, z0, m.beta[c], m.kk[c]);
            }
            __syncwarp();
        }
        const bool live = (lane < NC && m.st[lane] != kEmpty) || (lane + 32 < NC && m.st[lane + 32] != kEmpty);
        if (exhausted && !__any_sync(kFull, live)) break;
    }
    cp_async_wait_all();
    if (k.zero_nbits == 8) write_minmax<kPoolWarps>(k, zmin, zmax, sred);
}

// ======================================================== register kernel ==

constexpr int MODE_LOCAL = 0;
constexpr int MODE_TENSOR = 1;

// Chunk schedule of tensor mode: chunk 0 = iterations [0, 2), chunk c >= 1 =
// [4c - 2, 4c + 2) (clipped to iters).
__host__ __device__ inline int chunk_begin(int c, int iters) {
    const int b = c == 0 ? 0 : 4 * c - 2;
    return b < iters ? b : iters;
}
__host__ __device__ inline int chunk_of(int k) { return k < 2 ? 0 : (k + 2) / 4; }
__host__ __device__ inline int num_chunks(int iters) { return iters <= 0 ? 0 : chunk_of(iters - 1) + 1; }

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

// Packed codes of this lane's E elements with zero-point z.
template <int AXIS, int E>
__device__ __forceinline__ void store_lane_codes(const KParams& k, const WarpTile& w, const float* ws, float z) {
    if (!w.valid) return;
#pragma unroll
    for (int t = 0; t < E / kPiece; ++t) {
        uint32_t code[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) code[i] = eval_elem(ws[t * 8 + i], z, k.Lf).code;
        const uint64_t v = pack8(code, k.nbits);
        const int pc = (w.part * E) / kPiece + t;  // piece index within the group
        if (AXIS == 1) {
            store_piece(k.packed + (w.j * (k.g / kPiece) + pc) * k.nbits, v, k.nbits);
        } else {
            const int64_t rb = w.j / k.cols, c = w.j % k.cols;
            uint8_t* dst =
                k.packed + ((rb * k.g) / kPiece * k.nbits + static_cast<int64_t>(pc) * k.nbits) * k.cols + c;
            for (int b = 0; b < k.nbits; ++b) dst[b * k.cols] = static_cast<uint8_t>(v >> (8 * b));
        }
    }
}

// min/max -> s, z0; fp32 w*s; fp64 sum of w*s (over the group's P lanes).
// Also returns this lane's range of w*s (for the clamp-free test).
template <int E>
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
    float hi = 0.0f, lo = 0.0f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
        ws[i] = __fmul_rn(x[i], s);
        two_sum_acc(hi, lo, ws[i]);
    }
    const double acc = w.valid ? static_cast<double>(hi) + static_cast<double>(lo) : 0.0;
    *s_out = s;
    *z0_out = __fmul_rn(-mn, s);
    *sws_out = seg_sum_d(acc, k.P);
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
    float x[E];
    load_lane<DT, AXIS, E>(k, w, x);
    float err = 0.0f, sq = 0.0f;
    double swe = 0.0;
    const float beta = beta_at(k, it);
#pragma unroll 4
    for (int i = 0; i < E; ++i) {
        const ElemEval ee = eval_elem(__fmul_rn(x[i], s), z, k.Lf);
        err += pow_pos(fabsf(ee.r), k.p);
        sq += ee.q;
        if (sp) {
            const float we = shrink_elem(ee.r, s, k.p, beta);
            swe += static_cast<double>(__fmul_rn(__fsub_rn(x[i], we), s));
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
        if (w.valid) {
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const ElemEval e = eval_elem_nc(ws[i], z);
                err += pow_pos(fabsf(e.r), k.p);
                sq += e.q;
            }
        }
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

// The cheap part of one iteration (no |r|^p): the next zero-point.
template <int E>
__device__ __forceinline__ float step_lane(const KParams& k, bool valid, const float* x, const float* ws, float s,
                                           float z, float z0, float beta, float thr, double sws) {
    float sq = 0.0f;
    const bool sp = valid && shrink_possible(s, z, z0, thr, k.Lf);
    if (valid) {
#pragma unroll
        for (int i = 0; i < E; ++i) sq += eval_elem(ws[i], z, k.Lf).q;
    }
    sq = seg_sum(sq, k.P);
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
    return sp ? zero_from_sums(sq, swe, k.g) : zero_from_sums_f2(sq, split_f2(sws), 1.0f / static_cast<float>(k.g));
}

// One tensor-mode iteration of a warp tile: evaluate z, add this group's
// error term to its per-thread partial, step z.
template <int DT, int AXIS, int E>
__device__ __forceinline__ void tensor_iteration(const KParams& k, const WarpTile& w, const float* ws, float lmin,
                                                 float lmax, float s, float z0, int it, float thr, float spow,
                                                 F2 sws2, float inv_g, double& acc, float& z) {
    float err, sq;
    bool sp;
    double swe;
    eval_lane_reload<DT, AXIS, E>(k, w, ws, lmin, lmax, s, z, z0, it, thr, &err, &sq, &sp, &swe);
    if (w.valid && w.part == 0) acc += static_cast<double>(err * spow);
    z = sp ? zero_from_sums(sq, swe, k.g) : zero_from_sums_f2(sq, sws2, inv_g);
}

__device__ __forceinline__ double warp_sum_d(double x) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}

template <int DT, int AXIS, int E, int MODE>
__global__ void __launch_bounds__(kRegThreads, (MODE == 1 && E <= 16) ? 3 : 2)
    solve_reg_kernel(const KParams k, int chunk) {
    __shared__ float2 sred[kRegWarps];
    __shared__ double sacc[kChunkMax][kRegThreads];  // per-thread tensor error partials
    __shared__ float sthr[kChunkMax];                 // shrink threshold of each iteration of the chunk
    __shared__ int sflag;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t ntiles = num_warp_tiles<AXIS>(k);
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * kRegWarps;
    const int64_t G = k.G;
    const float inv_g = 1.0f / static_cast<float>(k.g);
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    if (MODE == MODE_LOCAL) {
        const bool stop_group = k.stop_mode == 0;
        for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp; t < ntiles; t += wstride) {
            const WarpTile w = warp_tile<AXIS>(k, t);
            float x[E], ws[E];
            load_lane<DT, AXIS, E>(k, w, x);
            float s, z0, lmin, lmax;
            double sws;
            init_lane<E>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
            const F2 sws2 = split_f2(sws);
            float z = z0, zb = z0, be = INFINITY, beta = k.beta;
            int bi = 0;
            bool active = w.valid && k.iters_eff > 0;
            for (int it = 0; it < k.iters_eff && __any_sync(kFull, active); ++it) {
                const float thr = shrink_threshold(beta, k.p);
                float err, sq;
                bool sp;
                double swe;
                eval_lane<E>(k, active, x, ws, s, z, z0, beta, thr, &err, &sq, &sp, &swe);
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
                        if (stop_group && zn == z) stop = true;
                        else z = zn;
                    }
                    if (stop) active = false;
                }
                beta = __fmul_rn(beta, k.kappa);
            }
            store_lane_codes<AXIS, E>(k, w, ws, zb);
            if (w.valid && w.part == 0)
                store_group(k, w.j, s, zb, bi, be * pow_pos(s, -k.p) / static_cast<float>(k.g), &zmin, &zmax);
        }
        if (k.zero_nbits == 8) write_minmax<kRegWarps>(k, zmin, zmax, sred);
        return;
    }

    // ---------------------------------------------------- tensor mode ----
    const int iters = k.iters_eff;
    const int nch = num_chunks(iters);
    // Stop rule on the tensor errors of iterations [0, k0) (same decision in every CTA).
    const int k0 = chunk_begin(chunk, iters);
    int best_it = -1, stop_at = -1;
    {
        double best = INFINITY;
        for (int it = 0; it < k0; ++it) {
            const double e = __ldcg(k.etot + it);
            if (e < best) {
                best = e;
                best_it = it;
            } else {
                stop_at = it;
                break;
            }
        }
    }
    const int prev_begin = chunk > 0 ? chunk_begin(chunk - 1, iters) : 0;
    bool finalize;
    if (stop_at >= 0) {
        if (stop_at < prev_begin) return;  // an earlier launch already wrote the outputs
        finalize = true;
    } else {
        finalize = chunk >= nch;
        if (finalize) best_it = iters - 1;
    }
    float* const Zs0 = k.t_zs;
    float* const Zs1 = k.t_zs + G;
    float* const Zs2 = k.t_zs + 2 * G;

    if (finalize) {
        const int kb = best_it < 0 ? 0 : best_it;  // iters == 0: z* = z0
        const int cb = chunk_of(kb), b0 = chunk_begin(cb, iters);
        const float* Zc = (cb % 3 == 0) ? Zs0 : (cb % 3 == 1 ? Zs1 : Zs2);
        for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRegWarps + warp; t < ntiles; t += wstride) {
            const WarpTile w = warp_tile<AXIS>(k, t);
            float x[E], ws[E];
            load_lane<DT, AXIS, E>(k, w, x);
            float s, z0, lmin, lmax;
            double sws;
            init_lane<E>(k, w, x, ws, &s, &z0, &sws, &lmin, &lmax);
            float z = (iters == 0 || cb == 0) ? z0 : (w.valid ? Zc[w.j] : 0.0f);
            float beta = beta_at(k, b0);
            for (int it = b0; it < kb; ++it) {
                z = step_lane<E>(k, w.valid, x, ws, s, z, z0, beta, shrink_threshold(beta, k.p), sws);
                beta = __fmul_rn(beta, k.kappa);
            }
            store_lane_codes<AXIS, E>(k, w, ws, z);
            float err_mean = 0.0f;
            if (k.dbg_err) {
                float err, sq;
                bool sp;
                double swe;
                eval_lane<E>(k, w.valid, x, ws, s, z, z0, beta, shrink_threshold(beta, k.p), &err, &sq, &sp, &swe);
                err_mean = err * pow_pos(s, -k.p) / static_cast<float>(k.g);
            }
            if (w.valid && w.part == 0) store_group(k, w.j, s, z, kb, err_mean, &zmin, &zmax);
        }
        if (k.zero_nbits == 8) write_minmax<kRegWarps>(k, zmin, zmax, sred);
        return;
    }

    // run iterations [k0, k1)
    const int k1 = chunk_begin(chunk + 1, iters);
    const int nk = k1 - k0;
    float* const Zin = (chunk % 3 == 0) ? Zs0 : (chunk % 3 == 1 ? Zs1 : Zs2);
    float* const Zout = ((chunk + 1) % 3 == 0) ? Zs0 : ((chunk + 1) % 3 == 1 ? Zs1 : Zs2);
    // per-thread tensor error partials: registers for small tiles, else shared
    double accr[kChunkMax] = {0.0, 0.0, 0.0, 0.0};
    for (int q = 0; q < kChunkMax; ++q) sacc[q][threadIdx.x] = 0.0;
    if (threadIdx.x < kChunkMax) sthr[threadIdx.x] = shrink_threshold(beta_at(k, k0 + threadIdx.x), k.p);
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
        if constexpr (E <= 16) {
#pragma unroll
            for (int q = 0; q < kChunkMax; ++q)
                if (q < nk) tensor_iteration<DT, AXIS, E>(k, w, ws, lmin, lmax, s, z0, k0 + q, sthr[q], spow, sws2,
                                                          inv_g, accr[q], z);
        } else {
#pragma unroll 1
            for (int q = 0; q < nk; ++q)
                tensor_iteration<DT, AXIS, E>(k, w, ws, lmin, lmax, s, z0, k0 + q, sthr[q], spow, sws2, inv_g,
                                              sacc[q][threadIdx.x], z);
        }
        if (w.valid && w.part == 0) Zout[w.j] = z;
    }
    // per-CTA partials (fixed order), then the last CTA sums them in a fixed order
    if constexpr (E <= 16) {
#pragma unroll
        for (int q = 0; q < kChunkMax; ++q) sacc[q][threadIdx.x] = accr[q];
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
        const unsigned prev = atomicAdd(k.counters + 1, 1u);
        sflag = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!sflag) return;
    __threadfence();
    for (int q = warp; q < nk; q += kRegWarps) {
        double v = 0.0;
        for (unsigned b = lane; b < gridDim.x; b += 32)
            v += __ldcg(k.tparts + static_cast<size_t>(q) * kMaxPartials + b);
        v = warp_sum_d(v);
        if (lane == 0) k.etot[k0 + q] = v / static_cast<double>(k.n);
    }
    if (threadIdx.x == 0) k.counters[1] = 0;
}

// ------------------------------------------------------- 8-bit zero ------

__global__ void __launch_bounds__(256) zero_q8_kernel(const float* zbest, int64_t G, const float2* minmax, int nparts,
                                                       uint8_t* zq, float* meta) {
    __shared__ float2 sred[8];
    float mn = FLT_MAX, mx = -FLT_MAX;
    for (int i = threadIdx.x; i < nparts; i += 256) {
        const float2 v = minmax[i];
        mn = fminf(mn, v.x);
        mx = fmaxf(mx, v.y);
    }
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    }
    if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = make_float2(mn, mx);
    __syncthreads();
    mn = sred[0].x;
    mx = sred[0].y;
    for (int w = 1; w < 8; ++w) {
        mn = fminf(mn, sred[w].x);
        mx = fmaxf(mx, sred[w].y);
    }
    if (G == 0) mn = mx = 0.0f;
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
    const uint16_t* scale;
    const void* zero;
    const float* meta;
    int64_t rows, cols;
    int nbits, g, zero_nbits;
    uint16_t* out;
};

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
            const float sc = __half2float(__ushort_as_half(d.scale[j]));
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
            const float sc = __half2float(__ushort_as_half(d.scale[j]));
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
};

DevInfo device_info() {
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!have[dev]) {
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cache[dev].sms = sms > 0 ? sms : 1;
        have[dev] = true;
    }
    return cache[dev];
}

template <typename K>
cudaError_t persistent_grid(K kernel, int threads, size_t smem, int64_t work_units, int* grid) {
    if (smem > 48 * 1024) {
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

// Cells per warp of the pool kernel: ~6 KB of fp32 data, at least one full
// pass of lanes, at most 64 cells.
int pool_cells(int g, int P) {
    int nc = 6144 / (4 * pool_cell_floats(g));
    if (nc * P < 32) nc = 32 / P;
    if (nc > 64) nc = 64;
    if (nc < 1) nc = 1;
    return nc;
}

template <int DT, int E, int NBITS>
cudaError_t launch_pool(KParams& k, cudaStream_t stream, int* grid) {
    k.NC = pool_cells(k.g, k.P);
    k.pool_warp_bytes = pool_warp_bytes(k.NC, k.g);
    const size_t smem = static_cast<size_t>(k.pool_warp_bytes) * kPoolWarps;
    auto kern = solve_pool_kernel<DT, E, NBITS>;
    const int64_t warps_needed = (k.G + k.NC - 1) / k.NC;
    cudaError_t err = persistent_grid(kern, kPoolThreads, smem, (warps_needed + kPoolWarps - 1) / kPoolWarps, grid);
    if (err != cudaSuccess) return err;
    kern<<<*grid, kPoolThreads, smem, stream>>>(k);
    return cudaGetLastError();
}

template <int DT, int E>
cudaError_t launch_pool_b(KParams& k, cudaStream_t stream, int* grid) {
    switch (k.nbits) {
        case 1: return launch_pool<DT, E, 1>(k, stream, grid);
        case 2: return launch_pool<DT, E, 2>(k, stream, grid);
        case 3: return launch_pool<DT, E, 3>(k, stream, grid);
        case 4: return launch_pool<DT, E, 4>(k, stream, grid);
        default: return launch_pool<DT, E, 8>(k, stream, grid);
    }
}

template <int DT, int AXIS, int E>
cudaError_t launch_reg(KParams& k, cudaStream_t stream, int* grid) {
    const int gpw = 32 >> k.logP;
    const int64_t tiles = AXIS == 1 ? (k.G + gpw - 1) / gpw : (k.rows / k.g) * ((k.cols + gpw - 1) / gpw);
    const int64_t ctas = (tiles + kRegWarps - 1) / kRegWarps;
    if (k.stop_mode != 1) {
        auto kern = solve_reg_kernel<DT, AXIS, E, MODE_LOCAL>;
        cudaError_t err = persistent_grid(kern, kRegThreads, 0, ctas, grid);
        if (err != cudaSuccess) return err;
        kern<<<*grid, kRegThreads, 0, stream>>>(k, 0);
        return cudaGetLastError();
    }
    auto kern = solve_reg_kernel<DT, AXIS, E, MODE_TENSOR>;
    cudaError_t err = persistent_grid(kern, kRegThreads, 0, ctas, grid);
    if (err != cudaSuccess) return err;
    const int nch = num_chunks(k.iters_eff);
    for (int c = 0; c <= nch; ++c) {  // nch chunks, then the launch that writes the outputs
        kern<<<*grid, kRegThreads, 0, stream>>>(k, c);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

// The register kernel holds a whole group per thread up to g = 32 (E = g,
// P = 1): every lane then has E independent elements per iteration and the
// group sums need no shuffles; larger groups spread over P = g/32 lanes.
template <int DT, int AXIS>
cudaError_t launch_reg_e(KParams& k, cudaStream_t stream, int* grid) {
    k.E = k.g < 32 ? k.g : 32;
    k.P = k.g / k.E;
    k.logP = 0;
    while ((1 << k.logP) < k.P) ++k.logP;
    if (k.E == 8) return launch_reg<DT, AXIS, 8>(k, stream, grid);
    if (k.E == 16) return launch_reg<DT, AXIS, 16>(k, stream, grid);
    return launch_reg<DT, AXIS, 32>(k, stream, grid);
}

template <int DT>
cudaError_t launch_pool_e(KParams& k, cudaStream_t stream, int* grid) {
    if (k.E == 8) return launch_pool_b<DT, 8>(k, stream, grid);
    if (k.E == 16) return launch_pool_b<DT, 16>(k, stream, grid);
    return launch_pool_b<DT, 32>(k, stream, grid);
}

}  // namespace

Geometry make_geometry(int g) {
    Geometry geo;
    geo.g = g;
    geo.E = g <= 8 ? 8 : (g <= 512 ? 16 : 32);
    geo.P = g / geo.E;
    return geo;
}

WorkspaceLayout workspace_layout(int64_t G, int stop_mode, int zero_nbits, int iters) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    WorkspaceLayout l{};
    size_t off = 0;
    l.header = off;
    off += 256;
    l.minmax = off;
    off = up(off + sizeof(float) * 2 * kMaxPartials);
    const size_t Gs = static_cast<size_t>(G > 0 ? G : 0);
    l.zbest = off;
    if (zero_nbits == 8) off = up(off + 4 * Gs);
    l.tparts = l.etot = l.t_s = l.t_z0 = l.t_sws = l.t_zs = off;
    if (stop_mode == 1) {
        const size_t it = static_cast<size_t>(iters > 0 ? iters : 1);
        l.tparts = off;
        off = up(off + sizeof(double) * kChunkMax * kMaxPartials);
        l.etot = off;
        off = up(off + sizeof(double) * it);
        l.t_s = off;
        off = up(off + 4 * Gs);
        l.t_z0 = off;
        off = up(off + 4 * Gs);
        l.t_sws = off;
        off = up(off + 8 * Gs);
        l.t_zs = off;
        off = up(off + 12 * Gs);
    }
    l.total = off;
    return l;
}

cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream) {
    const Geometry geo = make_geometry(a.g);
    const WorkspaceLayout L = workspace_layout(a.G, a.stop_mode, a.zero_nbits, kMaxIters);
    KParams k{};
    k.W = static_cast<const uint16_t*>(a.W);
    k.rows = a.rows;
    k.cols = a.cols;
    k.G = a.G;
    k.n = a.rows * a.cols;
    k.g = a.g;
    k.E = geo.E;
    k.P = geo.P;
    k.logP = 0;
    while ((1 << k.logP) < geo.P) ++k.logP;
    k.nbits = a.nbits;
    k.iters = a.iters;
    k.iters_eff = a.iters > 0 ? a.iters : (a.dbg_err ? 1 : 0);  // iters 0 == 1: z* = z0 either way
    k.stop_mode = a.stop_mode;
    k.zero_nbits = a.zero_nbits;
    k.axis = a.axis;
    k.p = a.p;
    k.beta = a.beta;
    k.kappa = a.kappa;
    k.Lf = static_cast<float>((1 << a.nbits) - 1);
    k.packed = a.packed;
    k.scale = a.scale;
    k.zero = a.zero;
    k.dbg_iter = a.dbg_iter;
    k.dbg_err = a.dbg_err;
    k.dbg_zero = a.dbg_zero;
    k.counters = reinterpret_cast<uint32_t*>(a.ws + L.header);
    k.minmax = reinterpret_cast<float2*>(a.ws + L.minmax);
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
    int grid = 0;
    if (a.G > 0) {
        const bool pool = a.axis == 1 && a.stop_mode != 1;
        if (pool) err = a.dtype == 0 ? launch_pool_e<0>(k, stream, &grid) : launch_pool_e<1>(k, stream, &grid);
        else if (a.dtype == 0 && a.axis == 1) err = launch_reg_e<0, 1>(k, stream, &grid);
        else if (a.dtype == 0) err = launch_reg_e<0, 0>(k, stream, &grid);
        else if (a.axis == 1) err = launch_reg_e<1, 1>(k, stream, &grid);
        else err = launch_reg_e<1, 0>(k, stream, &grid);
        if (err != cudaSuccess) return err;
    }
    if (a.zero_nbits == 8) {
        int64_t blocks = (a.G + 255) / 256;
        const int64_t cap = static_cast<int64_t>(device_info().sms) * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        zero_q8_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(k.zbest_ws, a.G, k.minmax, grid,
                                                                    static_cast<uint8_t*>(a.zero), a.zero_meta);
        err = cudaGetLastError();
    }
    return err;
}

cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream) {
    DqParams d;
    d.packed = a.packed;
    d.scale = a.scale;
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
