// hqq_kernels.cu -- sm_100a kernels of the HQQ zero-point solver.
//
// Method: techreport.ngo, "Weight-only quantization without the calibration
// tax" (Half-Quadratic Quantization of Large Machine Learning Models), section
// "Outlier-aware optimization without gradients" (lp loss, half-quadratic
// split, generalised soft-thresholding, group-mean zero update, fixed scale)
// and section "Benchmark results"/"Llama-2" (p, beta, kappa, 20 iterations,
// early stopping, 8-bit zero).  The step formulas are restated in include/hqq.h.
//
// The path has no dense contraction, so there is no tensor-core work.  Per
// element and iteration it costs about ten FP32-pipe instructions and two
// MUFU ops (|r|^p = ex2(p * lg2|r|)); with ~2.5-4 evaluations per group in
// group mode the MUFU pipe, not HBM, bounds the solver.
//
// Data path of the group-mode kernel (one HBM pass):
//   tile of <= 512 groups (<= 16384 elements) -> shared memory
//   init: min/max -> s, z0; sum of w*s in fp64             (all groups)
//   rounds k = 0..iters-1: compact the still-active groups into a list, map
//     each active group onto P = g/8 consecutive lanes (one 16-byte piece of 8
//     elements per lane and pass), evaluate, reduce over the P lanes with xor
//     shuffles, update the group state; groups that stop free their lanes
//   final: codes with the kept z -> bit-pack -> HBM; scale/zero -> HBM
// The tensor-mode kernel is persistent and cooperative: every iteration each
// CTA evaluates its tiles, writes one fp64 partial of the tensor error, meets
// the other CTAs at a grid barrier (bounded wait) and takes the same stop
// decision from the partials summed in a fixed order.

#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include <cfloat>
#include <cstdint>

#include "hqq_internal.h"

namespace hqq {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarps = kThreads / 32;

// ------------------------------------------------------------ helpers ----

__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// a^e for a >= 0 through the hardware base-2 log and exponential (0^e = 0 for e > 0).
__device__ __forceinline__ float pow_pos(float a, float e) { return ex2_approx(e * lg2_approx(a)); }

template <int DT>
__device__ __forceinline__ float elem_to_float(uint16_t b) {
    if (DT == 0) return __half2float(__ushort_as_half(b));
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Eight consecutive 16-bit elements (one aligned 16-byte piece) -> fp32.
template <int DT>
__device__ __forceinline__ void load8(const uint16_t* p, float* w) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (DT == 0) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x[i]));
            w[2 * i] = f.x;
            w[2 * i + 1] = f.y;
        } else {
            w[2 * i] = __uint_as_float(x[i] << 16);
            w[2 * i + 1] = __uint_as_float(x[i] & 0xffff0000u);
        }
    }
}

// W_q = clamp(round_half_even(w*s + z), 0, L); products and sums rounded separately.
__device__ __forceinline__ float quant(float w, float s, float z, float Lf, float* v_out) {
    const float v = __fadd_rn(__fmul_rn(w, s), z);
    *v_out = v;
    return fminf(fmaxf(rintf(v), 0.0f), Lf);
}

// Segment reductions over P consecutive lanes (P a power of two <= 32); every
// lane of the segment ends with the same value.
__device__ __forceinline__ float seg_sum(float x, int P) {
    for (int o = 1; o < P; o <<= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}
__device__ __forceinline__ double seg_sum_d(double x, int P) {
    for (int o = 1; o < P; o <<= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}
__device__ __forceinline__ float seg_min(float x, int P) {
    for (int o = 1; o < P; o <<= 1) x = fminf(x, __shfl_xor_sync(kFull, x, o));
    return x;
}
__device__ __forceinline__ float seg_max(float x, int P) {
    for (int o = 1; o < P; o <<= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
    return x;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ------------------------------------------------------------ params -----

struct KParams {
    const uint16_t* W;
    int64_t rows, cols, G;
    int g, P, logP, NP, tile_groups, tile_elems;
    int nbits, iters, iters_eff, stop_mode, zero_nbits;
    float p, beta, kappa, Lf;
    int64_t ntiles, ncoltiles;
    uint8_t* packed;
    uint16_t* scale;
    void* zero;
    int32_t* dbg_iter;
    float* dbg_err;
    float* dbg_zero;
    uint32_t* status;
    uint32_t* bar_count;
    uint32_t* bar_gen;
    float2* minmax;
    double* tparts;
    float* zbest_ws;
    float* t_s;
    float* t_is;
    float* t_z0;
    double* t_sws;
    float* t_z;
    float* t_e;
    int vec_ok;
    int skip_block;
    unsigned long long timeout_ns;
};

// ------------------------------------------------------------ tiles ------

struct TileInfo {
    int ntg;           // groups in this tile
    int64_t j0;        // axis 1: first group index
    int64_t rb, c0;    // axis 0: row block and first column
};

template <int AXIS>
__device__ __forceinline__ TileInfo tile_info(const KParams& k, int64_t tile) {
    TileInfo t;
    if (AXIS == 1) {
        t.j0 = tile * k.tile_groups;
        const int64_t left = k.G - t.j0;
        t.ntg = left < k.tile_groups ? static_cast<int>(left) : k.tile_groups;
        t.rb = t.c0 = 0;
    } else {
        t.rb = tile / k.ncoltiles;
        t.c0 = (tile % k.ncoltiles) * k.tile_groups;
        const int64_t left = k.cols - t.c0;
        t.ntg = left < k.tile_groups ? static_cast<int>(left) : k.tile_groups;
        t.j0 = 0;
    }
    return t;
}

template <int AXIS>
__device__ __forceinline__ int64_t group_index(const KParams& k, const TileInfo& t, int lt) {
    return AXIS == 1 ? t.j0 + lt : t.rb * k.cols + t.c0 + lt;
}

// Stage one tile in shared memory, group-major: element i of local group lt
// at sdata[lt*g + i].  For axis 1 that is a straight copy of a contiguous
// range; for axis 0 the g x ntg block of rows/columns is transposed.
template <int AXIS, bool STREAM>
__device__ __forceinline__ void load_tile(const KParams& k, const TileInfo& t, uint16_t* sdata) {
    const int tid = threadIdx.x;
    if (AXIS == 1) {
        const int npieces = t.ntg * k.g / kPiece;
        const uint4* src = reinterpret_cast<const uint4*>(k.W + t.j0 * k.g);
        uint4* dst = reinterpret_cast<uint4*>(sdata);
        for (int pc = tid; pc < npieces; pc += kThreads) dst[pc] = STREAM ? __ldcs(src + pc) : __ldg(src + pc);
    } else if (k.vec_ok) {
        // unit = (row pair rp, 8-column piece cp): two 16-byte row loads -> eight
        // 32-bit stores (rows 2rp, 2rp+1 of one column)
        const int half = k.g / 2;
        const int units = half * (t.ntg / kPiece);
        for (int u = tid; u < units; u += kThreads) {
            const int rp = u % half, cp = u / half;
            const int64_t r = t.rb * k.g + 2 * rp;
            const uint16_t* p0 = k.W + r * k.cols + t.c0 + cp * kPiece;
            const uint4 a = STREAM ? __ldcs(reinterpret_cast<const uint4*>(p0)) : __ldg(reinterpret_cast<const uint4*>(p0));
            const uint4 b = STREAM ? __ldcs(reinterpret_cast<const uint4*>(p0 + k.cols))
                                   : __ldg(reinterpret_cast<const uint4*>(p0 + k.cols));
            const uint32_t xa[4] = {a.x, a.y, a.z, a.w}, xb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t lo = (xa[j >> 1] >> (16 * (j & 1))) & 0xffffu;
                const uint32_t hi = (xb[j >> 1] >> (16 * (j & 1))) & 0xffffu;
                *reinterpret_cast<uint32_t*>(sdata + (cp * kPiece + j) * k.g + 2 * rp) = lo | (hi << 16);
            }
        }
    } else {
        const int n = k.g * t.ntg;
        for (int e = tid; e < n; e += kThreads) {
            const int i = e / t.ntg, cl = e % t.ntg;
            sdata[cl * k.g + i] = k.W[(t.rb * k.g + i) * k.cols + t.c0 + cl];
        }
    }
}

// ------------------------------------------------------ per-group steps --

// min/max -> s, z0 and the fp64 sum of w*s for the group of this item.
// Must be called by whole warps (lanes with valid == false contribute nothing).
template <int DT>
__device__ __forceinline__ void init_item(const KParams& k, const uint16_t* sg, int part, bool valid, float* s_out,
                                          float* z0_out, double* sws_out) {
    float mn = FLT_MAX, mx = -FLT_MAX;
    if (valid) {
        for (int n = 0; n < k.NP; ++n) {
            float w[8];
            load8<DT>(sg + (part + n * k.P) * kPiece, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mn = fminf(mn, w[i]);
                mx = fmaxf(mx, w[i]);
            }
        }
    }
    mn = seg_min(mn, k.P);
    mx = seg_max(mx, k.P);
    float s = kScaleCap;
    if (mx > mn) s = fminf(__fdiv_rn(k.Lf, __fsub_rn(mx, mn)), kScaleCap);
    const float z0 = __fmul_rn(-mn, s);
    double acc = 0.0;
    if (valid) {
        for (int n = 0; n < k.NP; ++n) {
            float w[8];
            load8<DT>(sg + (part + n * k.P) * kPiece, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc += static_cast<double>(__fmul_rn(w[i], s));
        }
    }
    acc = seg_sum_d(acc, k.P);
    *s_out = s;
    *z0_out = z0;
    *sws_out = acc;
}

struct Eval {
    float err;     // sum over the group of |w - W_r|^p
    float sq;      // sum of W_q (exact: integers < 2^24)
    double sws_e;  // sum of fl((w - W_e)*s), only when the shrink may be active
    bool sp;       // the shrink may be active for this group
};

// Evaluate zero-point z on the item's pieces and reduce over the group's lanes.
// Whole warps only.  W_r = (W_q - z) * (1/s) in fp32, the dequantiser's form.
// The shrink W_e is exactly zero unless some |w - W_r| exceeds
// beta^(-1/(2-p)) (= thr); |w - W_r|*s <= max(0.5, |z - z0|) up to rounding,
// so groups below that bound skip the per-element proximal step.
template <int DT>
__device__ __forceinline__ Eval eval_item(const KParams& k, const uint16_t* sg, int part, bool valid, float s,
                                          float inv_s, float z, float z0, float beta, float thr) {
    Eval e;
    float err = 0.0f, sq = 0.0f;
    const bool sp = valid && (fmaxf(0.5f, fabsf(z - z0)) + 1e-3f * (1.0f + k.Lf + fabsf(z)) >= 0.99f * thr * s);
    if (valid) {
        for (int n = 0; n < k.NP; ++n) {
            float w[8];
            load8<DT>(sg + (part + n * k.P) * kPiece, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float v;
                const float q = quant(w[i], s, z, k.Lf, &v);
                const float d = __fsub_rn(w[i], __fmul_rn(__fsub_rn(q, z), inv_s));
                err += pow_pos(fabsf(d), k.p);
                sq += q;
            }
        }
    }
    e.err = seg_sum(err, k.P);
    e.sq = seg_sum(sq, k.P);
    e.sws_e = 0.0;
    e.sp = sp;
    if (__any_sync(kFull, sp)) {
        double st = 0.0;
        if (sp) {
            for (int n = 0; n < k.NP; ++n) {
                float w[8];
                load8<DT>(sg + (part + n * k.P) * kPiece, w);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float v;
                    const float q = quant(w[i], s, z, k.Lf, &v);
                    const float d = __fsub_rn(w[i], __fmul_rn(__fsub_rn(q, z), inv_s));
                    const float a = fabsf(d);
                    float we = 0.0f;
                    if (a != 0.0f) {
                        const float t = __fsub_rn(a, __fdiv_rn(pow_pos(a, k.p - 1.0f), beta));
                        if (t > 0.0f) we = copysignf(t, d);
                    }
                    st += static_cast<double>(__fmul_rn(__fsub_rn(w[i], we), s));
                }
            }
        }
        e.sws_e = seg_sum_d(st, k.P);
    }
    return e;
}

// z_{k+1} = (sum W_q - sum fl((w - W_e)*s)) / g with fp64 sums; sws is the
// precomputed sum of fl(w*s) used when W_e is zero for the whole group.
__device__ __forceinline__ float next_zero(const Eval& e, double sws, int g) {
    const double t = e.sp ? e.sws_e : sws;
    return static_cast<float>((static_cast<double>(e.sq) - t) / static_cast<double>(g));
}

// beta^(-1/(2-p)): below this |w - W_r| the proximal step returns exactly 0.
__device__ __forceinline__ float shrink_threshold(float beta, float p) {
    return ex2_approx(-lg2_approx(beta) / (2.0f - p));
}

// Pack eight codes (LSB first) into the low nbits*8 bits of a 64-bit word.
__device__ __forceinline__ uint64_t pack8(const float* q, int nbits) {
    uint64_t v = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v |= static_cast<uint64_t>(static_cast<uint32_t>(q[i])) << (i * nbits);
    return v;
}

__device__ __forceinline__ void store_packed_contig(uint8_t* dst, uint64_t v, int nbits) {
    switch (nbits) {
        case 1: *dst = static_cast<uint8_t>(v); break;
        case 2: *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(v); break;
        case 4: *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(v); break;
        case 8: *reinterpret_cast<uint64_t*>(dst) = v; break;
        default:
            dst[0] = static_cast<uint8_t>(v);
            dst[1] = static_cast<uint8_t>(v >> 8);
            dst[2] = static_cast<uint8_t>(v >> 16);
            break;
    }
}

// Final codes of one tile with per-group (s, z*) from shared arrays, packed to HBM.
template <int DT, int AXIS>
__device__ __forceinline__ void pack_tile(const KParams& k, const TileInfo& t, const uint16_t* sdata,
                                          const float* s_arr, const float* z_arr) {
    const int ppg = k.g / kPiece;  // pieces per group
    const int npieces = t.ntg * ppg;
    for (int it = threadIdx.x; it < npieces; it += kThreads) {
        int lt, m;
        if (AXIS == 1) {
            lt = it / ppg;
            m = it % ppg;
        } else {
            m = it / t.ntg;
            lt = it % t.ntg;  // consecutive lanes -> consecutive columns
        }
        float w[8], q[8];
        load8<DT>(sdata + lt * k.g + m * kPiece, w);
        const float s = s_arr[lt], z = z_arr[lt];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float v;
            q[i] = quant(w[i], s, z, k.Lf, &v);
        }
        const uint64_t v = pack8(q, k.nbits);
        if (AXIS == 1) {
            const int64_t piece = (t.j0 * k.g) / kPiece + it;
            store_packed_contig(k.packed + piece * k.nbits, v, k.nbits);
        } else {
            const int64_t row_byte = (t.rb * k.g) / kPiece * k.nbits + static_cast<int64_t>(m) * k.nbits;
            uint8_t* dst = k.packed + row_byte * k.cols + t.c0 + lt;
            for (int b = 0; b < k.nbits; ++b) dst[b * k.cols] = static_cast<uint8_t>(v >> (8 * b));
        }
    }
}

__device__ __forceinline__ uint16_t half_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

// scale, zero and debug outputs of one group; tracks the zero-point min/max.
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

// Block-wide min/max -> one partial per CTA.
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
        for (int w = 1; w < kWarps; ++w) {
            r.x = fminf(r.x, sred[w].x);
            r.y = fmaxf(r.y, sred[w].y);
        }
        k.minmax[blockIdx.x] = r;
    }
}

// Ordered compaction of active[0..ntg) into list; returns the count.
__device__ __forceinline__ int compact(const uint8_t* active, uint16_t* list, int ntg, int* sscan) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g0 = tid * 2;
    const int f0 = (g0 < ntg) ? active[g0] : 0;
    const int f1 = (g0 + 1 < ntg) ? active[g0 + 1] : 0;
    const int c = f0 + f1;
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sscan[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kWarps ? sscan[lane] : 0;
#pragma unroll
        for (int o = 1; o < kWarps; o <<= 1) {
            const int y = __shfl_up_sync(kFull, v, o);
            if (lane >= o) v += y;
        }
        if (lane < kWarps) sscan[kWarps + lane] = v;
    }
    __syncthreads();
    int pos = x - c + (warp > 0 ? sscan[kWarps + warp - 1] : 0);
    if (f0) list[pos++] = static_cast<uint16_t>(g0);
    if (f1) list[pos] = static_cast<uint16_t>(g0 + 1);
    const int total = sscan[2 * kWarps - 1];
    __syncthreads();
    return total;
}

// ------------------------------------------------- group / no-stop kernel --

struct GroupSmem {
    uint16_t* data;
    float *s, *is, *z, *zb, *z0, *be;
    double* sws;
    int* bi;
    uint8_t* active;
    uint16_t* list;
};

__device__ __forceinline__ GroupSmem carve_group_smem(unsigned char* base, const KParams& k) {
    GroupSmem m;
    const int TG = k.tile_groups;
    size_t off = 0;
    m.data = reinterpret_cast<uint16_t*>(base + off);
    off += static_cast<size_t>(k.tile_elems) * 2;
    m.sws = reinterpret_cast<double*>(base + off);
    off += TG * 8;
    m.s = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.is = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.z = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.zb = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.z0 = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.be = reinterpret_cast<float*>(base + off);
    off += TG * 4;
    m.bi = reinterpret_cast<int*>(base + off);
    off += TG * 4;
    m.list = reinterpret_cast<uint16_t*>(base + off);
    off += TG * 2;
    m.active = reinterpret_cast<uint8_t*>(base + off);
    return m;
}

template <int DT, int AXIS>
__global__ void __launch_bounds__(kThreads) solve_group_kernel(const KParams k) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int sscan[2 * kWarps];
    __shared__ float2 sred[kWarps];
    const GroupSmem m = carve_group_smem(smem_raw, k);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool stop_group = k.stop_mode == 0;
    float zmin = FLT_MAX, zmax = -FLT_MAX;

    for (int64_t tile = blockIdx.x; tile < k.ntiles; tile += gridDim.x) {
        const TileInfo t = tile_info<AXIS>(k, tile);
        load_tile<AXIS, true>(k, t, m.data);
        __syncthreads();

        // init: every group of the tile
        const int items0 = t.ntg * k.P;
        for (int b = warp * 32; b < items0; b += kThreads) {
            const int item = b + lane;
            const bool valid = item < items0;
            const int lt = valid ? (item >> k.logP) : 0;
            const int part = item & (k.P - 1);
            float s, z0;
            double sws;
            init_item<DT>(k, m.data + lt * k.g, part, valid, &s, &z0, &sws);
            if (valid && part == 0) {
                m.s[lt] = s;
                m.is[lt] = __fdiv_rn(1.0f, s);
                m.z0[lt] = z0;
                m.z[lt] = z0;
                m.zb[lt] = z0;
                m.sws[lt] = sws;
                m.be[lt] = INFINITY;
                m.bi[lt] = 0;
            }
        }
        for (int lt = tid; lt < k.tile_groups; lt += kThreads) m.active[lt] = lt < t.ntg ? 1 : 0;
        __syncthreads();

        // rounds: all active groups are at iteration `it`
        float beta = k.beta;
        for (int it = 0; it < k.iters_eff; ++it) {
            const float thr = shrink_threshold(beta, k.p);
            const int A = compact(m.active, m.list, t.ntg, sscan);
            if (A == 0) break;
            const int items = A * k.P;
            for (int b = warp * 32; b < items; b += kThreads) {
                const int item = b + lane;
                const bool valid = item < items;
                const int lt = valid ? m.list[item >> k.logP] : 0;
                const int part = item & (k.P - 1);
                const float s = m.s[lt], is = m.is[lt], z = m.z[lt], z0 = m.z0[lt];
                const Eval e = eval_item<DT>(k, m.data + lt * k.g, part, valid, s, is, z, z0, beta, thr);
                if (valid && part == 0) {
                    bool alive = true;
                    if (e.err < m.be[lt]) {
                        m.be[lt] = e.err;
                        m.zb[lt] = z;
                        m.bi[lt] = it;
                    } else if (stop_group) {
                        alive = false;
                    }
                    if (alive) {
                        m.z[lt] = next_zero(e, m.sws[lt], k.g);
                        if (it == k.iters_eff - 1) alive = false;
                    }
                    if (!alive) m.active[lt] = 0;
                }
            }
            beta = __fmul_rn(beta, k.kappa);
            __syncthreads();
        }

        // final codes and group outputs
        pack_tile<DT, AXIS>(k, t, m.data, m.s, m.zb);
        for (int lt = tid; lt < t.ntg; lt += kThreads) {
            const float err_mean = m.be[lt] / static_cast<float>(k.g);
            store_group(k, group_index<AXIS>(k, t, lt), m.s[lt], m.zb[lt], m.bi[lt], err_mean, &zmin, &zmax);
        }
        __syncthreads();
    }
    if (k.zero_nbits == 8) write_minmax(k, zmin, zmax, sred);
}

// ------------------------------------------------------ tensor kernel ----

// Grid barrier for a cooperative launch.  The wait is bounded by k.timeout_ns;
// on expiry the CTA records HQQ_ERR_TIMEOUT and the caller returns.
__device__ bool grid_barrier(const KParams& k, int round, int* sflag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        const uint32_t gen = ld_acquire(k.bar_gen);
        const bool skip = (round == 0 && static_cast<int>(blockIdx.x) == k.skip_block);
        if (!skip) {
            __threadfence();
            const uint32_t arrived = atomicAdd(k.bar_count, 1u);
            if (arrived == gridDim.x - 1) {
                atomicExch(k.bar_count, 0u);
                __threadfence();
                st_release(k.bar_gen, gen + 1);
            }
        }
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire(k.bar_gen) == gen) {
            if (ld_acquire(k.status) != kStatusOk || globaltimer_ns() - t0 > k.timeout_ns) {
                atomicExch(k.status, kStatusTimeout);
                ok = 0;
                break;
            }
            __nanosleep(128);
        }
        *sflag = ok;
    }
    __syncthreads();
    return *sflag != 0;
}

__device__ __forceinline__ double block_sum_d(double x, double* sredd) {
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sredd[warp] = x;
    __syncthreads();
    double r = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kWarps; ++w) r += sredd[w];
    __syncthreads();
    return r;  // valid in thread 0
}

template <int DT, int AXIS>
__global__ void __launch_bounds__(kThreads) solve_tensor_kernel(const KParams k) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int sflag;
    __shared__ int sdecide[2];
    __shared__ double sredd[kWarps];
    __shared__ float2 sred[kWarps];
    uint16_t* sdata = reinterpret_cast<uint16_t*>(smem_raw);
    float* s_arr = reinterpret_cast<float*>(smem_raw + static_cast<size_t>(k.tile_elems) * 2);
    float* z_arr = s_arr + k.tile_groups;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool resident = k.ntiles <= static_cast<int64_t>(gridDim.x);
    const int64_t G = k.G;
    float* Z0 = k.t_z;
    float* Z1 = k.t_z + G;
    float* Z2 = k.t_z + 2 * G;
    float* const Zr[3] = {Z0, Z1, Z2};
    float* const Er[3] = {k.t_e, k.t_e ? k.t_e + G : nullptr, k.t_e ? k.t_e + 2 * G : nullptr};

    // init pass
    for (int64_t tile = blockIdx.x; tile < k.ntiles; tile += gridDim.x) {
        const TileInfo t = tile_info<AXIS>(k, tile);
        load_tile<AXIS, false>(k, t, sdata);
        __syncthreads();
        const int items0 = t.ntg * k.P;
        for (int b = warp * 32; b < items0; b += kThreads) {
            const int item = b + lane;
            const bool valid = item < items0;
            const int lt = valid ? (item >> k.logP) : 0;
            const int part = item & (k.P - 1);
            float s, z0;
            double sws;
            init_item<DT>(k, sdata + lt * k.g, part, valid, &s, &z0, &sws);
            if (valid && part == 0) {
                const int64_t j = group_index<AXIS>(k, t, lt);
                k.t_s[j] = s;
                k.t_is[j] = __fdiv_rn(1.0f, s);
                k.t_z0[j] = z0;
                k.t_sws[j] = sws;
                Z0[j] = z0;
            }
        }
        __syncthreads();
    }

    int best_it = 0;
    double best = INFINITY;
    float beta = k.beta;
    for (int it = 0; it < k.iters_eff; ++it) {
        const float thr = shrink_threshold(beta, k.p);
        const float* Zc = Zr[it % 3];
        float* Zn = Zr[(it + 1) % 3];
        float* Ec = Er[it % 3];
        double acc = 0.0;
        for (int64_t tile = blockIdx.x; tile < k.ntiles; tile += gridDim.x) {
            const TileInfo t = tile_info<AXIS>(k, tile);
            if (!resident) {
                load_tile<AXIS, false>(k, t, sdata);
                __syncthreads();
            }
            const int items = t.ntg * k.P;
            for (int b = warp * 32; b < items; b += kThreads) {
                const int item = b + lane;
                const bool valid = item < items;
                const int lt = valid ? (item >> k.logP) : 0;
                const int part = item & (k.P - 1);
                const int64_t j = group_index<AXIS>(k, t, valid ? lt : 0);
                const float s = valid ? k.t_s[j] : 1.0f;
                const float is = valid ? k.t_is[j] : 1.0f;
                const float z = valid ? Zc[j] : 0.0f;
                const float z0 = valid ? k.t_z0[j] : 0.0f;
                const Eval e = eval_item<DT>(k, sdata + lt * k.g, part, valid, s, is, z, z0, beta, thr);
                if (valid && part == 0) {
                    const float gerr = e.err;  // sum over the group of |w - W_r|^p
                    acc += static_cast<double>(gerr);
                    Zn[j] = next_zero(e, k.t_sws[j], k.g);
                    if (Ec) Ec[j] = gerr / static_cast<float>(k.g);
                }
            }
            if (!resident) __syncthreads();
        }
        const double cta = block_sum_d(acc, sredd);
        double* parts = k.tparts + (it & 1) * kMaxPartials;
        if (tid == 0) {
            parts[blockIdx.x] = cta;
            __threadfence();
        }
        if (!grid_barrier(k, it, &sflag)) return;
        if (tid == 0) {
            double total = 0.0;
            for (unsigned b = 0; b < gridDim.x; ++b) total += __ldcg(parts + b);
            const double E = total / (static_cast<double>(G) * k.g);
            const int improved = E < best;
            if (improved) {
                best = E;
                best_it = it;
            }
            sdecide[0] = improved;
            sdecide[1] = best_it;
        }
        __syncthreads();
        if (!sdecide[0]) break;
        beta = __fmul_rn(beta, k.kappa);
    }
    __syncthreads();
    best_it = sdecide[1];
    if (k.iters_eff == 0) best_it = 0;

    // final pass with the kept zero-points
    const float* Zb = Zr[best_it % 3];
    const float* Eb = Er[best_it % 3];
    float zmin = FLT_MAX, zmax = -FLT_MAX;
    for (int64_t tile = blockIdx.x; tile < k.ntiles; tile += gridDim.x) {
        const TileInfo t = tile_info<AXIS>(k, tile);
        if (!resident) load_tile<AXIS, false>(k, t, sdata);
        for (int lt = tid; lt < t.ntg; lt += kThreads) {
            const int64_t j = group_index<AXIS>(k, t, lt);
            s_arr[lt] = k.t_s[j];
            z_arr[lt] = Zb[j];
        }
        __syncthreads();
        pack_tile<DT, AXIS>(k, t, sdata, s_arr, z_arr);
        for (int lt = tid; lt < t.ntg; lt += kThreads) {
            const int64_t j = group_index<AXIS>(k, t, lt);
            store_group(k, j, s_arr[lt], z_arr[lt], best_it, Eb ? Eb[j] : 0.0f, &zmin, &zmax);
        }
        __syncthreads();
    }
    if (k.zero_nbits == 8) write_minmax(k, zmin, zmax, sred);
}

// ------------------------------------------------------- 8-bit zero ------

__global__ void __launch_bounds__(kThreads) zero_q8_kernel(const float* zbest, int64_t G, const float2* minmax,
                                                            int nparts, uint8_t* zq, float* meta) {
    __shared__ float2 sred[kWarps];
    float mn = FLT_MAX, mx = -FLT_MAX;
    for (int i = threadIdx.x; i < nparts; i += kThreads) {
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
    for (int w = 1; w < kWarps; ++w) {
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
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; j < G;
         j += static_cast<int64_t>(gridDim.x) * kThreads) {
        float v;
        zq[j] = static_cast<uint8_t>(quant(zbest[j], sz, zz, 255.0f, &v));
    }
}

// -------------------------------------------------------- dequantise -----

template <int OUT_DT>
__device__ __forceinline__ uint16_t float_to_out(float x) {
    if (OUT_DT == 0) return __half_as_ushort(__float2half_rn(x));
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint64_t load_packed_contig(const uint8_t* src, int nbits) {
    switch (nbits) {
        case 1: return *src;
        case 2: return *reinterpret_cast<const uint16_t*>(src);
        case 4: return *reinterpret_cast<const uint32_t*>(src);
        case 8: return *reinterpret_cast<const uint64_t*>(src);
        default: return static_cast<uint64_t>(src[0]) | (static_cast<uint64_t>(src[1]) << 8) |
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
__global__ void __launch_bounds__(kThreads) dequant_kernel(const DqParams d) {
    const uint32_t mask = (1u << d.nbits) - 1u;
    if (AXIS == 1) {
        const int64_t npieces = d.rows * d.cols / kPiece;
        for (int64_t pc = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; pc < npieces;
             pc += static_cast<int64_t>(gridDim.x) * kThreads) {
            const uint64_t v = load_packed_contig(d.packed + pc * d.nbits, d.nbits);
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
        const int64_t prow = d.rows / kPiece;  // 8-row pieces per column
        const int64_t n = prow * d.cols;
        for (int64_t u = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; u < n;
             u += static_cast<int64_t>(gridDim.x) * kThreads) {
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

int g_skip_block = -1;
unsigned long long g_timeout_ns = 0;

struct DevInfo {
    int sms = 0;
    bool coop = false;
};

DevInfo device_info() {
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!have[dev]) {
        int sms = 0, coop = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        cache[dev].sms = sms > 0 ? sms : 1;
        cache[dev].coop = coop != 0;
        have[dev] = true;
    }
    return cache[dev];
}

size_t group_smem_bytes(const Geometry& geo) {
    return static_cast<size_t>(geo.tile_elems) * 2 + static_cast<size_t>(geo.tile_groups) * (8 + 4 * 7 + 2 + 1);
}

size_t tensor_smem_bytes(const Geometry& geo) {
    return static_cast<size_t>(geo.tile_elems) * 2 + static_cast<size_t>(geo.tile_groups) * 8;
}

template <typename K>
cudaError_t occupancy_grid(K kernel, size_t smem, int64_t ntiles, int* grid) {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    int64_t cap = static_cast<int64_t>(device_info().sms) * per_sm;
    if (cap > kMaxPartials) cap = kMaxPartials;
    *grid = static_cast<int>(ntiles < cap ? (ntiles > 0 ? ntiles : 1) : cap);
    return cudaSuccess;
}

template <int DT, int AXIS>
cudaError_t launch_solve_t(KParams& k, cudaStream_t stream, int* coop_unsupported, int* grid_out) {
    const Geometry geo = make_geometry(k.g);
    if (k.stop_mode != 1) {
        auto kern = solve_group_kernel<DT, AXIS>;
        const size_t smem = group_smem_bytes(geo);
        int grid = 0;
        cudaError_t err = occupancy_grid(kern, smem, k.ntiles, &grid);
        if (err != cudaSuccess) return err;
        *grid_out = grid;
        kern<<<grid, kThreads, smem, stream>>>(k);
        return cudaGetLastError();
    }
    if (!device_info().coop) {
        *coop_unsupported = 1;
        return cudaSuccess;
    }
    auto kern = solve_tensor_kernel<DT, AXIS>;
    const size_t smem = tensor_smem_bytes(geo);
    int grid = 0;
    cudaError_t err = occupancy_grid(kern, smem, k.ntiles, &grid);
    if (err != cudaSuccess) return err;
    *grid_out = grid;
    void* args[] = {&k};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kThreads), args, smem,
                                       stream);
}

}  // namespace

Geometry make_geometry(int g) {
    Geometry geo;
    geo.g = g;
    geo.P = g / kPiece < 32 ? g / kPiece : 32;
    geo.NP = g / (kPiece * geo.P);
    int tg = kMaxTileElems / g;
    if (tg > kMaxTileGroups) tg = kMaxTileGroups;
    geo.tile_groups = tg;
    geo.tile_elems = tg * g;
    return geo;
}

WorkspaceLayout workspace_layout(int64_t G, int stop_mode, int zero_nbits) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    WorkspaceLayout l{};
    size_t off = 0;
    l.header = off;
    off += 256;
    l.minmax = off;
    off = up(off + sizeof(float) * 2 * kMaxPartials);
    l.tparts = off;
    off = up(off + sizeof(double) * 2 * kMaxPartials);
    const size_t Gs = static_cast<size_t>(G > 0 ? G : 0);
    l.zbest = off;
    if (zero_nbits == 8) off = up(off + 4 * Gs);
    l.t_s = l.t_is = l.t_z0 = l.t_sws = l.t_z = l.t_e = off;
    if (stop_mode == 1) {
        l.t_s = off;
        off = up(off + 4 * Gs);
        l.t_is = off;
        off = up(off + 4 * Gs);
        l.t_z0 = off;
        off = up(off + 4 * Gs);
        l.t_sws = off;
        off = up(off + 8 * Gs);
        l.t_z = off;
        off = up(off + 12 * Gs);
        l.t_e = off;
        off = up(off + 12 * Gs);
    }
    l.total = off;
    return l;
}

void set_barrier_debug(int skip_block, uint64_t timeout_ns) {
    g_skip_block = skip_block;
    g_timeout_ns = timeout_ns;
}

cudaError_t launch_solve(const SolveArgs& a, cudaStream_t stream, int* coop_unsupported) {
    *coop_unsupported = 0;
    const Geometry geo = make_geometry(a.g);
    const WorkspaceLayout L = workspace_layout(a.G, a.stop_mode, a.zero_nbits);
    KParams k{};
    k.W = static_cast<const uint16_t*>(a.W);
    k.rows = a.rows;
    k.cols = a.cols;
    k.G = a.G;
    k.g = a.g;
    k.P = geo.P;
    k.logP = 0;
    while ((1 << k.logP) < geo.P) ++k.logP;
    k.NP = geo.NP;
    k.tile_groups = geo.tile_groups;
    k.tile_elems = geo.tile_elems;
    k.nbits = a.nbits;
    k.iters = a.iters;
    k.iters_eff = a.iters > 0 ? a.iters : (a.dbg_err ? 1 : 0);  // iters 0 == 1: z* = z0 either way
    k.stop_mode = a.stop_mode;
    k.zero_nbits = a.zero_nbits;
    k.p = a.p;
    k.beta = a.beta;
    k.kappa = a.kappa;
    k.Lf = static_cast<float>((1 << a.nbits) - 1);
    if (a.axis == 1) {
        k.ncoltiles = 0;
        k.ntiles = (a.G + geo.tile_groups - 1) / geo.tile_groups;
    } else {
        k.ncoltiles = (a.cols + geo.tile_groups - 1) / geo.tile_groups;
        k.ntiles = (a.rows / a.g) * k.ncoltiles;
    }
    k.packed = a.packed;
    k.scale = a.scale;
    k.zero = a.zero;
    k.dbg_iter = a.dbg_iter;
    k.dbg_err = a.dbg_err;
    k.dbg_zero = a.dbg_zero;
    uint32_t* hdr = reinterpret_cast<uint32_t*>(a.ws + L.header);
    k.status = hdr;
    k.bar_count = hdr + 1;
    k.bar_gen = hdr + 2;
    k.minmax = reinterpret_cast<float2*>(a.ws + L.minmax);
    k.tparts = reinterpret_cast<double*>(a.ws + L.tparts);
    k.zbest_ws = a.zero_nbits == 8 ? reinterpret_cast<float*>(a.ws + L.zbest) : nullptr;
    if (a.stop_mode == 1) {
        k.t_s = reinterpret_cast<float*>(a.ws + L.t_s);
        k.t_is = reinterpret_cast<float*>(a.ws + L.t_is);
        k.t_z0 = reinterpret_cast<float*>(a.ws + L.t_z0);
        k.t_sws = reinterpret_cast<double*>(a.ws + L.t_sws);
        k.t_z = reinterpret_cast<float*>(a.ws + L.t_z);
        k.t_e = a.dbg_err ? reinterpret_cast<float*>(a.ws + L.t_e) : nullptr;
    }
    k.vec_ok = a.vec_ok ? 1 : 0;
    k.skip_block = g_skip_block;
    k.timeout_ns = g_timeout_ns ? g_timeout_ns : 4000000000ull;

    cudaError_t err = cudaMemsetAsync(a.ws + L.header, 0, 256, stream);
    if (err != cudaSuccess) return err;
    int grid = 0;
    if (a.G > 0) {
        if (a.dtype == 0 && a.axis == 1) err = launch_solve_t<0, 1>(k, stream, coop_unsupported, &grid);
        else if (a.dtype == 0) err = launch_solve_t<0, 0>(k, stream, coop_unsupported, &grid);
        else if (a.axis == 1) err = launch_solve_t<1, 1>(k, stream, coop_unsupported, &grid);
        else err = launch_solve_t<1, 0>(k, stream, coop_unsupported, &grid);
        if (err != cudaSuccess || *coop_unsupported) return err;
    }
    if (a.zero_nbits == 8) {
        int64_t blocks = (a.G + kThreads - 1) / kThreads;
        const int64_t cap = static_cast<int64_t>(device_info().sms) * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        zero_q8_kernel<<<static_cast<int>(blocks), kThreads, 0, stream>>>(
            k.zbest_ws, a.G, k.minmax, grid, static_cast<uint8_t*>(a.zero), a.zero_meta);
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
    int64_t blocks = (units + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(device_info().sms) * 16;
    if (blocks > cap) blocks = cap;
    const int nb = static_cast<int>(blocks);
    if (a.out_dtype == 0 && a.axis == 1) dequant_kernel<0, 1><<<nb, kThreads, 0, stream>>>(d);
    else if (a.out_dtype == 0) dequant_kernel<0, 0><<<nb, kThreads, 0, stream>>>(d);
    else if (a.axis == 1) dequant_kernel<1, 1><<<nb, kThreads, 0, stream>>>(d);
    else dequant_kernel<1, 0><<<nb, kThreads, 0, stream>>>(d);
    return cudaGetLastError();
}

}  // namespace hqq
