// hqq_device.cuh -- device-side building blocks shared by the solver kernels.
//
// Method: techreport.ngo, "Weight-only quantization without the calibration
// tax" (Half-Quadratic Quantization of Large Machine Learning Models), section
// "Outlier-aware optimization without gradients".  Per element, with
// ws = fl(w*s) and v = fl(ws + z):
//   W_q = clamp(round_half_even(v), 0, L)
//   r   = v - W_q                      (exact in fp32)
//   W - W_r = W - (W_q - z)/s = r/s    so |W - W_r|^p = |r|^p * s^-p
// The group sums are sum |r|^p (MUFU lg2/ex2), sum W_q (exact: integers) and,
// precomputed once per group, sum fl(w*s) in fp64; the zero update is
// z' = (sum W_q - sum fl((w - W_e)*s)) / g, which equals sum W_q - sum ws when
// the proximal step W_e is zero for the whole group.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include <cfloat>
#include <cstdint>

#include "hqq_internal.h"

namespace hqq {
namespace dev {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kMagic = 12582912.0f;        // 1.5 * 2^23: adding it rounds to an integer
constexpr uint32_t kMagicBits = 0x4B400000u;  // bit pattern of kMagic

// ------------------------------------------------------------ math ------

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

// a^e for a >= 0 through the hardware base-2 log and exponential (0^e = 0, e > 0).
__device__ __forceinline__ float pow_pos(float a, float e) { return ex2_approx(e * lg2_approx(a)); }

// beta^(-1/(2-p)): |d| at or below it gives a proximal step of exactly 0.
__device__ __forceinline__ float shrink_threshold(float beta, float p) {
    return ex2_approx(-lg2_approx(beta) / (2.0f - p));
}

// round_half_even(clamp(v, 0, L)) == clamp(round_half_even(v), 0, L) for
// integer bounds; adding 1.5*2^23 rounds to nearest-even exactly for
// |x| < 2^22, and the integer code is read from the sum's low mantissa bits.
__device__ __forceinline__ float round_clamp(float v, float Lf, uint32_t* code) {
    const float t = __fadd_rn(fminf(fmaxf(v, 0.0f), Lf), kMagic);
    *code = __float_as_uint(t) - kMagicBits;
    return __fsub_rn(t, kMagic);
}

// One element of one evaluation: ws = fl(w*s) precomputed.
struct ElemEval {
    float v, q, r;
    uint32_t code;
};
__device__ __forceinline__ ElemEval eval_elem(float ws, float z, float Lf) {
    ElemEval e;
    e.v = __fadd_rn(ws, z);
    e.q = round_clamp(e.v, Lf, &e.code);
    e.r = __fsub_rn(e.v, e.q);
    return e;
}

// Same without the clamp: exact when every v of the group lies in
// [-0.5, L + 0.5), where round-half-even(v) is already in [0, L].
__device__ __forceinline__ ElemEval eval_elem_nc(float ws, float z) {
    ElemEval e;
    e.v = __fadd_rn(ws, z);
    const float t = __fadd_rn(e.v, kMagic);
    e.code = __float_as_uint(t) - kMagicBits;
    e.q = __fsub_rn(t, kMagic);
    e.r = __fsub_rn(e.v, e.q);
    return e;
}

// ---- packed fp32 pairs (add/sub/mul .rn.f32x2: two IEEE fp32 operations,
// each rounded exactly as the scalar one, in one instruction) ----

__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The fast-path sums of one evaluation over a lane's E elements (E a multiple
// of 4, every v clamp-free): sum |r|^p and sum W_q, with v, t, q, r, p*lg2|r|
// formed pairwise by packed fp32 operations -- the same values as
// eval_elem_nc.  The error is accumulated one element at a time in element
// order: the stop decisions compare these sums, and this order agrees with
// the oracle's decisions at near ties more often than reordered partial sums
// do (measured: with four interleaved partial sums, 7 of 4,800 groups kept
// another iterate than the oracle in a 20-iteration no-stop run, against at
// most 1 in element order).  Sum W_q is exact in any order (integers), so it
// runs in two packed partial sums.
template <int E>
__device__ __forceinline__ void fast_sums(const float* ws, float z, float p, float* err_out, float* sq_out) {
    static_assert(E % 4 == 0, "two packed partial sums");
    const uint64_t z2 = f2_pack(z, z), m2 = f2_pack(kMagic, kMagic), p2 = f2_pack(p, p);
    uint64_t sq[2] = {f2_pack(0.0f, 0.0f), f2_pack(0.0f, 0.0f)};
    float err = 0.0f;
#pragma unroll
    for (int i = 0; i < E; i += 2) {
        const uint64_t v = f2_add(f2_pack(ws[i], ws[i + 1]), z2);
        const uint64_t q = f2_sub(f2_add(v, m2), m2);  // round half to even: fl(fl(v + M) - M)
        const uint64_t r = f2_sub(v, q);
        float r0, r1;
        f2_unpack(r, r0, r1);
        float l0, l1;
        f2_unpack(f2_mul(f2_pack(lg2_approx(fabsf(r0)), lg2_approx(fabsf(r1))), p2), l0, l1);
        err = __fadd_rn(__fadd_rn(err, ex2_approx(l0)), ex2_approx(l1));
        sq[(i >> 1) & 1] = f2_add(sq[(i >> 1) & 1], q);
    }
    float s0, s1;
    f2_unpack(f2_add(sq[0], sq[1]), s0, s1);
    *err_out = err;
    *sq_out = __fadd_rn(s0, s1);
}

// True when no v = fl(ws + z) of a set with ws in [wsmin, wsmax] needs the
// clamp (fl(. + z) is monotone, so the extremes decide).
__device__ __forceinline__ bool clamp_free(float wsmin, float wsmax, float z, float Lf) {
    return __fadd_rn(wsmin, z) >= -0.5f && __fadd_rn(wsmax, z) < Lf + 0.5f;
}

// Proximal step of the lp term for one element: d = r/s, W_e = shrink(d).
__device__ __forceinline__ float shrink_elem(float r, float s, float p, float beta) {
    const float d = __fdiv_rn(r, s);
    const float a = fabsf(d);
    if (a == 0.0f) return 0.0f;
    const float t = __fsub_rn(a, __fdiv_rn(pow_pos(a, p - 1.0f), beta));
    return t > 0.0f ? copysignf(t, d) : 0.0f;
}

// |w - W_r| * s <= max(0.5, |z - z0|) + rounding for every element of a
// group (v spans [z - z0, L + z - z0] up to rounding), so the proximal step
// is zero for the whole group unless this bound reaches thr * s.
__device__ __forceinline__ bool shrink_possible(float s, float z, float z0, float thr, float Lf) {
    return fmaxf(0.5f, fabsf(z - z0)) + 1e-3f * (1.0f + Lf + fabsf(z)) >= 0.99f * thr * s;
}

__device__ __forceinline__ float zero_from_sums(float sq, double sws, int g) {
    return static_cast<float>((static_cast<double>(sq) - sws) / static_cast<double>(g));
}

// A double split into two floats, hi = fl32(x), lo = fl32(x - hi).
struct F2 {
    float hi, lo;
};
__device__ __forceinline__ F2 split_f2(double x) {
    F2 r;
    r.hi = static_cast<float>(x);
    r.lo = static_cast<float>(x - static_cast<double>(r.hi));
    return r;
}

// zero_from_sums in fp32 only: (sq - hi) is formed exactly by TwoSum, the
// small remainder (e - lo) is added once, and the single rounding of that sum
// gives fl32(sq - sws) (ties aside), which is exact after scaling by 1/g (a
// power of two).  Short dependency chain: no fp64 conversions.
__device__ __forceinline__ float zero_from_sums_f2(float sq, F2 sws, float inv_g) {
    const float d = __fsub_rn(sq, sws.hi);
    const float bp = __fsub_rn(d, sq);
    const float e = __fadd_rn(__fsub_rn(sq, __fsub_rn(d, bp)), __fsub_rn(-sws.hi, bp));
    return __fmul_rn(__fadd_rn(d, __fsub_rn(e, sws.lo)), inv_g);
}

// ------------------------------------------------------ reductions -------

// Over P consecutive lanes (P a power of two <= 32); all lanes of the segment
// get the same value.
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

// --------------------------------------------------------- elements ------

template <int DT>
__device__ __forceinline__ float bits_to_float(uint32_t b16) {
    if (DT == 0) return __half2float(__ushort_as_half(static_cast<unsigned short>(b16)));
    return __uint_as_float(b16 << 16);
}

// Eight 16-bit elements held in a uint4 -> fp32.
template <int DT>
__device__ __forceinline__ void unpack8(const uint4 u, float* w) {
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

__device__ __forceinline__ uint16_t half_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

}  // namespace dev

// Kernel parameters shared by the solver kernels (passed by value).
struct KParams {
    const uint16_t* W;
    int64_t rows, cols, G;
    int g, P, logP, E, nbits, iters, iters_eff, stop_mode, zero_nbits, axis;
    float p, beta, kappa, Lf;
    float beta_last;     // beta of the last iteration (sequential fp32 products)
    int64_t n;  // rows * cols
    uint8_t* packed;
    uint16_t* scale;
    void* zero;
    int32_t* dbg_iter;
    float* dbg_err;
    float* dbg_zero;
    // workspace
    uint32_t* counters;  // workspace header words (status, CTA ticket, zero range, pass counts)
    double* tparts;      // per-iteration per-CTA tensor error partials [iters][kMaxPartials]
    double* etot;        // per-iteration tensor mean error [iters]
    float* zbest_ws;     // fp32 kept zero (8-bit zero path)
    float* t_s;          // tensor state: s, z0, sum ws, chunk-start zeros (ring of 3)
    float* t_z0;
    double* t_sws;
    float* t_zs;
};

}  // namespace hqq
