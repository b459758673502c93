// hqq_gemv.cu -- fused dequantisation + matrix-vector product of the packed
// layout (axis 1): y[b][r] = sum_c W_r[r][c] * x[b][c], W_r = (W_q - z) * scale.
//
// The step after quantisation: an inference backend dequantises W_q and
// multiplies (techreport.ngo, "Weight-only quantization without the
// calibration tax"; the dequantisation rule W_r = (W_q - z) * scale of section
// "Outlier-aware optimization without gradients").  For a batch of up to 8
// activation vectors this is HBM-bound: b/8 bytes of codes per weight plus
// 4/g of scale and zero, each weight used once.  No tensor cores: there is
// no contraction deep enough to feed them at batch <= 8.
//
// A CTA takes kGemvRows rows; its threads stride over 8-column pieces (one piece
// = nbits bytes of codes, always inside one quantisation group since g is a
// multiple of 8).  A thread loads the 8 activations of its piece once (16
// bytes per vector) and reuses them for the kGemvRows rows.  Within a piece the
// group's scale and zero are constant, so
//   sum_c (q_c - z) * s * x_c = s * (sum_c q_c * x_c - z * sum_c x_c),
// the same real number as the per-element form, in fp32 with one rounding
// fewer per element; a code q becomes a float by OR-ing it into the mantissa
// of 2^23 and subtracting 2^23 (integer-to-float conversion would issue on
// the XU pipe).  The per-thread sums are reduced in a fixed order, so the
// result does not depend on scheduling.

#include "hqq_device.cuh"

namespace hqq {
namespace {

using namespace dev;

constexpr int kGemvThreads = 256;
constexpr int kGemvRows = 4;

struct GemvParams {
    const uint8_t* packed;
    const uint16_t* scale;
    const void* zero;
    const float* zero_meta;
    const uint16_t* x;
    float* y;
    int64_t rows, cols;
    int log_g, zero_nbits, batch;
};

// The NBITS bytes of codes of piece pc (8 codes, LSB first).
template <int NBITS>
__device__ __forceinline__ uint64_t load_codes(const uint8_t* p) {
    if (NBITS == 8) return *reinterpret_cast<const uint64_t*>(p);
    if (NBITS == 4) return *reinterpret_cast<const uint32_t*>(p);
    if (NBITS == 2) return *reinterpret_cast<const uint16_t*>(p);
    if (NBITS == 1) return *p;
    return static_cast<uint64_t>(p[0]) | (static_cast<uint64_t>(p[1]) << 8) | (static_cast<uint64_t>(p[2]) << 16);
}

// q < 2^23 as a float: the bit pattern 0x4B000000 | q is 2^23 + q exactly.
__device__ __forceinline__ float code_to_float(uint32_t q) {
    return __fsub_rn(__uint_as_float(q | 0x4B000000u), 8388608.0f);
}

// Two pieces per thread and step: every load of both (codes, scale, zero of
// kGemvRows rows; activations) is issued before any is used.
constexpr int kUnroll = 2;

template <int NBITS, int XDT, int B>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvParams p) {
    constexpr uint32_t kMask = (1u << NBITS) - 1u;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kGemvRows;
    const int64_t npieces = p.cols / kPiece;
    const int nrows = static_cast<int>(p.rows - r0 < kGemvRows ? p.rows - r0 : kGemvRows);
    const bool z8 = p.zero_nbits == 8;
    const float zm0 = z8 ? p.zero_meta[0] : 0.0f, zm1 = z8 ? p.zero_meta[1] : 0.0f;
    float acc[kGemvRows][B];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[r][b] = 0.0f;

    for (int64_t pc0 = threadIdx.x; pc0 < npieces; pc0 += kGemvThreads * kUnroll) {
        uint64_t v[kUnroll][kGemvRows];
        uint16_t sb[kUnroll][kGemvRows];
        uint32_t zb[kUnroll][kGemvRows];
        uint4 xr[kUnroll][B];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t pc = pc0 + static_cast<int64_t>(u) * kGemvThreads;
            const bool ok = pc < npieces;
#pragma unroll
            for (int b = 0; b < B; ++b)
                xr[u][b] = (ok && b < p.batch) ? __ldg(reinterpret_cast<const uint4*>(p.x + b * p.cols) + pc)
                                               : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < kGemvRows; ++r) {
                v[u][r] = 0;
                sb[u][r] = 0;
                zb[u][r] = 0;
                if (ok && r < nrows) {
                    const int64_t e0 = (r0 + r) * p.cols + pc * kPiece;  // flat index of the piece's first element
                    const int64_t j = e0 >> p.log_g;
                    v[u][r] = load_codes<NBITS>(p.packed + (e0 >> 3) * NBITS);
                    sb[u][r] = __ldg(p.scale + j);
                    zb[u][r] = z8 ? __ldg(reinterpret_cast<const uint8_t*>(p.zero) + j)
                                  : __ldg(reinterpret_cast<const uint16_t*>(p.zero) + j);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float xv[B][kPiece], sx[B];
#pragma unroll
            for (int b = 0; b < B; ++b) {
                unpack8<XDT>(xr[u][b], xv[b]);
                float t = 0.0f;
#pragma unroll
                for (int i = 0; i < kPiece; ++i) t = __fadd_rn(t, xv[b][i]);
                sx[b] = t;
            }
#pragma unroll
            for (int r = 0; r < kGemvRows; ++r) {
                const float s = __half2float(__ushort_as_half(sb[u][r]));
                const float z = z8 ? __fmul_rn(__fsub_rn(static_cast<float>(zb[u][r]), zm1), zm0)
                                   : __half2float(__ushort_as_half(static_cast<uint16_t>(zb[u][r])));
                float q[kPiece];
#pragma unroll
                for (int i = 0; i < kPiece; ++i)
                    q[i] = code_to_float(static_cast<uint32_t>(v[u][r] >> (i * NBITS)) & kMask);
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    float d = 0.0f;
#pragma unroll
                    for (int i = 0; i < kPiece; ++i) d = __fmaf_rn(q[i], xv[b][i], d);
                    acc[r][b] = __fmaf_rn(s, __fmaf_rn(-z, sx[b], d), acc[r][b]);
                }
            }
        }
    }

    // fixed-order reduction: warps by shuffles, then the 8 warp sums in order
    __shared__ float red[kGemvThreads / 32][kGemvRows * B];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float v = acc[r][b];
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
            if (lane == 0) red[warp][r * B + b] = v;
        }
    __syncthreads();
    if (threadIdx.x < kGemvRows * B) {
        const int r = threadIdx.x / B, b = threadIdx.x % B;
        const int64_t row = r0 + r;
        if (row < p.rows && b < p.batch) {
            float v = 0.0f;
            for (int w = 0; w < kGemvThreads / 32; ++w) v += red[w][threadIdx.x];
            p.y[b * p.rows + row] = v;
        }
    }
}

template <int NBITS, int XDT>
cudaError_t launch_gemv_b(const GemvParams& p, cudaStream_t stream) {
    const int64_t ctas = (p.rows + kGemvRows - 1) / kGemvRows;
    const unsigned grid = static_cast<unsigned>(ctas);
    if (p.batch <= 1) gemv_kernel<NBITS, XDT, 1><<<grid, kGemvThreads, 0, stream>>>(p);
    else if (p.batch <= 2) gemv_kernel<NBITS, XDT, 2><<<grid, kGemvThreads, 0, stream>>>(p);
    else if (p.batch <= 4) gemv_kernel<NBITS, XDT, 4><<<grid, kGemvThreads, 0, stream>>>(p);
    else gemv_kernel<NBITS, XDT, 8><<<grid, kGemvThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int XDT>
cudaError_t launch_gemv_x(int nbits, const GemvParams& p, cudaStream_t stream) {
    switch (nbits) {
        case 1: return launch_gemv_b<1, XDT>(p, stream);
        case 2: return launch_gemv_b<2, XDT>(p, stream);
        case 3: return launch_gemv_b<3, XDT>(p, stream);
        case 4: return launch_gemv_b<4, XDT>(p, stream);
        default: return launch_gemv_b<8, XDT>(p, stream);
    }
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t stream) {
    if (a.rows == 0) return cudaSuccess;
    GemvParams p;
    p.packed = a.packed;
    p.scale = a.scale;
    p.zero = a.zero;
    p.zero_meta = a.zero_meta;
    p.x = static_cast<const uint16_t*>(a.x);
    p.y = a.y;
    p.rows = a.rows;
    p.cols = a.cols;
    p.log_g = 0;
    while ((1 << p.log_g) < a.g) ++p.log_g;  // g is a power of two
    p.zero_nbits = a.zero_nbits;
    p.batch = a.batch;
    return a.x_dtype == 0 ? launch_gemv_x<0>(a.nbits, p, stream) : launch_gemv_x<1>(a.nbits, p, stream);
}

}  // namespace hqq
