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

// ---------------------------------------------- 32-column chunks per lane --
//
// The common case (cols a multiple of 32, g >= 16, batch <= 2): a warp takes
// up to kWarpRows rows; each lane covers 32-column chunks (lane, lane + 32,
// ...), loads the chunk's 32 activations once (four 16-byte loads per vector)
// and uses them for all of the warp's rows; a row's 32 codes are nbits 32-bit
// words.  Codes become floats by a byte permute into the mantissa of 2^23 and
// one subtraction (about 2.4 instructions per code at 1, 2, 4 and 8 bits; a
// funnel shift at 3 bits).  Each row is reduced by one fixed shuffle tree.

constexpr int kWarpRows = 4;

// byte b of m placed in the low mantissa byte of 2^23: the float 2^23 + byte
__device__ __forceinline__ float byte_to_float(uint32_t m, int b) {
    return __fsub_rn(__uint_as_float(__byte_perm(m, 0x4B000000u, 0x7440u | static_cast<uint32_t>(b))), 8388608.0f);
}

// The 32 codes of a chunk (LSB first, NBITS words) as floats.
template <int NBITS>
__device__ __forceinline__ void chunk_codes(const uint32_t* w, float* q) {
    if (NBITS == 8) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int b = 0; b < 4; ++b) q[4 * k + b] = byte_to_float(w[k], b);
    } else if (NBITS == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = w[k] & 0x0F0F0F0Fu, hi = (w[k] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                q[8 * k + 2 * b] = byte_to_float(lo, b);
                q[8 * k + 2 * b + 1] = byte_to_float(hi, b);
            }
        }
    } else if (NBITS == 2) {
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t m = (w[k] >> (2 * t)) & 0x03030303u;
#pragma unroll
                for (int b = 0; b < 4; ++b) q[16 * k + 4 * b + t] = byte_to_float(m, b);
            }
    } else if (NBITS == 1) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t m = (w[0] >> t) & 0x01010101u;
#pragma unroll
            for (int b = 0; b < 4; ++b) q[8 * b + t] = byte_to_float(m, b);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int bit = NBITS * i, k = bit >> 5, off = bit & 31;
            const uint32_t v = (off + NBITS <= 32) ? (w[k] >> off) : __funnelshift_r(w[k], w[k + 1], off);
            q[i] = code_to_float(v & ((1u << NBITS) - 1u));
        }
    }
}

// GPC: quantisation groups per 32-column chunk (1 for g >= 32, 2 for g = 16).
// The NBITS words of a chunk's codes with the widest aligned loads.
template <int NBITS>
__device__ __forceinline__ void load_chunk_words(const uint8_t* p, uint32_t* w) {
    if (NBITS == 8) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(p)), b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if (NBITS == 4) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else if (NBITS == 2) {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = a.x; w[1] = a.y;
    } else {
#pragma unroll
        for (int k = 0; k < NBITS; ++k) w[k] = __ldg(reinterpret_cast<const uint32_t*>(p) + k);
    }
}

// One chunk's raw inputs for a warp's rows: activations, code words, scale
// and zero bits (loaded one chunk ahead of their use).
template <int NBITS, int B, int GPC>
struct ChunkRaw {
    uint4 x[B][4];
    uint32_t w[kWarpRows][NBITS];
    uint16_t sb[kWarpRows][GPC];
    uint16_t zb[kWarpRows][GPC];
};

template <int NBITS, int B, int GPC>
__device__ __forceinline__ void load_chunk(const GemvParams& p, int64_t r0, int nrows, int64_t ch, bool z8,
                                           ChunkRaw<NBITS, B, GPC>& c) {
    constexpr int GW = 32 / GPC;
#pragma unroll
    for (int b = 0; b < B; ++b) {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + b * p.cols + ch * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t) c.x[b][t] = __ldg(src + t);
    }
#pragma unroll
    for (int r = 0; r < kWarpRows; ++r) {
        if (r < nrows) {
            const int64_t e0 = (r0 + r) * p.cols + ch * 32;  // flat index of the chunk's first element
            load_chunk_words<NBITS>(p.packed + (e0 >> 3) * NBITS, c.w[r]);
#pragma unroll
            for (int gi = 0; gi < GPC; ++gi) {
                const int64_t j = (e0 + gi * GW) >> p.log_g;
                c.sb[r][gi] = __ldg(p.scale + j);
                c.zb[r][gi] = z8 ? __ldg(reinterpret_cast<const uint8_t*>(p.zero) + j)
                                 : __ldg(reinterpret_cast<const uint16_t*>(p.zero) + j);
            }
        }
    }
}

// Persistent: warps loop over tiles of rows_per_warp rows; within a tile each
// lane's chunks are software-pipelined (the next chunk's loads are in flight
// while the current one is computed).
// Two CTAs per SM (128 registers) where the pipelined state fits without
// spilling (1-4 bits, one group per chunk, one vector); one elsewhere.
template <int NBITS, int XDT, int B, int GPC>
__global__ void __launch_bounds__(kGemvThreads, (NBITS <= 4 && GPC == 1 && B == 1) ? 2 : 1)
    gemv_warp_kernel(const GemvParams p, int rows_per_warp) {
    constexpr int GW = 32 / GPC;  // columns per group within a chunk
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = p.cols >> 5;
    const bool z8 = p.zero_nbits == 8;
    const float zm0 = z8 ? p.zero_meta[0] : 0.0f, zm1 = z8 ? p.zero_meta[1] : 0.0f;
    const int64_t ntiles = (p.rows + rows_per_warp - 1) / rows_per_warp;
    const int64_t wstride = static_cast<int64_t>(gridDim.x) * (kGemvThreads / 32);
    for (int64_t tile = static_cast<int64_t>(blockIdx.x) * (kGemvThreads / 32) + (threadIdx.x >> 5); tile < ntiles;
         tile += wstride) {
        const int64_t r0 = tile * rows_per_warp;
        const int nrows = static_cast<int>(p.rows - r0 < rows_per_warp ? p.rows - r0 : rows_per_warp);
        float acc[kWarpRows][B];
#pragma unroll
        for (int r = 0; r < kWarpRows; ++r)
#pragma unroll
            for (int b = 0; b < B; ++b) acc[r][b] = 0.0f;
        ChunkRaw<NBITS, B, GPC> nxt;
        if (lane < nchunks) load_chunk<NBITS, B, GPC>(p, r0, nrows, lane, z8, nxt);
        for (int64_t ch = lane; ch < nchunks; ch += 32) {
            const ChunkRaw<NBITS, B, GPC> cur = nxt;
            if (ch + 32 < nchunks) load_chunk<NBITS, B, GPC>(p, r0, nrows, ch + 32, z8, nxt);
            float xv[B][32], sx[B][GPC];
#pragma unroll
            for (int b = 0; b < B; ++b) {
#pragma unroll
                for (int t = 0; t < 4; ++t) unpack8<XDT>(cur.x[b][t], xv[b] + 8 * t);
#pragma unroll
                for (int gi = 0; gi < GPC; ++gi) {
                    float t = 0.0f;
#pragma unroll
                    for (int i = 0; i < GW; ++i) t = __fadd_rn(t, xv[b][gi * GW + i]);
                    sx[b][gi] = t;
                }
            }
#pragma unroll
            for (int r = 0; r < kWarpRows; ++r) {
                if (r >= nrows) break;
                float q[32];
                chunk_codes<NBITS>(cur.w[r], q);
#pragma unroll
                for (int gi = 0; gi < GPC; ++gi) {
                    const float s = __half2float(__ushort_as_half(cur.sb[r][gi]));
                    const float z = z8 ? __fmul_rn(__fsub_rn(static_cast<float>(cur.zb[r][gi]), zm1), zm0)
                                       : __half2float(__ushort_as_half(cur.zb[r][gi]));
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        float d = 0.0f;
#pragma unroll
                        for (int i = 0; i < GW; ++i) d = __fmaf_rn(q[gi * GW + i], xv[b][gi * GW + i], d);
                        acc[r][b] = __fmaf_rn(s, __fmaf_rn(-z, sx[b][gi], d), acc[r][b]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kWarpRows; ++r)
#pragma unroll
            for (int b = 0; b < B; ++b) {
                float v = acc[r][b];
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
                if (lane == 0 && r < nrows && b < p.batch) p.y[b * p.rows + r0 + r] = v;
            }
    }
}

template <int NBITS, int XDT, int B>
cudaError_t launch_gemv_warp(const GemvParams& p, int g, cudaStream_t stream) {
    // 4 rows per warp (activations reused 4 times) when that still gives >= 8
    // warps per SM, else 1
    const int rpw = p.rows >= static_cast<int64_t>(kWarpRows) * 148 * 8 ? kWarpRows : 1;
    const int64_t warps = (p.rows + rpw - 1) / rpw;
    const int64_t ctas = (warps + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
    auto kern = g >= 32 ? gemv_warp_kernel<NBITS, XDT, B, 1> : gemv_warp_kernel<NBITS, XDT, B, 2>;
    int per_sm = 0, dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, 0);
    if (err != cudaSuccess) return err;
    const int64_t cap = static_cast<int64_t>(sms > 0 ? sms : 1) * (per_sm > 0 ? per_sm : 1);
    const unsigned grid = static_cast<unsigned>(ctas < cap ? ctas : cap);
    kern<<<grid, kGemvThreads, 0, stream>>>(p, rpw);
    return cudaGetLastError();
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
cudaError_t launch_gemv_x(int nbits, int g, const GemvParams& p, cudaStream_t stream) {
    if (p.cols % 32 == 0 && g >= 16 && p.batch <= 2) {  // 32-column chunks per lane
        switch (nbits) {
            case 1: return p.batch == 1 ? launch_gemv_warp<1, XDT, 1>(p, g, stream) : launch_gemv_warp<1, XDT, 2>(p, g, stream);
            case 2: return p.batch == 1 ? launch_gemv_warp<2, XDT, 1>(p, g, stream) : launch_gemv_warp<2, XDT, 2>(p, g, stream);
            case 3: return p.batch == 1 ? launch_gemv_warp<3, XDT, 1>(p, g, stream) : launch_gemv_warp<3, XDT, 2>(p, g, stream);
            case 4: return p.batch == 1 ? launch_gemv_warp<4, XDT, 1>(p, g, stream) : launch_gemv_warp<4, XDT, 2>(p, g, stream);
            default: return p.batch == 1 ? launch_gemv_warp<8, XDT, 1>(p, g, stream) : launch_gemv_warp<8, XDT, 2>(p, g, stream);
        }
    }
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
    return a.x_dtype == 0 ? launch_gemv_x<0>(a.nbits, a.g, p, stream) : launch_gemv_x<1>(a.nbits, a.g, p, stream);
}

}  // namespace hqq
