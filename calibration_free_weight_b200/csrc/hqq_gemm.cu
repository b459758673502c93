// hqq_gemm.cu -- fused dequantisation + matrix product on the 5th-generation
// tensor cores (tcgen05), the consumer of the packed layout for batches of
// activation vectors (an inference backend's role: "HQQ - Half-Quadratic
// Quantization" (skill4agent.com), section "Backends"):
//   y[b][r] = sum_c round16(W_r[r][c]) * x[b][c],
//   W_r = (W_q - zero) * scale formed in fp32 (techreport.ngo, "Weight-only
//   quantization without the calibration tax", section "Outlier-aware
//   optimization without gradients"), rounded to the activations' 16-bit type
//   (round to nearest even: both operands of one tcgen05 kind::f16 product
//   share a type), accumulated in fp32 in tensor memory.
//
// One CTA computes a 128-row x N tile of y^T (N = the batch tile, a multiple
// of 16 up to 256): A = W_r[128 rows][K] and B = x[N][K], both K-major, so the
// weight side fills the MMA's M = 128 and the (small) batch is the MMA's N.
// K is walked in 64-element tiles through a ring of S shared-memory
// stages, each in the canonical 128-byte-swizzled K-major layout (row r of a
// tile at r * 128 bytes, its 16-byte chunk c at chunk c ^ (r % 8)):
//   * 16 producer warps dequantise, 16 weights of the A tile per thread
//     (codes, scales and zeros prefetched in registers three tiles ahead),
//     store them as 16-bit values and arrive on the stage's "A full" mbarrier;
//   * one thread of a 17th warp issues the x tile's 2-D tensor copy (TMA,
//     128-byte swizzle, from this GPU's own memory, into this CTA only) S - 2 tiles
//     ahead, completing on the stage's "x full" mbarrier (rows past the batch
//     are zero-filled by the copy), and, once both halves of a stage are full,
//     four tcgen05.mma (K = 16 each) into the fp32 accumulator in tensor
//     memory, committed to the stage's "empty" mbarrier, which frees the
//     stage for the tile S later.
// The epilogue reads the accumulator with tcgen05.ld (producer warp w reads
// the 32 rows of its lane quarter w % 4, every fourth 8-column chunk) and
// stores y.
//
// Waits: every mbarrier wait gives up after ~1 s of global time, records a
// timeout in a device status word (read by hqq_gemm_get_status) and makes the
// whole CTA skip to the release of its tensor memory; no wait can hang.

#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched at run time; no driver library link)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "hqq_internal.h"

namespace {

constexpr int kWpt = 16;                      // weights per producer thread per K tile (two 8-weight pieces)
constexpr int kPieces = kWpt / 8;
constexpr int kProducers = 128 * 64 / kWpt;   // 512 threads, 16 warps: dequantisation
constexpr int kThreads = kProducers + 32;     // + 1 warp: tensor copies and MMA issue
constexpr int kTileM = 128;          // MMA M: weight rows per CTA
constexpr int kTileK = 64;           // elements per K tile: one 128-byte swizzle row of 16-bit values
constexpr int kMaxStages = 8;        // shared-memory ring: as many stages as fit (4 at N = 256, 8 at N <= 48)
constexpr size_t kSmemBudget = 227 * 1024;
constexpr int kStageA = kTileM * 128;  // bytes of one A stage
constexpr unsigned long long kWaitNs = 1000000000ull;

__device__ unsigned int g_gemm_status;  // 0, or 1 after a wait timed out

// ------------------------------------------------------------ PTX -------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Completion of the phase with this parity; false once the CTA's abort flag
// is set or after limit_ns (which sets the flag, so the other roles give up
// their waits too).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitNs) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_test(bar, parity)) {
        if (*abort_flag) return false;
        if (global_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 2-D tiled tensor copy global -> shared (box of the tensor map at {x0, y0}),
// completing on `bar` by transaction bytes.  x0 * 2 bytes is a multiple of 16.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x0, int y0, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x0), "r"(y0), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: 128-byte swizzle, K-major, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset 16 (unused by
// this layout), descriptor version 1, start address in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    return (static_cast<uint64_t>((addr >> 4) & 0x3FFFu)) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B of one
// 16-bit type (0 fp16, 1 bf16), both K-major, N / 8 and M / 16.
__host__ __device__ constexpr uint32_t instr_desc(int n, int bf16) {
    return (1u << 4) | (static_cast<uint32_t>(bf16) << 7) | (static_cast<uint32_t>(bf16) << 10) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kTileM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------ tiles -----

struct GemmParams {
    const uint8_t* packed;
    const uint16_t* scale;
    const void* zero;
    const float* zero_meta;
    const uint16_t* x;  // [batch][cols]
    float* y;           // [batch][rows]
    int64_t rows, cols;
    int g_log;          // log2(group size)
    int batch;
    int ntile;          // MMA N: batch rows per CTA, a multiple of 16 in [16, 256]
    int stages;         // S, in [3, kMaxStages]
    int splits;         // K splits (grid z); 1: each CTA writes y directly
    int kps;            // K tiles per split
    float* part;        // splits > 1: [tile][split][ntile][128] fp32 partial tiles
    uint32_t* tickets;  // splits > 1: [tile] arrival counts, zero at launch
};

// Inputs of one thread's kWpt consecutive weights of one K tile (one row):
// the codes as a little-endian bit stream (weight e at bit e * NBITS) and the
// scale and zero of each 8-weight piece.  Loaded ahead of use.
template <int NBITS>
struct ARaw {
    static constexpr int kWords = (kWpt * NBITS + 31) / 32;
    uint32_t w[kWords];
    float s[kPieces], z[kPieces];
};

__device__ __forceinline__ float half_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

template <int NBITS, int ZB>
__device__ __forceinline__ void load_a(const GemmParams& p, int64_t row, int64_t c0, ARaw<NBITS>& a) {
    if (row >= p.rows) {  // rows past the matrix: W_r = (0 - 0) * 0
#pragma unroll
        for (int i = 0; i < ARaw<NBITS>::kWords; ++i) a.w[i] = 0u;
#pragma unroll
        for (int i = 0; i < kPieces; ++i) a.s[i] = a.z[i] = 0.0f;
        return;
    }
    const int64_t e0 = row * p.cols + c0;  // first weight, a multiple of 16: its codes start on 2 * NBITS bytes
    const uint8_t* src = p.packed + (e0 / 16) * (2 * NBITS);
    if (NBITS == 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
        a.w[0] = v.x;
        a.w[1 % ARaw<NBITS>::kWords] = v.y;
        a.w[2 % ARaw<NBITS>::kWords] = v.z;
        a.w[3 % ARaw<NBITS>::kWords] = v.w;
    } else if (NBITS == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
        a.w[0] = v.x;
        a.w[1 % ARaw<NBITS>::kWords] = v.y;
    } else if (NBITS == 2) {
        a.w[0] = __ldg(reinterpret_cast<const uint32_t*>(src));
    } else if (NBITS == 1) {
        a.w[0] = __ldg(reinterpret_cast<const uint16_t*>(src));
    } else {  // 3 bits: 6 bytes on a 2-byte boundary
        const uint16_t* h = reinterpret_cast<const uint16_t*>(src);
        a.w[0] = static_cast<uint32_t>(__ldg(h)) | (static_cast<uint32_t>(__ldg(h + 1)) << 16);
        a.w[1 % ARaw<NBITS>::kWords] = __ldg(h + 2);
    }
    // one group for both pieces when g >= 16, else one per piece
    const int npc = p.g_log >= 4 ? 1 : kPieces;
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
        if (q < npc) {
            const int64_t j = (e0 + 8 * q) >> p.g_log;
            a.s[q] = half_to_float(__ldg(p.scale + j));
            if (ZB == 16) {
                a.z[q] = half_to_float(__ldg(reinterpret_cast<const uint16_t*>(p.zero) + j));
            } else {
                const float zq = static_cast<float>(__ldg(reinterpret_cast<const uint8_t*>(p.zero) + j));
                a.z[q] = __fmul_rn(__fsub_rn(zq, __ldg(p.zero_meta + 1)), __ldg(p.zero_meta));
            }
        } else {
            a.s[q] = a.s[0];
            a.z[q] = a.z[0];
        }
    }
}

// Code e of the bit stream (e a constant once the callers' loops unroll, so
// the word index and shifts fold and w stays in registers).
template <int NBITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t* w, int e) {
    const int b = e * NBITS, word = b / 32, off = b % 32;
    constexpr uint32_t mask = (1u << NBITS) - 1u;
    uint32_t v = w[word] >> off;
    if (off + NBITS > 32) v |= w[(word + 1) % ARaw<NBITS>::kWords] << (32 - off);
    return v & mask;
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if (BF16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t*>(&v);
    }
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// The 8 codes of piece P as the bit patterns of 2^23 + code (an exact float):
// byte-sized fields are moved into the mantissa by one byte permute each.
template <int NBITS, int P>
__device__ __forceinline__ void piece_codes_f(const uint32_t* w, uint32_t* f) {
    if (NBITS == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = __byte_perm(w[2 * P + i / 4], 0x4B00u, 0x5440u | (i % 4));
    } else if (NBITS == 4) {
        const uint32_t lo = w[P] & 0x0F0F0F0Fu, hi = (w[P] >> 4) & 0x0F0F0F0Fu;  // codes 0,2,4,6 and 1,3,5,7
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __byte_perm(lo, 0x4B00u, 0x5440u | i);
            f[2 * i + 1] = __byte_perm(hi, 0x4B00u, 0x5440u | i);
        }
    } else if (NBITS == 2) {
        const uint32_t h = w[P / 2] >> (16 * (P % 2));  // 8 codes in 16 bits
        const uint32_t t0 = h & 0x0303u, t1 = (h >> 2) & 0x0303u, t2 = (h >> 4) & 0x0303u, t3 = (h >> 6) & 0x0303u;
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // byte i of t_k holds code 4i + k
            f[4 * i] = __byte_perm(t0, 0x4B00u, 0x5440u | i);
            f[4 * i + 1] = __byte_perm(t1, 0x4B00u, 0x5440u | i);
            f[4 * i + 2] = __byte_perm(t2, 0x4B00u, 0x5440u | i);
            f[4 * i + 3] = __byte_perm(t3, 0x4B00u, 0x5440u | i);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0x4B000000u | code_at<NBITS>(w, 8 * P + i);
    }
}

// Packed fp32 pairs: two IEEE fp32 operations, each rounded as the scalar
// one, per instruction.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
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

template <int NBITS, bool BF16, int P>
__device__ __forceinline__ void piece_to_smem(const ARaw<NBITS>& a, uint32_t dst) {
    uint32_t f[8], v[4];
    piece_codes_f<NBITS, P>(a.w, f);
    const uint64_t two23 = f2_pack(8388608.0f, 8388608.0f), z2 = f2_pack(a.z[P], a.z[P]),
                   s2 = f2_pack(a.s[P], a.s[P]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // (q - z) * s for a pair of weights, q = (2^23 + q) - 2^23 exactly
        const uint64_t q = f2_sub(f2_pack(__uint_as_float(f[2 * i]), __uint_as_float(f[2 * i + 1])), two23);
        float w0, w1;
        f2_unpack(f2_mul(f2_sub(q, z2), s2), w0, w1);
        v[i] = pack2<BF16>(w0, w1);
    }
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

// W_r of this thread's kWpt weights, rounded to 16 bits, into row r, chunks
// kPieces*h .. kPieces*h + kPieces-1 of an A stage (128-byte swizzle: chunk c of
// row r at c ^ (r % 8)).
template <int NBITS, bool BF16>
__device__ __forceinline__ void store_a(const ARaw<NBITS>& a, uint32_t stage, int r, int h) {
    static_assert(kPieces == 2, "two pieces per thread");
    const uint32_t row = stage + static_cast<uint32_t>(r) * 128u;
    const int sw = r & 7;
    piece_to_smem<NBITS, BF16, 0>(a, row + ((((kPieces * h) + 0) ^ sw) << 4));
    piece_to_smem<NBITS, BF16, 1>(a, row + ((((kPieces * h) + 1) ^ sw) << 4));
}

__host__ __device__ constexpr uint32_t tmem_columns(int ntile) {
    return ntile <= 32 ? 32u : ntile <= 64 ? 64u : ntile <= 128 ? 128u : 256u;
}

__host__ __device__ constexpr size_t gemm_smem_bytes(int ntile, int stages) {
    // 1024 bytes of slack to align the stages to the 1024-byte swizzle period
    return 1024 + static_cast<size_t>(stages) * (kStageA + static_cast<size_t>(ntile) * 128) + 3 * stages * 8 + 16;
}

// As many stages as the shared memory holds (the x tiles are then issued
// S - 2 tiles ahead).
int gemm_stages(int ntile) {
    int st = kMaxStages;
    while (st > 3 && gemm_smem_bytes(ntile, st) > kSmemBudget) --st;
    return st;
}

template <int NBITS, bool BF16, int ZB>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const GemmParams p, const __grid_constant__ CUtensorMap xmap) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* const smem = smem_raw + (base - smem_u32(smem_raw));
    const int S = p.stages;
    const uint32_t sA = base;                                               // S x 16 KB
    const uint32_t sB = sA + S * kStageA;                                   // S x ntile x 128 B
    const uint32_t bars = sB + S * static_cast<uint32_t>(p.ntile) * 128u;  // S "stage empty" (MMAs done)
    const uint32_t xbars = bars + S * 8;                                    // S "x full" (tensor copy landed)
    const uint32_t abars = xbars + S * 8;                                   // S "A full" (producers done)
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + (abars + S * 8 - base));
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTileM, n0 = static_cast<int64_t>(blockIdx.y) * p.ntile;
    // this CTA's K tiles: [kbase, kbase + num_k) of the split blockIdx.z
    const int kbase = static_cast<int>(blockIdx.z) * p.kps;
    const int ktot = static_cast<int>(p.cols / kTileK);
    const int num_k = min(p.kps, ktot - kbase);
    const uint32_t ncols = tmem_columns(p.ntile);
    auto bar = [&](int s) { return bars + 8u * static_cast<uint32_t>(s); };
    auto xbar = [&](int s) { return xbars + 8u * static_cast<uint32_t>(s); };
    auto abar = [&](int s) { return abars + 8u * static_cast<uint32_t>(s); };
    const uint32_t xbytes = static_cast<uint32_t>(p.ntile) * 128u;
    auto stage_a = [&](int s) { return sA + static_cast<uint32_t>(s) * kStageA; };
    auto stage_b = [&](int s) { return sB + static_cast<uint32_t>(s) * static_cast<uint32_t>(p.ntile) * 128u; };

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar(s), 1);
            mbar_init(xbar(s), 1);
            mbar_init(abar(s), kProducers);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = instr_desc(p.ntile, BF16 ? 1 : 0);

    bool ok = true;
    if (warp < kProducers / 32) {
        // producers: row r of the A tile, weights [16h, 16h + 16) of each K
        // tile; codes, scales and zeros of tiles kt+1 .. kt+3 in flight in
        // registers (global latency hidden behind three tiles of work)
        const int r = tid >> 2, h = tid & 3;
        const int64_t row = m0 + r;
        auto col = [&](int kt) { return static_cast<int64_t>(kbase + kt) * kTileK + kWpt * h; };
        ARaw<NBITS> a0, a1, a2;
        load_a<NBITS, ZB>(p, row, col(0), a0);
        if (num_k > 1) load_a<NBITS, ZB>(p, row, col(1), a1);
        if (num_k > 2) load_a<NBITS, ZB>(p, row, col(2), a2);
        int s = 0, ph = 0;  // stage of tile kt and the parity of its use of that stage
#pragma unroll 4
        for (int kt = 0; kt < num_k; ++kt) {
            ARaw<NBITS> a3;
            if (kt + 3 < num_k) load_a<NBITS, ZB>(p, row, col(kt + 3), a3);
            // the stage is free once the MMAs of its previous use (tile kt-S) are done
            if (kt >= S && !mbar_wait(bar(s), static_cast<uint32_t>(ph ^ 1), abort_flag)) {
                ok = false;
                break;
            }
            store_a<NBITS, BF16>(a0, stage_a(s), r, h);
            fence_async_smem();  // generic-proxy shared-memory writes -> visible to the tensor core
            mbar_arrive(abar(s));
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
            a0 = a1;
            a1 = a2;
            a2 = a3;
        }
    } else if (lane == 0) {
        // tensor copies of x (kPB = S - 2 tiles ahead) and the MMAs
        const int kPB = S - 2;
        for (int d = 0; d < kPB && d < num_k; ++d) {
            mbar_expect_tx(xbar(d), xbytes);
            tma_load_2d(stage_b(d), &xmap, (kbase + d) * kTileK, static_cast<int>(n0), xbar(d));
        }
        int s = 0, ph = 0, sb = kPB, phb = 0, sl = 0, phl = 0;
        for (int kt = 0; kt < num_k && ok; ++kt) {
            const int kb = kt + kPB;  // its stage is free once the MMAs of tile kb-S (issued two tiles ago) are done
            if (kb < num_k) {
                if (kb >= S && !mbar_wait(bar(sb), static_cast<uint32_t>(phb ^ 1), abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(xbar(sb), xbytes);
                tma_load_2d(stage_b(sb), &xmap, (kbase + kb) * kTileK, static_cast<int>(n0), xbar(sb));
            }
            if (!mbar_wait(abar(s), static_cast<uint32_t>(ph), abort_flag) ||
                !mbar_wait(xbar(s), static_cast<uint32_t>(ph), abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < kTileK / 16; ++j)
                mma_f16(tmem, smem_desc(stage_a(s) + 32u * j), smem_desc(stage_b(s) + 32u * j), idesc,
                        (kt | j) != 0 ? 1u : 0u);
            mma_commit(bar(s));
            sl = s;
            phl = ph;
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
            if (++sb == S) {
                sb = 0;
                phb ^= 1;
            }
        }
        // the last commit covers every MMA of this CTA
        if (ok && !mbar_wait(bar(sl), static_cast<uint32_t>(phl), abort_flag)) ok = false;
    }
    if (!ok) *abort_flag = 1;
    __syncthreads();  // the MMA thread has seen its last commit complete (or someone gave up)
    ok = !*abort_flag;
    if (ok && warp < kProducers / 32) {
        tc_fence_after();
        // warp w reads lane quarter w % 4 (rows 32q .. 32q+31), every
        // (kProducers/128)-th 8-column chunk from chunk w / 4
        constexpr int kColWarps = kProducers / 128;
        const int q = warp & 3;
        const int64_t orow = m0 + 32 * q + lane;
        const int64_t tile = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        float* const mine = p.splits > 1 ? p.part + (tile * p.splits + blockIdx.z) * p.ntile * kTileM : nullptr;
        for (int c0 = 8 * (warp >> 2); c0 < p.ntile; c0 += 8 * kColWarps) {
            float v[8];
            tmem_ld8(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0), v);
            if (mine) {  // this split's partial tile, column-major, rows contiguous
#pragma unroll
                for (int i = 0; i < 8; ++i) __stcg(mine + (c0 + i) * kTileM + 32 * q + lane, v[i]);
            } else if (orow < p.rows) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t b = n0 + c0 + i;
                    if (b < p.batch) p.y[b * p.rows + orow] = v[i];
                }
            }
        }
    } else if (tid == 0) {
        atomicExch(&g_gemm_status, 1u);
    }
    if (p.splits > 1) {
        // The last split of this tile to arrive sums the partials in split
        // order (deterministic).  The ticket counts arrivals in its low 16 bits
        // and splits that gave up a wait in its high bits; if any did, a
        // partial is missing and the tile of y is filled with NaN instead.
        __shared__ int last, torn;
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const int64_t tile = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
            const uint32_t inc = *abort_flag ? (1u << 16) + 1u : 1u;
            const uint32_t old = atomicAdd(p.tickets + tile, inc);
            last = (old & 0xffffu) == static_cast<uint32_t>(p.splits - 1);
            torn = (old >> 16) != 0u || *abort_flag;
        }
        __syncthreads();
        if (last) {
            __threadfence();
            const int64_t tile = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
            const float* const base = p.part + tile * p.splits * p.ntile * kTileM;
            for (int e = tid; e < p.ntile * kTileM; e += kThreads) {
                const int c = e / kTileM, rr = e % kTileM;
                const int64_t orow = m0 + rr, b = n0 + c;
                float acc = __int_as_float(0x7fc00000);  // NaN
                if (!torn) {
                    acc = 0.0f;
                    for (int z = 0; z < p.splits; ++z)
                        acc = __fadd_rn(acc, __ldcg(base + z * p.ntile * kTileM + e));
                }
                if (orow < p.rows && b < p.batch) p.y[b * p.rows + orow] = acc;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
    }
}

// Diagnostic: the product's bounded wait on an mbarrier that nothing arrives
// on, with a short limit; it gives up and records the timeout exactly as the
// product does.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait(smem_u32(&bar), 0u, &abort_flag, limit_ns)) atomicExch(&g_gemm_status, 1u);
}

template <int NBITS, bool BF16, int ZB>
cudaError_t launch_t(const GemmParams& p, const CUtensorMap& xmap, dim3 grid, size_t smem, cudaStream_t stream) {
    auto kern = gemm_kernel<NBITS, BF16, ZB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(p, xmap);
    return cudaGetLastError();
}

template <int NBITS>
cudaError_t launch_n(const GemmParams& p, const CUtensorMap& xmap, bool bf16, int zb, dim3 grid, size_t smem,
                     cudaStream_t stream) {
    if (bf16) return zb == 8 ? launch_t<NBITS, true, 8>(p, xmap, grid, smem, stream)
                             : launch_t<NBITS, true, 16>(p, xmap, grid, smem, stream);
    return zb == 8 ? launch_t<NBITS, false, 8>(p, xmap, grid, smem, stream)
                   : launch_t<NBITS, false, 16>(p, xmap, grid, smem, stream);
}

// The driver's tensor-map encoder, fetched once through the runtime (the
// library links no driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            f = nullptr;
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// x [batch][cols] as a 2-D tensor (cols innermost), boxes of 64 x ntile in
// the 128-byte swizzle; reads past the batch fill zeros.
bool encode_x_map(CUtensorMap* map, const void* x, int bf16, int64_t batch, int64_t cols, int ntile) {
    const auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(batch)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(ntile)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                           const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

namespace hqq {

int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;  // no device here: the B200's count
    }
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

// K splits for grids too small to fill the GPU: about one CTA per SM, each
// split long enough to amortise its pipeline fill and partial-tile traffic
// (at least 8 K tiles, 40 for batch tiles of 128 and more).  Measured on
// 4096-row matrices: 4096x11008 batch 256 (4 splits of 43 tiles) 0.132 ->
// 0.080 ms, 4096x4096 batch 16 (4 of 16) 0.046 -> 0.025 ms; 4096x4096 batch
// 256 stays unsplit (0.055 ms; 4 splits of 16 tiles 0.059, 2 of 32 0.070).
int gemm_splits(int64_t rows, int64_t cols, int batch) {
    int ntile = 0, ntiles = 0;
    gemm_tiles(batch, &ntile, &ntiles);
    const int64_t ctas = ((rows + kTileM - 1) / kTileM) * ntiles;
    const int sms = sm_count();
    const int64_t ktot = cols / kTileK, min_kps = ntile >= 128 ? 40 : 8;
    int64_t sp = ctas >= (sms * 3) / 4 ? 1 : sms / ctas;
    if (sp > ktot / min_kps) sp = ktot / min_kps;
    return sp < 1 ? 1 : static_cast<int>(sp);
}

// Workspace of a split product: tickets [tiles] (rounded to 256 bytes), then
// the fp32 partial tiles; 0 when the product runs unsplit.
size_t gemm_workspace_bytes(int64_t rows, int64_t cols, int batch) {
    const int sp = gemm_splits(rows, cols, batch);
    if (sp <= 1) return 0;
    int ntile = 0, ntiles = 0;
    gemm_tiles(batch, &ntile, &ntiles);
    const int64_t ktot = cols / kTileK, kps = (ktot + sp - 1) / sp, splits = (ktot + kps - 1) / kps;
    const int64_t tiles = ((rows + kTileM - 1) / kTileM) * ntiles;
    return static_cast<size_t>(((tiles * 4 + 255) / 256) * 256 + tiles * splits * ntile * kTileM * 4);
}

// Batch tiles: as few as possible (N <= 256 each), of equal size rounded up to 16.
void gemm_tiles(int batch, int* ntile, int* ntiles) {
    const int nt = (batch + 255) / 256;
    const int per = (batch + nt - 1) / nt;
    *ntiles = nt;
    *ntile = (per + 15) / 16 * 16;
}

cudaError_t launch_gemm(const GemvArgs& a, cudaStream_t stream) {
    GemmParams p{};
    p.packed = a.packed;
    p.scale = a.scale;
    p.zero = a.zero;
    p.zero_meta = a.zero_meta;
    p.x = static_cast<const uint16_t*>(a.x);
    p.y = a.y;
    p.rows = a.rows;
    p.cols = a.cols;
    p.g_log = 0;
    while ((1 << p.g_log) < a.g) ++p.g_log;
    p.batch = a.batch;
    int ntiles = 1;
    gemm_tiles(a.batch, &p.ntile, &ntiles);
    p.stages = gemm_stages(p.ntile);
    const int ktot = static_cast<int>(a.cols / kTileK);
    p.splits = gemm_splits(a.rows, a.cols, a.batch);
    if (p.splits > 1 && (a.workspace == nullptr || a.workspace_bytes < gemm_workspace_bytes(a.rows, a.cols, a.batch)))
        p.splits = 1;  // no room for the partials: run unsplit
    p.kps = (ktot + p.splits - 1) / p.splits;
    p.splits = (ktot + p.kps - 1) / p.kps;
    if (p.splits > 1) {
        const int64_t tiles = ((a.rows + kTileM - 1) / kTileM) * ((a.batch + p.ntile - 1) / p.ntile);
        p.tickets = static_cast<uint32_t*>(a.workspace);
        p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + ((tiles * 4 + 255) / 256) * 256);
        const cudaError_t e = cudaMemsetAsync(p.tickets, 0, static_cast<size_t>(tiles) * 4, stream);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(static_cast<unsigned>((a.rows + kTileM - 1) / kTileM), static_cast<unsigned>(ntiles),
                    static_cast<unsigned>(p.splits));
    const size_t smem = gemm_smem_bytes(p.ntile, p.stages);
    const bool bf16 = a.x_dtype == 1;
    alignas(64) CUtensorMap xmap;
    if (!encode_x_map(&xmap, a.x, bf16 ? 1 : 0, a.batch, a.cols, p.ntile)) return cudaErrorInvalidValue;
    switch (a.nbits) {
        case 1: return launch_n<1>(p, xmap, bf16, a.zero_nbits, grid, smem, stream);
        case 2: return launch_n<2>(p, xmap, bf16, a.zero_nbits, grid, smem, stream);
        case 3: return launch_n<3>(p, xmap, bf16, a.zero_nbits, grid, smem, stream);
        case 4: return launch_n<4>(p, xmap, bf16, a.zero_nbits, grid, smem, stream);
        default: return launch_n<8>(p, xmap, bf16, a.zero_nbits, grid, smem, stream);
    }
}

cudaError_t launch_gemm_wait_selftest(unsigned long long limit_ns, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

// HQQ_OK, or HQQ_ERR_TIMEOUT if a product since the last call gave up a wait
// (the flag is cleared); HQQ_ERR_CUDA if the stream failed.
int gemm_take_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return 5;
    }
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_status, sizeof(v)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(zero)) != cudaSuccess) {
        cudaGetLastError();
        return 5;
    }
    return v ? 6 : 0;
}

}  // namespace hqq
