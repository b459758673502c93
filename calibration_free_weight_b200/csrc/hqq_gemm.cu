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
// K is walked in 64-element tiles through a ring of kStages shared-memory
// stages, each in the canonical 128-byte-swizzled K-major layout (row r of a
// tile at r * 128 bytes, its 16-byte chunk c at chunk c ^ (r % 8)):
//   * every thread dequantises 32 weights of the A tile (codes prefetched in
//     registers one tile ahead) and stores them as 16-bit values;
//   * the x tile arrives by cp.async, issued one tile ahead (rows past the
//     batch are zero-filled);
//   * thread 0 issues four tcgen05.mma (K = 16 each) into the fp32 accumulator
//     in tensor memory and commits them to the stage's mbarrier, which frees
//     the stage for the tile kStages later.
// The epilogue reads the accumulator with tcgen05.ld (warp w reads the 32 rows
// of its lane quarter w % 4, half of the columns) and stores y.
//
// Waits: every mbarrier wait gives up after ~1 s of global time, records a
// timeout in a device status word (read by hqq_gemm_get_status) and makes the
// whole CTA skip to the release of its tensor memory; no wait can hang.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "hqq_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kTileM = 128;          // MMA M: weight rows per CTA
constexpr int kTileK = 64;           // elements per K tile: one 128-byte swizzle row of 16-bit values
constexpr int kStages = 4;           // shared-memory ring
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

// Completion of the phase with this parity, or false after kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_test(bar, parity))
        if (global_ns() - t0 > kWaitNs) return false;
    return true;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
};

// Inputs of one thread's 32 consecutive weights of one K tile (one row):
// the codes as a little-endian bit stream (weight e at bit e * NBITS) and the
// scale and zero of each 8-weight piece.  Loaded one tile ahead.
template <int NBITS>
struct ARaw {
    uint32_t w[NBITS];
    float s[4], z[4];
};

__device__ __forceinline__ float half_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

template <int NBITS, int ZB>
__device__ __forceinline__ void load_a(const GemmParams& p, int64_t row, int64_t c0, ARaw<NBITS>& a) {
    if (row >= p.rows) {  // rows past the matrix: W_r = (0 - 0) * 0
#pragma unroll
        for (int i = 0; i < NBITS; ++i) a.w[i] = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) a.s[i] = a.z[i] = 0.0f;
        return;
    }
    const int64_t e0 = row * p.cols + c0;  // first weight; a multiple of 32, so its codes start on 4 * NBITS bytes
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.packed + (e0 / 32) * (4 * NBITS));
    if (NBITS == 4 || NBITS == 8) {
#pragma unroll
        for (int i = 0; i < NBITS; i += 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i / 4);
            a.w[i] = v.x;
            a.w[(i + 1) % NBITS] = v.y;
            a.w[(i + 2) % NBITS] = v.z;
            a.w[(i + 3) % NBITS] = v.w;
        }
    } else if (NBITS == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
        a.w[0] = v.x;
        a.w[1 % NBITS] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < NBITS; ++i) a.w[i] = __ldg(src + i);
    }
    // one group for all 32 weights when g >= 32, else one per piece
    const int npc = p.g_log >= 5 ? 1 : 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
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
    if (off + NBITS > 32) v |= w[(word + 1) % NBITS] << (32 - off);
    return v & mask;
}

// Exact small integer -> float through the mantissa of 2^23 (integer-to-float
// conversion issues on the XU pipe).
__device__ __forceinline__ float small_int_to_float(uint32_t q) {
    return __fsub_rn(__uint_as_float(0x4B000000u | q), 8388608.0f);
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

template <int NBITS, bool BF16, int P>
__device__ __forceinline__ void piece_to_smem(const ARaw<NBITS>& a, uint32_t dst) {
    uint32_t v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float q0 = small_int_to_float(code_at<NBITS>(a.w, 8 * P + 2 * i));
        const float q1 = small_int_to_float(code_at<NBITS>(a.w, 8 * P + 2 * i + 1));
        v[i] = pack2<BF16>(__fmul_rn(__fsub_rn(q0, a.z[P]), a.s[P]), __fmul_rn(__fsub_rn(q1, a.z[P]), a.s[P]));
    }
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

// W_r of this thread's 32 weights, rounded to 16 bits, into row r, chunks
// 4h .. 4h+3 of an A stage (128-byte swizzle: chunk c of row r at c ^ (r % 8)).
template <int NBITS, bool BF16>
__device__ __forceinline__ void store_a(const ARaw<NBITS>& a, uint32_t stage, int r, int h) {
    const uint32_t row = stage + static_cast<uint32_t>(r) * 128u;
    const int sw = r & 7;
    piece_to_smem<NBITS, BF16, 0>(a, row + ((((4 * h) + 0) ^ sw) << 4));
    piece_to_smem<NBITS, BF16, 1>(a, row + ((((4 * h) + 1) ^ sw) << 4));
    piece_to_smem<NBITS, BF16, 2>(a, row + ((((4 * h) + 2) ^ sw) << 4));
    piece_to_smem<NBITS, BF16, 3>(a, row + ((((4 * h) + 3) ^ sw) << 4));
}

// The x tile [ntile][64] of K tile kt into a B stage, by cp.async (rows past
// the batch are zero-filled: source size 0).
__device__ __forceinline__ void issue_b(const GemmParams& p, int64_t n0, int kt, uint32_t stage) {
    const int chunks = p.ntile * 8;
    for (int q = threadIdx.x; q < chunks; q += kThreads) {
        const int n = q >> 3, c = q & 7;
        const int64_t b = n0 + n;
        const bool in = b < p.batch;
        const uint16_t* src = p.x + (in ? b : 0) * p.cols + static_cast<int64_t>(kt) * kTileK + c * 8;
        cp_async16(stage + static_cast<uint32_t>(n) * 128u + ((c ^ (n & 7)) << 4), src, in ? 16u : 0u);
    }
}

__host__ __device__ constexpr uint32_t tmem_columns(int ntile) {
    return ntile <= 32 ? 32u : ntile <= 64 ? 64u : ntile <= 128 ? 128u : 256u;
}

__host__ __device__ constexpr size_t gemm_smem_bytes(int ntile) {
    // 1024 bytes of slack to align the stages to the 1024-byte swizzle period
    return 1024 + static_cast<size_t>(kStages) * (kStageA + static_cast<size_t>(ntile) * 128) + kStages * 8 + 16;
}

template <int NBITS, bool BF16, int ZB>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t* const smem = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sA = base;                                      // kStages x 16 KB
    const uint32_t sB = sA + kStages * kStageA;                    // kStages x ntile x 128 B
    const uint32_t bars = sB + kStages * static_cast<uint32_t>(p.ntile) * 128u;  // kStages mbarriers
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + (bars + kStages * 8 - base));
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTileM, n0 = static_cast<int64_t>(blockIdx.y) * p.ntile;
    const int num_k = static_cast<int>(p.cols / kTileK);
    const uint32_t ncols = tmem_columns(p.ntile);
    auto bar = [&](int s) { return bars + 8u * static_cast<uint32_t>(s); };
    auto stage_a = [&](int s) { return sA + static_cast<uint32_t>(s) * kStageA; };
    auto stage_b = [&](int s) { return sB + static_cast<uint32_t>(s) * static_cast<uint32_t>(p.ntile) * 128u; };

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar(s), 1);
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

    // producer role: row r of the A tile, weights [32h, 32h + 32) of each K tile
    const int r = tid >> 1, h = tid & 1;
    const int64_t row = m0 + r;
    ARaw<NBITS> cur, nxt;
    load_a<NBITS, ZB>(p, row, 32 * h, cur);
    issue_b(p, n0, 0, stage_b(0));
    cp_async_commit();
    bool ok = true;
    for (int kt = 0; kt < num_k; ++kt) {
        const int s = kt % kStages;
        if (kt + 1 < num_k) {
            // tile kt+1's stage is free once the MMAs of tile kt+1-kStages are done
            const int s1 = (kt + 1) % kStages;
            if (kt + 1 >= kStages && !mbar_wait(bar(s1), static_cast<uint32_t>((kt + 1) / kStages - 1) & 1u))
                *abort_flag = 1;
            issue_b(p, n0, kt + 1, stage_b(s1));
            load_a<NBITS, ZB>(p, row, static_cast<int64_t>(kt + 1) * kTileK + 32 * h, nxt);
        }
        cp_async_commit();  // one group per iteration (empty on the last): uniform group accounting
        store_a<NBITS, BF16>(cur, stage_a(s), r, h);
        cp_async_wait<1>();  // tile kt's x has landed
        fence_async_smem();  // generic-proxy shared-memory writes -> visible to the tensor core
        __syncthreads();
        if (*abort_flag) {
            ok = false;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < kTileK / 16; ++j)
                mma_f16(tmem, smem_desc(stage_a(s) + 32u * j), smem_desc(stage_b(s) + 32u * j), idesc,
                        (kt | j) != 0 ? 1u : 0u);
            mma_commit(bar(s));
        }
        cur = nxt;
    }
    cp_async_wait<0>();
    if (ok) {  // the last commit covers every MMA of this CTA
        const int kl = num_k - 1;
        if (!mbar_wait(bar(kl % kStages), static_cast<uint32_t>(kl / kStages) & 1u)) *abort_flag = 1;
    }
    __syncthreads();
    ok = ok && !*abort_flag;
    if (ok) {
        tc_fence_after();
        const int q = warp & 3, half = warp >> 2, nh = p.ntile / 2;
        const int64_t orow = m0 + 32 * q + lane;
        for (int c0 = half * nh; c0 < (half + 1) * nh; c0 += 8) {
            float v[8];
            tmem_ld8(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0), v);
            if (orow < p.rows) {
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
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
    }
}

template <int NBITS, bool BF16, int ZB>
cudaError_t launch_t(const GemmParams& p, dim3 grid, size_t smem, cudaStream_t stream) {
    auto kern = gemm_kernel<NBITS, BF16, ZB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int NBITS>
cudaError_t launch_n(const GemmParams& p, bool bf16, int zb, dim3 grid, size_t smem, cudaStream_t stream) {
    if (bf16) return zb == 8 ? launch_t<NBITS, true, 8>(p, grid, smem, stream)
                             : launch_t<NBITS, true, 16>(p, grid, smem, stream);
    return zb == 8 ? launch_t<NBITS, false, 8>(p, grid, smem, stream)
                   : launch_t<NBITS, false, 16>(p, grid, smem, stream);
}

}  // namespace

namespace hqq {

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
    const dim3 grid(static_cast<unsigned>((a.rows + kTileM - 1) / kTileM), static_cast<unsigned>(ntiles));
    const size_t smem = gemm_smem_bytes(p.ntile);
    const bool bf16 = a.x_dtype == 1;
    switch (a.nbits) {
        case 1: return launch_n<1>(p, bf16, a.zero_nbits, grid, smem, stream);
        case 2: return launch_n<2>(p, bf16, a.zero_nbits, grid, smem, stream);
        case 3: return launch_n<3>(p, bf16, a.zero_nbits, grid, smem, stream);
        case 4: return launch_n<4>(p, bf16, a.zero_nbits, grid, smem, stream);
        default: return launch_n<8>(p, bf16, a.zero_nbits, grid, smem, stream);
    }
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
