/*
 * hqq.h -- C ABI of the B200 (sm_100a) Half-Quadratic Quantization library.
 *
 * The library quantises an fp16/bf16 weight matrix to 8/4/3/2/1-bit codes with
 * the HQQ zero-point solver, with no calibration data.  Method: techreport.ngo,
 * "Weight-only quantization without the calibration tax" (Half-Quadratic
 * Quantization of Large Machine Learning Models):
 *   - section "Outlier-aware optimization without gradients": lp loss with
 *     p < 1, half-quadratic split with an auxiliary variable W_e, scale s fixed,
 *     zero-point z optimised; sub-problem 1 = generalised soft-thresholding,
 *     sub-problem 2 = average over the quantisation group axis; ~20 closed-form
 *     iterations;
 *   - section "Benchmark results" / "Llama-2": p = 0.7, beta = 1,
 *     kappa = 1.01, 20 iterations, early stopping, zero-point quantised to 8
 *     bit without extra grouping.
 * The interface nouns (nbits, group_size, axis -> W_q, scale, zero, and a
 * dequantize() for inspection) follow "HQQ - Half-Quadratic Quantization"
 * (skill4agent.com), section "Core concepts" ("Quantization configuration",
 * "HQQLinear layer").
 *
 * Per group of g weights w (L = 2^nbits - 1), all arithmetic in fp32:
 *   s  = min(L / (max w - min w), 2e4)   (2e4 when max == min)
 *   z0 = -min(w) * s
 *   iteration k (k = 0 .. iters-1), beta_0 = beta, beta_{k+1} = kappa * beta_k:
 *     W_q = clamp(round_half_even(w*s + z_k), 0, L);  W_r = (W_q - z_k) / s
 *     e_k = mean |w - W_r|^p
 *     stop rule (below); then
 *     W_e = sign(w - W_r) * max(|w - W_r| - |w - W_r|^(p-1) / beta_k, 0)
 *     z_{k+1} = mean(W_q - (w - W_e) * s)
 *   stop rule: keep going while e_k is strictly below every earlier error; the
 *   kept zero-point z* is the iterate with the lowest error so far.
 *     HQQ_STOP_GROUP : each group stops at its own first non-improvement;
 *     HQQ_STOP_TENSOR: all groups stop together at the first non-improvement of
 *                      the tensor-wide mean error (summed in fp64);
 *     HQQ_STOP_NONE  : all `iters` iterations, z* = lowest-error iterate.
 *   Output codes: clamp(round(w*s + z*), 0, L).  scale = fp16(1/s).
 *   iters = 0 gives plain min/max round-to-nearest (z* = z0).
 *
 * Layout.  W is row-major [rows, cols] (rows = output features).
 *   axis = 1: group j = the g contiguous elements [j*g, (j+1)*g) of the
 *             flattened matrix (g must divide cols); scale/zero are
 *             [rows, cols/g] row-major.
 *   axis = 0: group (rb, c) = rows rb*g .. rb*g+g-1 of column c (g must divide
 *             rows); scale/zero are [rows/g, cols] row-major.
 *   Packed codes (LSB-first bit streams, nbits bits per code):
 *   axis = 1: one stream over the flattened matrix; element e occupies bits
 *             e*nbits .. e*nbits+nbits-1, bit k of byte B is stream bit 8B+k.
 *             Size rows*cols*nbits/8 bytes (3-bit: 8 codes per 3 bytes).
 *   axis = 0: one stream per column running down the rows; byte R of column c
 *             is stored at R*cols + c (packed shape [rows*nbits/8, cols]).
 *   This layout is this library's own; it is not claimed compatible with any
 *   other HQQ format.
 *
 * Conventions for every call:
 *   - All buffers are caller-owned device memory (cudaMalloc, torch, ...).
 *     The library allocates and frees no device memory (hqq_quantize_noalloc
 *     uses a static device array of the library; the stream executors create
 *     and destroy their own copy streams and events within the call).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream).  Argument errors are detected on the host
 *     and returned before anything is launched; no output is touched then.
 *   - Inputs must be finite.
 */
#ifndef HQQ_B200_H
#define HQQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HQQ_OK = 0,
    HQQ_ERR_INVALID_ARG = 1,      /* bad nbits/p/beta/kappa/iters/mode, NULL pointer, host pointer */
    HQQ_ERR_SHAPE = 2,            /* group_size not a power of two in [8,1024] or not dividing the group axis */
    HQQ_ERR_DTYPE = 3,            /* dtype not HQQ_F16 / HQQ_BF16 */
    HQQ_ERR_ALIGN = 4,            /* a buffer is not aligned as documented */
    HQQ_ERR_CUDA = 5,             /* a CUDA runtime call failed (launch, attribute query) */
    HQQ_ERR_TIMEOUT = 6,          /* a bounded device wait gave up: the tensor-stop solver's (hqq_get_status)
                                     or hqq_gemm's (hqq_gemm_get_status) */
    HQQ_ERR_COOP_UNSUPPORTED = 7, /* reserved, not returned: without cooperative launches the tensor-stop
                                     solver takes its chunked launches instead */
    HQQ_ERR_WORKSPACE = 8         /* workspace missing or smaller than hqq_workspace_bytes() */
} hqq_status;

typedef enum { HQQ_F16 = 0, HQQ_BF16 = 1 } hqq_dtype;

typedef enum { HQQ_STOP_GROUP = 0, HQQ_STOP_TENSOR = 1, HQQ_STOP_NONE = 2 } hqq_stop_mode;

/* Bytes of the packed code buffer: rows*cols*nbits/8.  0 for invalid args.
 * The bit widths are those of "HQQ - Half-Quadratic Quantization"
 * (skill4agent.com), section "Core concepts" (nbits 1-8, of which the pages
 * use 8/4/3/2/1); the pages print no storage layout, so the bit stream above
 * is this library's own. */
size_t hqq_packed_bytes(int64_t rows, int64_t cols, int nbits, int group_size, int axis);

/* Number of groups G = rows*cols/group_size (one scale and one zero each).
 * -1 for invalid args.  Groups of group_size consecutive weights along `axis`
 * ("HQQ - Half-Quadratic Quantization" (skill4agent.com), section "Core
 * concepts": BaseQuantizeConfig(nbits, group_size, axis)). */
int64_t hqq_num_groups(int64_t rows, int64_t cols, int group_size, int axis);

/* Bytes of device workspace hqq_quantize needs for this problem (always > 0;
 * holds the status word, the work counters, the fp32 kept zeros of the 8-bit
 * zero path (4 bytes per group, hence zero_nbits), for axis 0 the running
 * state of groups between passes and, for the tensor stop, the per-group
 * state, per-CTA partials and per-iteration errors).  0 for invalid args.  The pages
 * have no counterpart: their solver runs as whole-tensor operations that
 * allocate as they go; here the caller owns every byte. */
size_t hqq_workspace_bytes(int64_t rows, int64_t cols, int group_size, int axis, int stop_mode, int zero_nbits);

/*
 * Quantise W.
 *   W            device, dtype [rows, cols] row-major, 16-byte aligned.
 *   p, beta, kappa, iters
 *                0 < p < 2, beta > 0, kappa >= 1, 0 <= iters <= 1000.
 *   stop_mode    hqq_stop_mode.
 *   zero_nbits   16: zero is fp16[G];  8: zero is uint8[G] and zero_meta is
 *                fp32[2] = (1/sz, zz), one round-to-nearest quantiser for the
 *                whole tensor: sz = min(255/(max z* - min z*), 2e4) (2e4 when
 *                all equal), zz = -min(z*)*sz, zq = clamp(round(z*sz + zz), 0,
 *                255); the dequantised zero is (zq - zz) * (1/sz).  The codes
 *                W_q use the unquantised fp32 z*.
 *   W_q_packed   device uint8[hqq_packed_bytes], 16-byte aligned.
 *   scale        device fp16[G] (= 1/s), 2-byte aligned.
 *   zero         device fp16[G] or uint8[G], see zero_nbits.
 *   zero_meta    device fp32[2] when zero_nbits == 8, else ignored (may be NULL).
 *   workspace    device, >= hqq_workspace_bytes(...), 256-byte aligned;
 *                contents need no initialisation and are overwritten.
 *   debug_best_iter  optional device int32[G]: index k of the kept iterate.
 *   debug_best_err   optional device fp32[G]: mean |w - W_r|^p of the kept
 *                    zero-point (lg2/ex2 hardware approximations, ~1e-6 rel).
 *   debug_zero_f32   optional device fp32[G]: z* before storage.
 *   stream       cudaStream_t as void*.
 * Returns HQQ_OK or an error code.  Tensor stop on axis 1 runs, when the
 * problem fits (hqq_tensor_resident), as one cooperative launch whose warps
 * wait for the tensor error of earlier iterations; each such wait gives up
 * after about 1 s, and then the call's outputs are undefined and the
 * workspace's status word holds HQQ_ERR_TIMEOUT (hqq_get_status).  No other
 * path waits on another CTA.  Calls that share a workspace must not run
 * concurrently.
 */
int hqq_quantize(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis,
                 float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits,
                 void* W_q_packed, void* scale, void* zero, void* zero_meta,
                 void* workspace, size_t workspace_bytes,
                 int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32,
                 void* stream);

/*
 * hqq_quantize_half -- the solver in half precision, the variant the pages run
 * on the GPU (techreport.ngo, "Weight-only quantization without the
 * calibration tax", section "Speed: from hours to minutes"; the steps of
 * section "Outlier-aware optimization without gradients").  This library's
 * reading of half precision: every element-wise value is rounded to fp16 (to
 * nearest, ties to even) -- s = h(min(L/(max w - min w), 2e4)), z0 = h(-min w
 * * s), w*s, v = h(h(w*s) + z), W_q = clamp(round(v), 0, L), r = h(v - W_q),
 * the error terms h(|r|^p) (their sum exact); each z update rounds an exact
 * mean to fp16 once; the proximal step rounds d = h(fl32(r/s)), W_e =
 * h(shrink(d)) and h(h(w - W_e)*s).  The stop rules group and none, beta and
 * the 8-bit zero are as in hqq_quantize; scale = h(fl32(1/s)), zero = the fp16
 * z*.  |r|^p is evaluated with the hardware base-2 log and exponential in fp32
 * and then rounded to fp16, so a term can sit one fp16 step from the exactly
 * rounded value and a stop decision whose two sums differ by less than about
 * 2^-9 relative may go the other way.
 * Arguments as hqq_quantize, with: dtype must be HQQ_F16 (else HQQ_ERR_DTYPE);
 * axis must be 1 and stop_mode HQQ_STOP_GROUP or HQQ_STOP_NONE (else
 * HQQ_ERR_INVALID_ARG); workspace as for hqq_quantize with the same arguments.
 */
int hqq_quantize_half(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis,
                      float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits,
                      void* W_q_packed, void* scale, void* zero, void* zero_meta,
                      void* workspace, size_t workspace_bytes,
                      int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32,
                      void* stream);

/*
 * Dequantise for inspection ("HQQ - Half-Quadratic Quantization"
 * (skill4agent.com), section "Core concepts": HQQLinear's dequantize(); the
 * rule W_r = (W_q - z) / s of techreport.ngo, "Weight-only quantization
 * without the calibration tax", section "Outlier-aware optimization without
 * gradients", with scale = 1/s): W_out = (W_q - zero) * scale computed in fp32 and
 * rounded (to nearest even) to out_dtype; with zero_nbits == 8 the zero is
 * first rebuilt as (zq - zz) * (1/sz) from zero_meta.  Buffers as in
 * hqq_quantize; W_out is device out_dtype [rows, cols], 16-byte aligned.
 */
int hqq_dequantize(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta,
                   int64_t rows, int64_t cols, int nbits, int group_size, int axis, int zero_nbits,
                   int out_dtype, void* W_out, void* stream);

/*
 * hqq_quantize_scale8 -- the "_s*" variant of the Llama-2 table
 * (techreport.ngo, "Weight-only quantization without the calibration tax",
 * section "Benchmark results" / "Llama-2", table footnote: the scale is also
 * quantised to 8 bit with a group size of 128).  The pages give no formula;
 * this library reads it as one round-to-nearest 8-bit quantiser per run of
 * scale_group consecutive scales (in group order; the last run may be shorter):
 *   sc = 255 / (max - min) over the run (1 when max == min), zc = -min * sc,
 *   code = clamp(round_half_even(scale * sc + zc), 0, 255),
 * all in fp32 from the fp16 scales, stored meta per run (1/sc, zc) in fp32.
 * The codes W_q are not recomputed; hqq_dequantize_s8 rebuilds each scale as
 * (code - zc) * (1/sc).
 *   scale        device fp16[G] from hqq_quantize, 2-byte aligned (read only).
 *   num_groups   G >= 0.
 *   scale_group  run length S >= 1 (128 in the pages).
 *   scale_q      device uint8[G] (output).
 *   scale_meta   device fp32[2 * ceil(G / S)] (output), 4-byte aligned.
 *   stream       cudaStream_t as void*.
 * Returns HQQ_OK, HQQ_ERR_INVALID_ARG (bad pointer or S < 1, G < 0),
 * HQQ_ERR_ALIGN or HQQ_ERR_CUDA.  Allocates nothing.
 */
int hqq_quantize_scale8(const void* scale, int64_t num_groups, int scale_group, void* scale_q, void* scale_meta,
                        void* stream);

/*
 * hqq_dequantize with 8-bit scales: as hqq_dequantize, but the scale of
 * group j is (scale_q[j] - zc) * (1/sc) with the (1/sc, zc) pair of run
 * j / scale_group from hqq_quantize_scale8.  scale_q is device uint8[G],
 * scale_meta device fp32[2 * ceil(G / scale_group)] (4-byte aligned).
 */
int hqq_dequantize_s8(const void* W_q_packed, const void* scale_q, const void* scale_meta, int scale_group,
                      const void* zero, const void* zero_meta, int64_t rows, int64_t cols, int nbits,
                      int group_size, int axis, int zero_nbits, int out_dtype, void* W_out, void* stream);

/*
 * Streaming a list of host-resident matrices through one GPU (a model
 * quantised layer by layer; the pages run the solver on the GPU and move the
 * data once, techreport.ngo, "Weight-only quantization without the
 * calibration tax", section "Speed: from hours to minutes").
 *
 * hqq_host_matrix: one matrix and its outputs, all in HOST memory (pinned
 * for the copies to overlap the solver):
 *   W            [rows, cols] fp16/bf16 (dtype of the call), read.
 *   W_q_packed   uint8[hqq_packed_bytes], scale fp16[G], zero fp16[G] or
 *                uint8[G], zero_meta fp32[2] (zero_nbits == 8): written.
 */
typedef struct hqq_host_matrix {
    const void* W;
    int64_t rows, cols;
    void* W_q_packed;
    void* scale;
    void* zero;
    void* zero_meta;
} hqq_host_matrix;

/* Device bytes hqq_quantize_stream needs for this list: two slots, each
 * sized for the largest matrix (W, outputs and solver workspace).  0 on
 * invalid arguments. */
size_t hqq_stream_device_bytes(const hqq_host_matrix* mats, int n, int nbits, int group_size, int axis,
                               int stop_mode, int zero_nbits);

/*
 * hqq_quantize_stream -- hqq_quantize on each of the n matrices (the same
 * settings for all; hqq_quantize_stream_jobs below takes them per matrix), with the
 * copy of matrix i+1 to the GPU and of matrix i-1's outputs back to the host
 * overlapping the solver on matrix i (two device slots; copies on two
 * streams the call creates; the solver on `stream`).  Solver arguments as in
 * hqq_quantize, the same for every matrix.  device_buffer: device memory of
 * at least hqq_stream_device_bytes(...), 256-byte aligned, owned by the
 * caller.  Blocks until every output is in host memory.  Returns HQQ_OK or
 * the first error (HQQ_ERR_WORKSPACE if device_bytes is too small).
 */
int hqq_quantize_stream(const hqq_host_matrix* mats, int n, int dtype, int nbits, int group_size, int axis, float p,
                        float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* device_buffer,
                        size_t device_bytes, void* stream);

/*
 * Per-matrix settings for a streamed model: attention and MLP layers at
 * different bit widths and group sizes ("HQQ - Half-Quadratic Quantization"
 * (skill4agent.com), section "Mixed precision quantization": attention 4-bit
 * g64, MLP 2-bit g32), quantised layer by layer (same page, section "Common
 * issues", out of memory during quantization).
 *   m            the matrix and its host outputs, as for hqq_quantize_stream
 *                (zero_meta needed when zero_nbits == 8).
 *   nbits, group_size, axis, stop_mode, zero_nbits: as in hqq_quantize, for
 *                this matrix only.
 */
typedef struct hqq_stream_job {
    hqq_host_matrix m;
    int nbits, group_size, axis, stop_mode, zero_nbits;
} hqq_stream_job;

/* Called by hqq_quantize_stream_jobs on the calling thread, once per job and
 * in job order, as soon as the outputs of job `index` are complete in host
 * memory (e.g. to write them to disk while later jobs run).  It may not free
 * or reuse the job's host buffers before the call returns. */
typedef void (*hqq_stream_done_fn)(int index, void* user);

/* Device bytes hqq_quantize_stream_jobs needs: two slots, each buffer kind
 * (W, codes, scale, zero, workspace) sized for the largest job.  0 on invalid
 * arguments (n < 1, a bad job setting or shape). */
size_t hqq_stream_jobs_device_bytes(const hqq_stream_job* jobs, int n);

/*
 * hqq_quantize_stream_jobs -- hqq_quantize_stream with settings per matrix,
 * and completion reporting for resumable runs.  p, beta, kappa, iters and the
 * input dtype are the same for every job.  Every job's settings and pointers
 * are checked before anything is copied or launched (an invalid job returns
 * its hqq_quantize status and touches nothing).  on_done (may be NULL) is
 * called for each finished job, in order, with `user`.  jobs_done (may be
 * NULL) receives the number of leading jobs whose outputs are complete in
 * host memory when the call returns: n on success.  A caller that persists
 * each job in on_done resumes an interrupted run by passing the jobs not yet
 * persisted.  A job whose matrix is the previous job's (the same host W
 * pointer and shape, e.g. one weight quantised at two settings) reuses the
 * device copy: the matrix crosses PCIe once.  device_buffer: device memory
 * of at least hqq_stream_jobs_device_bytes(jobs, n), 256-byte aligned,
 * caller-owned.
 * Blocks until every output is in host memory.  Returns HQQ_OK or the first
 * error (HQQ_ERR_WORKSPACE if device_bytes is too small).
 */
int hqq_quantize_stream_jobs(const hqq_stream_job* jobs, int n, int dtype, float p, float beta, float kappa, int iters,
                             void* device_buffer, size_t device_bytes, hqq_stream_done_fn on_done, void* user,
                             int* jobs_done, void* stream);

/*
 * hqq_gemv -- fused dequantisation + matrix-vector product of the packed
 * layout, the step an inference backend runs after quantisation (the
 * dequantisation rule W_r = (W_q - z) * scale of techreport.ngo, "Weight-only
 * quantization without the calibration tax", section "Outlier-aware
 * optimization without gradients"):
 *   y[b][r] = sum_c W_r[r][c] * x[b][c],  b < batch <= 8.
 * Groups along the input dimension (axis 1 of an [out, in] = [rows, cols]
 * weight).  W_q_packed, scale, zero, zero_meta as produced by hqq_quantize
 * (fp16 scale; fp16 or 8-bit zero).  x: device [batch][cols] fp16/bf16
 * (x_dtype), 16-byte aligned; y: device fp32 [batch][rows], 4-byte aligned.
 * Arithmetic in fp32 (per 8-column piece s * (sum q x - z * sum x), the sum of
 * each row in a fixed order): the same real number as the fp64 product of the
 * dequantised weights, up to rounding.  Returns HQQ_OK, HQQ_ERR_DTYPE,
 * HQQ_ERR_SHAPE, HQQ_ERR_INVALID_ARG (batch outside 1..8, bad pointer),
 * HQQ_ERR_ALIGN or HQQ_ERR_CUDA.  Allocates nothing.
 */
int hqq_gemv(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta, int64_t rows,
             int64_t cols, int nbits, int group_size, int zero_nbits, const void* x, int x_dtype, int batch, float* y,
             void* stream);

/*
 * hqq_gemm -- fused dequantisation + matrix product on the tensor cores
 * (tcgen05) for batches of activation vectors, the product a 16-bit
 * tensor-core backend computes with the packed layout ("HQQ - Half-Quadratic
 * Quantization" (skill4agent.com), section "Backends"; dequantisation rule
 * W_r = (W_q - z) * scale of techreport.ngo, "Weight-only quantization
 * without the calibration tax", section "Outlier-aware optimization without
 * gradients"):
 *   y[b][r] = sum_c round16(W_r[r][c]) * x[b][c],  1 <= batch <= 65536,
 * with W_r formed in fp32 exactly as hqq_dequantize does, then rounded to the
 * activations' type (x_dtype; round to nearest even: both operands of one
 * 16-bit tensor-core product share a type), products exact and sums in fp32
 * (accumulated in tensor memory, order unspecified: |error| <= cols * 2^-23 *
 * sum_c |round16(W_r) x|).  Groups along the input dimension (axis 1 of an
 * [out, in] = [rows, cols] weight); cols must be a multiple of 64.
 * W_q_packed, scale, zero, zero_meta as produced by hqq_quantize.  x: device
 * [batch][cols] fp16/bf16, 16-byte aligned; y: device fp32 [batch][rows],
 * 4-byte aligned.  workspace (may be NULL): device memory of at least
 * hqq_gemm_workspace_bytes(rows, cols, batch), 256-byte aligned, caller-owned;
 * with it, a product whose 128-row x batch tiles are too few to fill the GPU
 * splits K across CTAs and the last split of each tile sums the partial tiles
 * in split order (the result is deterministic, but its fp32 summation order,
 * within the bound above, differs from the unsplit product's); without it, or
 * when it is smaller, the product runs unsplit.  Returns HQQ_OK,
 * HQQ_ERR_DTYPE, HQQ_ERR_SHAPE, HQQ_ERR_INVALID_ARG (batch out of range, bad
 * pointer), HQQ_ERR_ALIGN or HQQ_ERR_CUDA.  Allocates nothing.  Every wait
 * inside the kernel is bounded (about 1 s); a wait that gives up is reported
 * by hqq_gemm_get_status.
 */
int hqq_gemm(const void* W_q_packed, const void* scale, const void* zero, const void* zero_meta, int64_t rows,
             int64_t cols, int nbits, int group_size, int zero_nbits, const void* x, int x_dtype, int batch, float* y,
             void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes hqq_gemm uses to split K for this shape on the current
 * device (0: the product runs unsplit; also 0 on invalid sizes). */
size_t hqq_gemm_workspace_bytes(int64_t rows, int64_t cols, int batch);

/* Synchronises `stream`; HQQ_OK, or HQQ_ERR_TIMEOUT if a hqq_gemm since the
 * last call gave up a wait (the flag is then cleared), or HQQ_ERR_CUDA.
 * After HQQ_ERR_TIMEOUT the y of that product is undefined: a tile whose CTA
 * gave up keeps whatever y held before, and a tile of a split product that
 * lost one of its partials is filled with NaN. */
int hqq_gemm_get_status(void* stream);

/* Diagnostic of the bounded waits: one thread runs hqq_gemm's mbarrier wait,
 * with a limit of limit_us microseconds (1 .. 1e6), on a barrier that nothing
 * arrives on; it gives up and records the timeout as hqq_gemm does, so the
 * next hqq_gemm_get_status returns HQQ_ERR_TIMEOUT (and the one after that
 * HQQ_OK).  Asynchronous on `stream`; returns HQQ_OK, HQQ_ERR_INVALID_ARG or
 * HQQ_ERR_CUDA. */
int hqq_gemm_wait_selftest(int64_t limit_us, void* stream);

/* Synchronise `stream` and return the device status word held in `workspace`
 * by the last hqq_quantize on it: HQQ_OK, or HQQ_ERR_TIMEOUT when a wait of the
 * resident tensor-stop solver gave up; HQQ_ERR_CUDA if the synchronisation or
 * copy fails.  No counterpart on the pages: the channel for errors found on
 * the device after an asynchronous call returned (the hot-path table's
 * "grid barrier with a bounded spin"). */
int hqq_get_status(const void* workspace, void* stream);

/* Tensor stop (techreport.ngo, "Weight-only quantization without the
 * calibration tax", section "Outlier-aware optimization without gradients":
 * the mean error over the whole tensor decides the stop) keeps W on chip
 * where it fits: one cooperative launch runs every iteration, the per-group
 * state stays in shared memory and W (within half the L2) is read from L2 at
 * each iteration; one grid-wide fp64 reduction per iteration, no grid
 * barrier.  Otherwise the iterations run in chunks of launches that re-read W.
 * Both give the outputs the stop rule defines; their tensor errors are summed
 * in different orders, so a near-tied decision may differ.
 * hqq_tensor_resident: 1 if hqq_quantize with stop_mode HQQ_STOP_TENSOR and
 * these arguments (iters >= 1) takes the resident launch on the current
 * device, else 0 (also for invalid arguments).
 * hqq_set_tensor_resident: for the whole process, mode 0 never takes the
 * resident launch, 1 (the default) takes it for group sizes >= 32 where it
 * fits (below that it measured slower than the chunks), 2 wherever it fits;
 * returns the previous mode, or -1 (nothing changed) for another value.  Not
 * synchronised with calls in flight on other threads. */
int hqq_tensor_resident(int64_t rows, int64_t cols, int dtype, int group_size, int axis, int iters);
int hqq_set_tensor_resident(int mode);

/* Diagnostic of the resident tensor-stop solver's bounded wait: zeroes the
 * first 256 bytes of `workspace` (device, 256-byte aligned, workspace_bytes >=
 * 256), then one thread runs the solver's wait, with a limit of limit_us
 * microseconds (1 .. 1e6), on a decision that nothing publishes; it gives up
 * and records the timeout as the solver does, so hqq_get_status(workspace)
 * then returns HQQ_ERR_TIMEOUT.  Asynchronous on `stream`; returns HQQ_OK,
 * HQQ_ERR_INVALID_ARG or HQQ_ERR_CUDA. */
int hqq_quantize_wait_selftest(void* workspace, size_t workspace_bytes, int64_t limit_us, void* stream);

/* Static English description of a status code (no counterpart on the pages). */
const char* hqq_status_string(int status);

/* Size of the library-owned scratch buffer used by hqq_quantize_noalloc. */
#define HQQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * hqq_quantize_noalloc -- hqq_quantize for callers that cannot allocate
 * device memory, such as a plugin inside a host runtime that owns every device
 * allocation, or a latency-critical loop that must not pay for cudaMalloc and
 * the device synchronisation it can cause.  The HQQ pages have no counterpart:
 * this is an interface convenience of this library.
 *
 * Same arguments and results as hqq_quantize minus workspace/workspace_bytes.
 * The caller still passes (and owns) W and every output buffer.  stop_mode must
 * be HQQ_STOP_GROUP or HQQ_STOP_NONE; HQQ_STOP_TENSOR returns
 * HQQ_ERR_INVALID_ARG (use hqq_quantize for it).
 * Scratch: one buffer of HQQ_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory per
 * GPU, held by the library from load until the process exits.  Axis 1 needs a
 * 256-byte header and, with zero_nbits = 8, the kept zeros of all groups (4
 * bytes each): 4,194,240 groups fit exactly.  Axis 0 keeps running state per
 * group; a problem whose hqq_workspace_bytes() exceeds the scratch runs in
 * slices of groups, one after another on `stream` (same results); each slice
 * needs 44 bytes per entry and at least 4,096 entries (an entry is a group;
 * the columns of each block of group_size rows are counted up to whole warp
 * tiles of 32/P groups, P = group_size/32 for group_size >= 32, else 1), and
 * with zero_nbits = 8 the kept zeros (the array rounded up to 256 bytes) must
 * fit beside one slice and the header: 4,149,184 groups fit exactly.  More
 * return HQQ_ERR_WORKSPACE before anything is launched.  With zero_nbits = 16
 * every size fits.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).  The first call on each device looks up the buffer's device
 * address (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call on a device shares the buffer, which
 * keeps the last call's contents (each call clears what must start at zero);
 * calls whose work overlaps on the GPU race on it, so keep them ordered, e.g.
 * on one stream.
 */
int hqq_quantize_noalloc(const void* W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis,
                         float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits,
                         void* W_q_packed, void* scale, void* zero, void* zero_meta,
                         int32_t* debug_best_iter, float* debug_best_err, float* debug_zero_f32,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HQQ_B200_H */
