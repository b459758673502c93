/*
 * hqq_oracle.c -- plain, slow CPU restatement of the HQQ zero-point solver.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library; the product path never does.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes follows the technical description of Half-Quadratic
 * Quantization in "Weight-only quantization without the calibration tax"
 * (techreport.ngo, "Half-Quadratic Quantization of Large Machine Learning
 * Models"):
 *   - section "Outlier-aware optimization without gradients": an lp loss with
 *     p < 1 on the weight error, a half-quadratic split with an auxiliary
 *     variable W_e, the scale s fixed and only the zero-point z optimised;
 *     sub-problem 1 is the generalised soft-thresholding (proximal) operator,
 *     sub-problem 2 is an average over the quantisation group axis; about 20
 *     closed-form iterations;
 *   - section "Benchmark results" / "Llama-2": p = 0.7, beta = 1,
 *     kappa = 1.01, 20 iterations with early stopping, and the zero-point
 *     quantised to 8 bit with no extra grouping or optimisation.
 * The per-step formulas, in the pages' notation (L = 2^nbits - 1):
 *   W_q = clamp(round(W*s + z), 0, L)
 *   W_r = (W_q - z) / s
 *   W_e = sign(W - W_r) * max(|W - W_r| - |W - W_r|^(p-1) / beta, 0)
 *   z   = mean over the group of (W_q - (W - W_e) * s)
 *   beta <- kappa * beta
 * and the solver keeps the best zero-point seen, stopping once the lp error
 * stops falling.
 *
 * Readings of points the pages leave open:
 *   R1  s = min(L / (max - min), 2e4) when max > min, else 2e4.
 *   R2  round() is round-half-to-even (nearbyintf, default rounding mode).
 *   R3  the lp error of a zero-point is mean(|W - W_r|^p) with the same p.
 *   R4  the loop continues only on a strict improvement; an equal or larger
 *       error stops it and the earlier zero-point is kept.  The zero-point
 *       computed by the last allowed iteration is never evaluated.
 *   R5  shrink(0) = 0.
 *   R6  stop_mode = tensor: every group steps together and the stop test uses
 *       the mean error over the whole tensor (summed in fp64).
 *   R7  8-bit zero: one RTN (scale, zero) pair for the whole tensor from the
 *       min/max of the fp32 zero-points, cap as R1; W_q keeps the fp32 z.
 *   R8  packing: LSB-first bitstream along the group axis (layout below).
 *   R9  scale (= 1/s) and a 16-bit zero are stored as IEEE fp16.
 *   R10 element-wise arithmetic in fp32; every sum is accumulated in fp64.
 *   R13 W - W_r = W - (W_q - z)/s is evaluated as (fl(fl(W*s) + z) - W_q)/s:
 *       the same real number, from the residual of the rounding step (exact
 *       in fp32).
 *   R14 the group mean of W_q - (W - W_e)*s is evaluated as
 *       (sum W_q - sum fl((W - W_e)*s)) / g, both sums in fp64.
 *
 * Layout.  W is row-major [rows, cols].  axis = 1: group j holds the g
 * contiguous elements [j*g, (j+1)*g) of the flattened tensor (g | cols);
 * scale/zero are [rows, cols/g].  axis = 0: group j = (rb, c), j = rb*cols + c,
 * holds rows rb*g .. rb*g+g-1 of column c (g | rows); scale/zero are
 * [rows/g, cols].  Packed codes: axis = 1, element with flat index e occupies
 * bits [e*b, e*b+b) of one byte stream (bit k of byte B is stream bit 8B+k);
 * axis = 0, the stream runs down each column, byte R of column c is stored at
 * R*cols + c (packed shape [rows*b/8, cols]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_S_CAP 2.0e4f

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };
enum { ORACLE_STOP_GROUP = 0, ORACLE_STOP_TENSOR = 1, ORACLE_STOP_NONE = 2 };

/* ---- number formats: plain IEEE conversions --------------------------- */

static float from_f16(uint16_t h) { _Float16 x; memcpy(&x, &h, 2); return (float)x; }

static uint16_t to_f16(float f) { _Float16 x = (_Float16)f; uint16_t h; memcpy(&h, &x, 2); return h; }

static float from_bf16(uint16_t b) { uint32_t u = (uint32_t)b << 16; float f; memcpy(&f, &u, 4); return f; }

/* fp32 -> bf16, round to nearest, ties to even. */
static uint16_t to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float load_elem(const uint16_t *W, int dtype, int64_t idx)
{
    return dtype == ORACLE_BF16 ? from_bf16(W[idx]) : from_f16(W[idx]);
}

/* Flat index of element i of group j. */
static int64_t elem_index(int64_t j, int i, int64_t cols, int g, int axis)
{
    if (axis == 1) return j * g + i;
    int64_t rb = j / cols, c = j % cols;
    return (rb * g + i) * cols + c;
}

/* ---- the two sub-problems ---------------------------------------------- */

/* Sub-problem 1: generalised soft-thresholding, the proximal operator of the
 * lp term with weight 1/beta. */
float oracle_shrink(float x, float p, float beta)
{
    if (x == 0.0f) return 0.0f; /* R5 */
    float a = fabsf(x);
    float t = a - powf(a, p - 1.0f) / beta;
    if (!(t > 0.0f)) return 0.0f;
    return copysignf(t, x);
}

/* Initial scale and zero-point from the group's min and max (R1). */
static void init_scale_zero(const float *w, int g, int L, float *s_out, float *z_out)
{
    float mn = w[0], mx = w[0];
    for (int i = 1; i < g; ++i) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    float s = ORACLE_S_CAP;
    if (mx > mn) {
        s = (float)L / (mx - mn);
        if (s > ORACLE_S_CAP) s = ORACLE_S_CAP;
    }
    *s_out = s;
    *z_out = -mn * s;
}

/* W_q = clamp(round(W*s + z), 0, L) for one element (R2). */
static float quantize_elem(float w, float s, float z, int L)
{
    float ws = w * s;
    float v = ws + z;
    float q = nearbyintf(v);
    if (q < 0.0f) q = 0.0f;
    if (q > (float)L) q = (float)L;
    return q;
}

/* Quantise the group with zero-point z and return the sum of |W - W_r|^p (R3).
 * W - W_r = W - (W_q - z)/s = (W*s + z - W_q)/s: the residual of the rounding
 * step, which is exact in fp32, divided by s (R13).  q and d receive W_q and
 * W - W_r. */
static double evaluate(const float *w, int g, int L, float s, float z, float p, float *q, float *d)
{
    double acc = 0.0;
    for (int i = 0; i < g; ++i) {
        float ws = w[i] * s;
        float v = ws + z;
        float qi = nearbyintf(v);
        if (qi < 0.0f) qi = 0.0f;
        if (qi > (float)L) qi = (float)L;
        float r = v - qi;
        q[i] = qi;
        d[i] = r / s;
        acc += (double)powf(fabsf(d[i]), p);
    }
    return acc;
}

/* Sub-problem 2: W_e = shrink(W - W_r), then z = mean(W_q - (W - W_e)*s),
 * evaluated as mean(W_q) - mean((W - W_e)*s) with both sums in fp64 (R14). */
static float update_zero(const float *w, const float *q, const float *d, int g, float s, float p, float beta)
{
    double sq = 0.0, sws = 0.0;
    for (int i = 0; i < g; ++i) {
        float we = oracle_shrink(d[i], p, beta);
        float ws = (w[i] - we) * s;
        sq += (double)q[i];
        sws += (double)ws;
    }
    return (float)((sq - sws) / (double)g);
}

/* ---- one group, group-wise (or no) early stopping ------------------------ */

typedef struct {
    float s, zbest;
    double best_err; /* mean |W - W_r|^p of the kept zero-point */
    int best_iter;
} group_result;

static void solve_one_group(const float *w, int g, int L, float p, float beta0, float kappa, int iters,
                            int stop_mode, float *q, float *d, group_result *res)
{
    float s, z;
    init_scale_zero(w, g, L, &s, &z);
    double best = INFINITY;
    float zbest = z;
    int best_iter = 0;
    float beta = beta0;
    for (int it = 0; it < iters; ++it) {
        double e = evaluate(w, g, L, s, z, p, q, d) / (double)g;
        if (e < best) {
            best = e;
            zbest = z;
            best_iter = it;
        } else if (stop_mode == ORACLE_STOP_GROUP) {
            break; /* R4 */
        }
        z = update_zero(w, q, d, g, s, p, beta);
        beta = beta * kappa;
    }
    if (iters == 0) best = evaluate(w, g, L, s, z, p, q, d) / (double)g; /* reported only */
    res->s = s;
    res->zbest = zbest;
    res->best_err = best;
    res->best_iter = best_iter;
}

/* ---- packing (R8) -------------------------------------------------------- */

static void put_bits(uint8_t *stream_byte0, int64_t byte_stride, int64_t bitpos, unsigned level, int b)
{
    int64_t B = bitpos >> 3;
    int off = (int)(bitpos & 7);
    unsigned v = level << off; /* at most 8 + 7 bits */
    stream_byte0[B * byte_stride] |= (uint8_t)(v & 0xffu);
    if (off + b > 8) stream_byte0[(B + 1) * byte_stride] |= (uint8_t)(v >> 8);
}

static unsigned get_bits(const uint8_t *stream_byte0, int64_t byte_stride, int64_t bitpos, int b)
{
    int64_t B = bitpos >> 3;
    int off = (int)(bitpos & 7);
    unsigned v = stream_byte0[B * byte_stride];
    if (off + b > 8) v |= (unsigned)stream_byte0[(B + 1) * byte_stride] << 8;
    return (v >> off) & ((1u << b) - 1u);
}

/* Write the code of element (r, c) into the packed buffer (zeroed by caller). */
static void pack_elem(uint8_t *packed, int64_t r, int64_t c, int64_t cols, int b, int axis, unsigned level)
{
    if (axis == 1) put_bits(packed, 1, (r * cols + c) * b, level, b);
    else put_bits(packed + c, cols, r * b, level, b);
}

static unsigned unpack_elem(const uint8_t *packed, int64_t r, int64_t c, int64_t cols, int b, int axis)
{
    if (axis == 1) return get_bits(packed, 1, (r * cols + c) * b, b);
    return get_bits(packed + c, cols, r * b, b);
}

/* Pack a [rows, cols] array of levels (one byte each) in the library layout. */
void oracle_pack_levels(const uint8_t *levels, int64_t rows, int64_t cols, int nbits, int axis, uint8_t *packed)
{
    memset(packed, 0, (size_t)(rows * cols * nbits / 8));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) pack_elem(packed, r, c, cols, nbits, axis, levels[r * cols + c]);
}

void oracle_unpack_levels(const uint8_t *packed, int64_t rows, int64_t cols, int nbits, int axis, uint8_t *levels)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) levels[r * cols + c] = (uint8_t)unpack_elem(packed, r, c, cols, nbits, axis);
}

/* ---- the quantiser --------------------------------------------------------- */

static int valid_args(int64_t rows, int64_t cols, int dtype, int nbits, int g, int axis, int stop_mode, int zero_nbits)
{
    if (rows < 0 || cols < 0) return 0;
    if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return 0;
    if (!(nbits == 1 || nbits == 2 || nbits == 3 || nbits == 4 || nbits == 8)) return 0;
    if (g < 8 || g > 1024 || (g & (g - 1))) return 0;
    if (axis != 0 && axis != 1) return 0;
    if (axis == 1 && cols % g) return 0;
    if (axis == 0 && rows % g) return 0;
    if (stop_mode < 0 || stop_mode > 2) return 0;
    if (zero_nbits != 8 && zero_nbits != 16) return 0;
    return 1;
}

static int thread_count(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Write one group's codes into the packed buffer using zero-point z. */
static void store_codes(const float *w, int64_t j, int g, int L, float s, float z, int64_t cols, int nbits, int axis,
                        uint8_t *packed)
{
    for (int i = 0; i < g; ++i) {
        int64_t e = elem_index(j, i, cols, g, axis);
        unsigned level = (unsigned)quantize_elem(w[i], s, z, L);
        pack_elem(packed, e / cols, e % cols, cols, nbits, axis, level);
    }
}

/*
 * Quantise W.  Outputs (all host memory, caller-owned):
 *   W_q_packed  uint8[rows*cols*nbits/8]
 *   scale       fp16[G]  (= 1/s)
 *   zero        fp16[G] (zero_nbits 16) or uint8[G] (zero_nbits 8)
 *   zero_meta   fp32[2] = (1/sz, zz) for zero_nbits 8, else unused (may be NULL)
 *   best_iter   int32[G] or NULL: index of the kept iterate
 *   best_err    fp32[G]  or NULL: mean |W - W_r|^p of the kept zero-point
 *   zero_f32    fp32[G]  or NULL: the kept zero-point before storage
 * Packing is done serially (several groups share bytes for axis = 0).
 * Returns 0 on success, 1 on an invalid argument, 2 on an allocation failure.
 */
int oracle_quantize(const uint16_t *W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size, int axis,
                    float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits, uint8_t *W_q_packed,
                    uint16_t *scale, void *zero, float *zero_meta, int32_t *best_iter, float *best_err,
                    float *zero_f32, int nthreads)
{
    if (!valid_args(rows, cols, dtype, nbits, group_size, axis, stop_mode, zero_nbits) || iters < 0) return 1;
    const int g = group_size, L = (1 << nbits) - 1;
    const int64_t G = rows * cols / g;
    const int nth = thread_count(nthreads);
    float *s_all = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
    float *zb_all = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
    if (!s_all || !zb_all) { free(s_all); free(zb_all); return 2; }
    memset(W_q_packed, 0, (size_t)(rows * cols * nbits / 8));

    if (stop_mode != ORACLE_STOP_TENSOR) {
#pragma omp parallel num_threads(nth)
        {
            float *w = (float *)malloc(sizeof(float) * (size_t)g * 3);
            float *q = w + g, *d = w + 2 * g;
#pragma omp for schedule(dynamic, 256)
            for (int64_t j = 0; j < G; ++j) {
                for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
                group_result res;
                solve_one_group(w, g, L, p, beta, kappa, iters, stop_mode, q, d, &res);
                s_all[j] = res.s;
                zb_all[j] = res.zbest;
                if (best_iter) best_iter[j] = res.best_iter;
                if (best_err) best_err[j] = (float)res.best_err;
            }
            free(w);
        }
    } else {
        /* R6: all groups step together; the stop test uses the tensor mean. */
        float *z = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
        float *znext = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
        double *gerr = (double *)malloc(sizeof(double) * (size_t)(G ? G : 1));
        double *gbest = (double *)malloc(sizeof(double) * (size_t)(G ? G : 1));
        if (!z || !znext || !gerr || !gbest) { free(z); free(znext); free(gerr); free(gbest); free(s_all); free(zb_all); return 2; }
#pragma omp parallel num_threads(nth)
        {
            float *w = (float *)malloc(sizeof(float) * (size_t)g);
#pragma omp for schedule(static)
            for (int64_t j = 0; j < G; ++j) {
                for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
                init_scale_zero(w, g, L, &s_all[j], &z[j]);
                zb_all[j] = z[j];
            }
            free(w);
        }
        double best = INFINITY;
        int bi = 0;
        float bt = beta;
        for (int it = 0; it < iters; ++it) {
#pragma omp parallel num_threads(nth)
            {
                float *w = (float *)malloc(sizeof(float) * (size_t)g * 3);
                float *q = w + g, *d = w + 2 * g;
#pragma omp for schedule(dynamic, 256)
                for (int64_t j = 0; j < G; ++j) {
                    for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
                    gerr[j] = evaluate(w, g, L, s_all[j], z[j], p, q, d);
                    znext[j] = update_zero(w, q, d, g, s_all[j], p, bt);
                }
                free(w);
            }
            double total = 0.0;
            for (int64_t j = 0; j < G; ++j) total += gerr[j];
            double e = G ? total / (double)(G * g) : 0.0;
            if (!(e < best)) break; /* R4 applied to the tensor mean */
            best = e;
            bi = it;
            for (int64_t j = 0; j < G; ++j) { zb_all[j] = z[j]; gbest[j] = gerr[j] / (double)g; }
            for (int64_t j = 0; j < G; ++j) z[j] = znext[j];
            bt = bt * kappa;
        }
        if (iters == 0) {
            float *w = (float *)malloc(sizeof(float) * (size_t)g * 3);
            for (int64_t j = 0; j < G; ++j) {
                for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
                gbest[j] = evaluate(w, g, L, s_all[j], z[j], p, w + g, w + 2 * g) / (double)g;
            }
            free(w);
        }
        for (int64_t j = 0; j < G; ++j) {
            if (best_iter) best_iter[j] = bi;
            if (best_err) best_err[j] = (float)gbest[j];
        }
        free(z); free(znext); free(gerr); free(gbest);
    }

    /* Final codes with the kept zero-point, then scale and zero storage. */
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)g);
        for (int64_t j = 0; j < G; ++j) {
            for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
            store_codes(w, j, g, L, s_all[j], zb_all[j], cols, nbits, axis, W_q_packed);
            scale[j] = to_f16(1.0f / s_all[j]);
            if (zero_f32) zero_f32[j] = zb_all[j];
        }
        free(w);
    }
    if (zero_nbits == 16) {
        uint16_t *z16 = (uint16_t *)zero;
        for (int64_t j = 0; j < G; ++j) z16[j] = to_f16(zb_all[j]);
    } else {
        /* R7: one RTN pair for the whole tensor. */
        uint8_t *z8 = (uint8_t *)zero;
        float zmn = G ? zb_all[0] : 0.0f, zmx = zmn;
        for (int64_t j = 1; j < G; ++j) {
            if (zb_all[j] < zmn) zmn = zb_all[j];
            if (zb_all[j] > zmx) zmx = zb_all[j];
        }
        float sz = ORACLE_S_CAP;
        if (zmx > zmn) {
            sz = 255.0f / (zmx - zmn);
            if (sz > ORACLE_S_CAP) sz = ORACLE_S_CAP;
        }
        float zz = -zmn * sz;
        for (int64_t j = 0; j < G; ++j) z8[j] = (uint8_t)quantize_elem(zb_all[j], sz, zz, 255);
        zero_meta[0] = 1.0f / sz;
        zero_meta[1] = zz;
    }
    free(s_all);
    free(zb_all);
    return 0;
}

/*
 * Dequantise: W_r = (W_q - zero) * scale in fp32, cast to out_dtype.  With
 * zero_nbits = 8 the zero is first rebuilt as (zq - zz) * (1/sz).
 */
/*
 * Dequantise: W_r = (W_q - zero) * scale per element, in fp32, then rounded to
 * the output dtype.  The scale of group j is either the stored fp16 value
 * (scale_meta == NULL) or, for the "_s*" variant, rebuilt from its 8-bit code:
 * (code - zc) * (1/sc) with the pair of its scale group j / scale_group.
 */
static int dequantize_impl(const uint8_t *W_q_packed, const void *scale, const float *scale_meta, int scale_group,
                           const void *zero, const float *zero_meta, int64_t rows, int64_t cols, int nbits,
                           int group_size, int axis, int zero_nbits, int out_dtype, uint16_t *W_out)
{
    if (!valid_args(rows, cols, out_dtype, nbits, group_size, axis, 0, zero_nbits)) return 1;
    if (scale_meta && scale_group < 1) return 1;
    const int g = group_size;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            int64_t j = axis == 1 ? (r * cols + c) / g : (r / g) * cols + c;
            float q = (float)unpack_elem(W_q_packed, r, c, cols, nbits, axis);
            float z;
            if (zero_nbits == 16) z = from_f16(((const uint16_t *)zero)[j]);
            else z = ((float)((const uint8_t *)zero)[j] - zero_meta[1]) * zero_meta[0];
            float sc;
            if (scale_meta == NULL) {
                sc = from_f16(((const uint16_t *)scale)[j]);
            } else {
                const float *m = scale_meta + 2 * (j / scale_group);
                sc = ((float)((const uint8_t *)scale)[j] - m[1]) * m[0];
            }
            float v = (q - z) * sc;
            W_out[r * cols + c] = out_dtype == ORACLE_BF16 ? to_bf16(v) : to_f16(v);
        }
    }
    return 0;
}

int oracle_dequantize(const uint8_t *W_q_packed, const uint16_t *scale, const void *zero, const float *zero_meta,
                      int64_t rows, int64_t cols, int nbits, int group_size, int axis, int zero_nbits, int out_dtype,
                      uint16_t *W_out)
{
    return dequantize_impl(W_q_packed, scale, NULL, 0, zero, zero_meta, rows, cols, nbits, group_size, axis,
                           zero_nbits, out_dtype, W_out);
}

int oracle_dequantize_s8(const uint8_t *W_q_packed, const uint8_t *scale_q, const float *scale_meta, int scale_group,
                         const void *zero, const float *zero_meta, int64_t rows, int64_t cols, int nbits,
                         int group_size, int axis, int zero_nbits, int out_dtype, uint16_t *W_out)
{
    if (scale_meta == NULL) return 1;
    return dequantize_impl(W_q_packed, scale_q, scale_meta, scale_group, zero, zero_meta, rows, cols, nbits,
                           group_size, axis, zero_nbits, out_dtype, W_out);
}

/*
 * Fused consumer of the packed layout (the step after quantisation: the
 * inference backends of "Weight-only quantization without the calibration
 * tax" dequantise W_q and multiply): y[b][r] = sum_c W_r[r][c] * x[b][c] for a
 * batch of activation vectors, with W_r = (W_q - zero) * scale rebuilt per
 * element exactly as oracle_dequantize does before its final rounding (fp32),
 * and every product and sum in fp64.  Groups along the input dimension
 * (axis 1).  x: [batch][cols] fp16/bf16 bits; y: [batch][rows] fp64.
 */
int oracle_gemv(const uint8_t *W_q_packed, const uint16_t *scale, const void *zero, const float *zero_meta,
                int64_t rows, int64_t cols, int nbits, int group_size, int zero_nbits, const uint16_t *x,
                int x_dtype, int batch, double *y)
{
    if (!valid_args(rows, cols, x_dtype, nbits, group_size, 1, 0, zero_nbits) || batch < 1) return 1;
    const int g = group_size;
    for (int b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r) y[b * rows + r] = 0.0;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t j = (r * cols + c) / g;
            const float q = (float)unpack_elem(W_q_packed, r, c, cols, nbits, 1);
            float z;
            if (zero_nbits == 16) z = from_f16(((const uint16_t *)zero)[j]);
            else z = ((float)((const uint8_t *)zero)[j] - zero_meta[1]) * zero_meta[0];
            const float w = (q - z) * from_f16(scale[j]);
            for (int b = 0; b < batch; ++b) y[b * rows + r] += (double)w * (double)load_elem(x + b * cols, x_dtype, c);
        }
    }
    return 0;
}

/*
 * The same product as a tensor-core backend forms it (the consumer of the
 * packed layout: "HQQ - Half-Quadratic Quantization" (skill4agent.com),
 * section "Backends"): W_r rebuilt per element exactly as in
 * oracle_gemv (fp32), then rounded to the activations' 16-bit type (x_dtype;
 * round to nearest, ties to even) because both operands of a 16-bit
 * tensor-core product share one type; every product and sum in fp64.
 * yabs[b][r] receives the sum of |w16 * x| over the row (the scale of a
 * bound on fp32 accumulation error).  Groups along the input dimension.
 */
int oracle_gemm(const uint8_t *W_q_packed, const uint16_t *scale, const void *zero, const float *zero_meta,
                int64_t rows, int64_t cols, int nbits, int group_size, int zero_nbits, const uint16_t *x,
                int x_dtype, int batch, double *y, double *yabs)
{
    if (!valid_args(rows, cols, x_dtype, nbits, group_size, 1, 0, zero_nbits) || batch < 1) return 1;
    const int g = group_size;
    for (int64_t i = 0; i < (int64_t)batch * rows; ++i) {
        y[i] = 0.0;
        yabs[i] = 0.0;
    }
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t grp = (r * cols + c) / g;
            const float q = (float)unpack_elem(W_q_packed, r, c, cols, nbits, 1);
            float z;
            if (zero_nbits == 16) z = from_f16(((const uint16_t *)zero)[grp]);
            else z = ((float)((const uint8_t *)zero)[grp] - zero_meta[1]) * zero_meta[0];
            const float wr = (q - z) * from_f16(scale[grp]);
            const double w16 = x_dtype == ORACLE_BF16 ? (double)from_bf16(to_bf16(wr)) : (double)from_f16(to_f16(wr));
            for (int b = 0; b < batch; ++b) {
                const double p = w16 * (double)load_elem(x + b * cols, x_dtype, c);
                y[b * rows + r] += p;
                yabs[b * rows + r] += fabs(p);
            }
        }
    }
    return 0;
}

/*
 * The "_s*" variant of the Llama-2 table ("Benchmark results"/"Llama-2",
 * footnote of the table): the scale is also quantised to 8 bit, with a group
 * size of 128.  Reading R15: the quantity quantised is the stored fp16 scale
 * (the dequantisation multiplier 1/s); its G values, in group order, are cut
 * into runs of scale_group consecutive values (the last run may be shorter);
 * each run gets one round-to-nearest quantiser from its min and max:
 *   sc = 255 / (max - min)  (1 when max == min),  zc = -min * sc,
 *   code = clamp(round_half_even(scale * sc + zc), 0, 255),
 *   stored meta per run: (1/sc, zc) in fp32, and the scale is rebuilt as
 *   (code - zc) * (1/sc).
 * No cap on sc is needed: two distinct fp16 values differ by at least 2^-24.
 */
int oracle_quantize_scale8(const uint16_t *scale, int64_t G, int scale_group, uint8_t *codes, float *meta)
{
    if (G < 0 || scale_group < 1) return 1;
    for (int64_t k0 = 0; k0 < G; k0 += scale_group) {
        const int64_t k1 = k0 + scale_group < G ? k0 + scale_group : G;
        float mn = from_f16(scale[k0]), mx = mn;
        for (int64_t i = k0 + 1; i < k1; ++i) {
            const float v = from_f16(scale[i]);
            if (v < mn) mn = v;
            if (v > mx) mx = v;
        }
        const float sc = mx > mn ? 255.0f / (mx - mn) : 1.0f;
        const float zc = -mn * sc;
        for (int64_t i = k0; i < k1; ++i) {
            float c = nearbyintf(from_f16(scale[i]) * sc + zc);
            c = c < 0.0f ? 0.0f : (c > 255.0f ? 255.0f : c);
            codes[i] = (uint8_t)c;
        }
        meta[2 * (k0 / scale_group)] = 1.0f / sc;
        meta[2 * (k0 / scale_group) + 1] = zc;
    }
    return 0;
}

/*
 * Trace one group (fp32 values) through `iters` iterations with no early
 * stop.  Records, for iterate k: the zero-point z_k, the mean lp error e_k of
 * z_k, and beta_k (the beta used by the shrink that produces z_{k+1}).
 */
int oracle_trace_group(const float *w, int g, int nbits, float p, float beta0, float kappa, int iters, float *s_out,
                       float *z_traj, double *e_traj, float *beta_traj)
{
    if (g < 1 || iters < 0) return 1;
    const int L = (1 << nbits) - 1;
    float *q = (float *)malloc(sizeof(float) * (size_t)g * 2);
    float *d = q + g;
    float s, z;
    init_scale_zero(w, g, L, &s, &z);
    float beta = beta0;
    for (int it = 0; it < iters; ++it) {
        z_traj[it] = z;
        e_traj[it] = evaluate(w, g, L, s, z, p, q, d) / (double)g;
        beta_traj[it] = beta;
        z = update_zero(w, q, d, g, s, p, beta);
        beta = beta * kappa;
    }
    *s_out = s;
    free(q);
    return 0;
}

/* Codes W_q of one group for a given zero-point (used to re-check groups
 * whose stop decision was a near tie). */
void oracle_group_codes(const float *w, int g, int nbits, float s, float z, uint8_t *levels)
{
    const int L = (1 << nbits) - 1;
    for (int i = 0; i < g; ++i) levels[i] = (uint8_t)quantize_elem(w[i], s, z, L);
}

/* The z update alone (sub-problem 2 given W_q), exposed for its pin. */
float oracle_update_zero(const float *w, const float *q, const float *d, int g, float s, float p, float beta)
{
    return update_zero(w, q, d, g, s, p, beta);
}

/* Quantise an explicit list of groups (group mode or no early stop only).
 * Per listed group: levels[n*g] (codes in group order), s, zbest, best_iter,
 * best_err.  Lets tests check large tensors on a sample of groups. */
int oracle_quantize_groups(const uint16_t *W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size,
                           int axis, float p, float beta, float kappa, int iters, int stop_mode,
                           const int64_t *group_ids, int64_t n, uint8_t *levels, float *s_out, float *zbest_out,
                           int32_t *best_iter, float *best_err, int nthreads)
{
    if (!valid_args(rows, cols, dtype, nbits, group_size, axis, stop_mode, 16) || iters < 0) return 1;
    if (stop_mode == ORACLE_STOP_TENSOR) return 1;
    const int g = group_size, L = (1 << nbits) - 1;
    const int nth = thread_count(nthreads);
#pragma omp parallel num_threads(nth)
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)g * 3);
        float *q = w + g, *d = w + 2 * g;
#pragma omp for schedule(dynamic, 16)
        for (int64_t k = 0; k < n; ++k) {
            int64_t j = group_ids[k];
            for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
            group_result res;
            solve_one_group(w, g, L, p, beta, kappa, iters, stop_mode, q, d, &res);
            for (int i = 0; i < g; ++i) levels[k * g + i] = (uint8_t)quantize_elem(w[i], res.s, res.zbest, L);
            s_out[k] = res.s;
            zbest_out[k] = res.zbest;
            best_iter[k] = res.best_iter;
            best_err[k] = (float)res.best_err;
        }
        free(w);
    }
    return 0;
}

/* ==== the half-precision solver variant ====================================
 *
 * The pages run the solver on the GPU in half precision ("Speed: from hours
 * to minutes"), with the steps of "Outlier-aware optimization without
 * gradients".  Reading H (this library's restatement of "half precision" for
 * the steps of the solver above; h(x) rounds x to fp16, to nearest, ties to
 * even):
 *   H1 input fp16 only.
 *   H2 s = h(min(L/(max - min), 2e4)) from the fp32 quotient (R1);
 *      z0 = h(-min * s).
 *   H3 ws = h(w*s); v = h(ws + z); W_q = clamp(round_half_even(v), 0, L);
 *      r = h(v - W_q).
 *   H4 the lp error of z is s^-p/g times the exact sum of the terms
 *      h(|r|^p); the stop rule (R4) compares these sums within the group.
 *   H5 proximal step: d = h(fl32(r / s)), W_e = h(shrink(d)) with the shrink
 *      in fp32 (oracle_shrink); z' = h((sum W_q - sum h(h(w - W_e) * s)) / g),
 *      both sums exact.
 *   H6 beta, the stop modes group and none, the kept iterate and the 8-bit
 *      zero (R7, from the fp16 zero-points): as the fp32 solver.  Outputs:
 *      codes clamp(round(h(h(w*s) + z*)), 0, L), scale h(fl32(1/s)), zero z*.
 * Every product of two fp16 values and every sum of two is exact in fp64, so
 * each h() below rounds an exact value once.
 */

static float h16(double x) { return (float)(_Float16)x; }

/* H6: the stored zero-points -- fp16, or R7's 8-bit quantiser over the tensor. */
static void store_zero_half(const float *zb, int64_t G, int zero_nbits, void *zero, float *zero_meta)
{
    if (zero_nbits == 16) {
        uint16_t *z16 = (uint16_t *)zero;
        for (int64_t j = 0; j < G; ++j) z16[j] = to_f16(zb[j]);
        return;
    }
    uint8_t *z8 = (uint8_t *)zero;
    float zmn = G ? zb[0] : 0.0f, zmx = zmn;
    for (int64_t j = 1; j < G; ++j) {
        if (zb[j] < zmn) zmn = zb[j];
        if (zb[j] > zmx) zmx = zb[j];
    }
    float sz = ORACLE_S_CAP;
    if (zmx > zmn) {
        sz = 255.0f / (zmx - zmn);
        if (sz > ORACLE_S_CAP) sz = ORACLE_S_CAP;
    }
    float zz = -zmn * sz;
    for (int64_t j = 0; j < G; ++j) z8[j] = (uint8_t)quantize_elem(zb[j], sz, zz, 255);
    zero_meta[0] = 1.0f / sz;
    zero_meta[1] = zz;
}

static void init_half(const float *w, int g, int L, float *s_out, float *z_out)
{
    float mn = w[0], mx = w[0];
    for (int i = 1; i < g; ++i) {
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
    }
    float s = ORACLE_S_CAP;
    if (mx > mn) {
        s = (float)L / (mx - mn);
        if (s > ORACLE_S_CAP) s = ORACLE_S_CAP;
    }
    s = h16(s);
    *s_out = s;
    *z_out = h16(-(double)mn * (double)s);
}

/* H3: the code of one element at zero-point z. */
static float quantize_half(float w, float s, float z, int L)
{
    float ws = h16((double)w * (double)s);
    float v = h16((double)ws + (double)z);
    float q = nearbyintf(v);
    if (q < 0.0f) q = 0.0f;
    if (q > (float)L) q = (float)L;
    return q;
}

/* H3, H4: codes, residuals and the exact sum of the rounded terms |r|^p. */
static double evaluate_half(const float *w, int g, int L, float s, float z, float p, float *q, float *r)
{
    double acc = 0.0;
    for (int i = 0; i < g; ++i) {
        float ws = h16((double)w[i] * (double)s);
        float v = h16((double)ws + (double)z);
        float qi = nearbyintf(v);
        if (qi < 0.0f) qi = 0.0f;
        if (qi > (float)L) qi = (float)L;
        q[i] = qi;
        r[i] = h16((double)v - (double)qi);
        acc += (double)h16(pow(fabs((double)r[i]), (double)p));
    }
    return acc;
}

/* H5: the z update from the codes and residuals. */
static float update_zero_half(const float *w, const float *q, const float *r, int g, float s, float p, float beta)
{
    double sq = 0.0, sws = 0.0;
    for (int i = 0; i < g; ++i) {
        float d = h16((double)(r[i] / s));
        float we = h16((double)oracle_shrink(d, p, beta));
        float ws = h16((double)h16((double)w[i] - (double)we) * (double)s);
        sq += (double)q[i];
        sws += (double)ws;
    }
    return h16((sq - sws) / (double)g);
}

static void solve_one_group_half(const float *w, int g, int L, float p, float beta0, float kappa, int iters,
                                 int stop_mode, float *q, float *r, group_result *res)
{
    float s, z;
    init_half(w, g, L, &s, &z);
    double best = INFINITY;
    float zbest = z;
    int best_iter = 0;
    float beta = beta0;
    for (int it = 0; it < iters; ++it) {
        double e = evaluate_half(w, g, L, s, z, p, q, r);
        if (e < best) {
            best = e;
            zbest = z;
            best_iter = it;
        } else if (stop_mode == ORACLE_STOP_GROUP) {
            break;
        }
        z = update_zero_half(w, q, r, g, s, p, beta);
        beta = beta * kappa;
    }
    if (iters == 0) best = evaluate_half(w, g, L, s, z, p, q, r);
    res->s = s;
    res->zbest = zbest;
    res->best_err = best * pow((double)s, -(double)p) / (double)g;
    res->best_iter = best_iter;
}

/*
 * The half-precision variant of oracle_quantize: fp16 input (dtype must be
 * ORACLE_F16), group or no stop, either axis; outputs as oracle_quantize
 * (zero_f32 receives the fp16 zero-points).  Returns 0, or 1 on an invalid
 * argument, 2 on an allocation failure.
 */
int oracle_quantize_half(const uint16_t *W, int64_t rows, int64_t cols, int dtype, int nbits, int group_size,
                         int axis, float p, float beta, float kappa, int iters, int stop_mode, int zero_nbits,
                         uint8_t *W_q_packed, uint16_t *scale, void *zero, float *zero_meta, int32_t *best_iter,
                         float *best_err, float *zero_f32, int nthreads)
{
    if (!valid_args(rows, cols, dtype, nbits, group_size, axis, stop_mode, zero_nbits) || iters < 0) return 1;
    if (dtype != ORACLE_F16 || stop_mode == ORACLE_STOP_TENSOR) return 1;
    const int g = group_size, L = (1 << nbits) - 1;
    const int64_t G = rows * cols / g;
    const int nth = thread_count(nthreads);
    float *s_all = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
    float *zb_all = (float *)malloc(sizeof(float) * (size_t)(G ? G : 1));
    if (!s_all || !zb_all) { free(s_all); free(zb_all); return 2; }
    memset(W_q_packed, 0, (size_t)(rows * cols * nbits / 8));
#pragma omp parallel num_threads(nth)
    {
        float *w = (float *)malloc(sizeof(float) * (size_t)g * 3);
        float *q = w + g, *r = w + 2 * g;
#pragma omp for schedule(dynamic, 256)
        for (int64_t j = 0; j < G; ++j) {
            for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
            group_result res;
            solve_one_group_half(w, g, L, p, beta, kappa, iters, stop_mode, q, r, &res);
            s_all[j] = res.s;
            zb_all[j] = res.zbest;
            if (best_iter) best_iter[j] = res.best_iter;
            if (best_err) best_err[j] = (float)res.best_err;
        }
        free(w);
    }
    float *w = (float *)malloc(sizeof(float) * (size_t)g);
    for (int64_t j = 0; j < G; ++j) {
        for (int i = 0; i < g; ++i) w[i] = load_elem(W, dtype, elem_index(j, i, cols, g, axis));
        for (int i = 0; i < g; ++i) {
            int64_t e = elem_index(j, i, cols, g, axis);
            pack_elem(W_q_packed, e / cols, e % cols, cols, nbits, axis,
                      (unsigned)quantize_half(w[i], s_all[j], zb_all[j], L));
        }
        scale[j] = to_f16(1.0f / s_all[j]);
        if (zero_f32) zero_f32[j] = zb_all[j];
    }
    free(w);
    store_zero_half(zb_all, G, zero_nbits, zero, zero_meta);
    free(s_all);
    free(zb_all);
    return 0;
}

/* Trace one fp16 group (values as floats) through `iters` iterations of the
 * half-precision variant without early stop: z_k, the error of z_k (H4, mean
 * form) and beta_k, as oracle_trace_group. */
int oracle_trace_group_half(const float *w, int g, int nbits, float p, float beta0, float kappa, int iters,
                            float *s_out, float *z_traj, double *e_traj, float *beta_traj)
{
    if (g < 1 || iters < 0) return 1;
    const int L = (1 << nbits) - 1;
    float *q = (float *)malloc(sizeof(float) * (size_t)g * 2);
    float *r = q + g;
    float s, z;
    init_half(w, g, L, &s, &z);
    float beta = beta0;
    for (int it = 0; it < iters; ++it) {
        z_traj[it] = z;
        e_traj[it] = evaluate_half(w, g, L, s, z, p, q, r) * pow((double)s, -(double)p) / (double)g;
        beta_traj[it] = beta;
        z = update_zero_half(w, q, r, g, s, p, beta);
        beta = beta * kappa;
    }
    *s_out = s;
    free(q);
    return 0;
}

/* Codes of one group of the half-precision variant for a given zero-point. */
void oracle_group_codes_half(const float *w, int g, int nbits, float s, float z, uint8_t *levels)
{
    const int L = (1 << nbits) - 1;
    for (int i = 0; i < g; ++i) levels[i] = (uint8_t)quantize_half(w[i], s, z, L);
}
