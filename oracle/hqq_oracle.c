/*
 * hqq_oracle.c -- plain CPU oracle for HQQ group-wise weight quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__.py and the
 * CPU-baseline leg of bench.py may load this library.  The CUDA library never links,
 * includes or calls anything here, and nothing here calls the CUDA library.
 *
 * What it computes, and where each step comes from.  The source is the web page
 * "HQQ 算法解读：不用校准数据，怎样把大模型权重压到 4 bit"
 * (ludovicoyin.github.io/blog/posts/hqq-half-quadratic-quantization), cited below as
 * [HQQ 算法解读, <section>]:
 *
 *   group view ........ [HQQ 算法解读, "`axis` 不是一个无关紧要的开关"] (reshape [-1, g] / [g, -1])
 *   quantize formula .. [HQQ 算法解读, "量化公式：把尺子写出来"]  q = clip(round(W*s+z), 0, 2^b-1),
 *                       W_hat = (q - z)/s, metadata Delta = 1/s, dequant (q - z)*Delta
 *   min-max init ...... [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"]
 *                       s0 = (2^b-1)/(max-min), z0 = -min*s0; s = 1 for a tiny denominator,
 *                       then s clamped below 2e4
 *   proximal loop ..... [HQQ 算法解读, "第二拍：half-quadratic 迭代修正零点"]
 *                       quantize -> reconstruct -> e = shrink(W - W_hat) (p = 0.7, beta = 10,
 *                       beta *= 1.01 per round) -> z = mean(q - (W - e)*s); stop and revert
 *                       when the reconstruction MAE is not better than the best so far;
 *                       quantize once more with the original W
 *   packing ........... [HQQ 算法解读, "为什么一定要分组"] two 4-bit codes per byte, four 2-bit
 *                       codes per byte, ten 3-bit codes per 32-bit word; 5- and 6-bit codes one
 *                       per byte
 *   forward product ... [HQQ 算法解读, "从压缩文件到一次前向"] unpack -> (q - zero)*scale ->
 *                       x @ W_hat.T (hqo_gemv, one input vector)
 *
 * Readings taken where the page is silent (each is also listed in the design notes):
 *   - arithmetic is IEEE binary32, round-to-nearest-even, every product and sum rounded
 *     separately (built with -ffp-contract=off); W is converted exactly from fp16;
 *   - "round" is round-half-to-even; a zero code is +0;
 *   - "denominator too small" means max-min < eps_tiny (a parameter, 1e-4 by default);
 *   - z0 is written 0 - min*s0 so that a zero minimum gives +0;
 *   - the shrink operator is the generalized lp soft threshold of the HQQ paper
 *     (Badri et al. 2023, cited at the end of the page):
 *         e = sign(r) * max(|r| - |r|^(p-1) / beta, 0),
 *     evaluated in binary64 and rounded once to binary32; e = 0 at r = 0;
 *   - beta_i = beta * kappa^i formed by repeated binary64 multiplication;
 *   - the group sums (the mean for z, and the per-group sum of |W - W_hat|) are binary32
 *     pairwise sums: the elements, in index order and padded with +0 up to the next power
 *     of two, are summed as (sum of the first half) + (sum of the second half),
 *     recursively; the mean divides that sum by g;
 *   - the tensor-wide MAE is compared exactly: each group's binary32 error sum is
 *     truncated to a multiple of 2^-32 (an integer), and those integers are added in
 *     128-bit arithmetic, so the comparison does not depend on summation order;
 *   - "better" means strictly smaller; iteration i is measured with the z it starts
 *     from (z_i); when iteration i is accepted z_i becomes the kept zero; the kept zero
 *     after the loop is the one whose MAE was best (never an unmeasured z);
 *   - codes are packed in flat row-major order for both axes, lowest index in the
 *     lowest bits; the tail of the last byte or word is zero;
 *   - 7- and 8-bit codes are stored one per byte like 5 and 6 bits; 1-bit codes, which the
 *     pages name only in passing, are packed eight per byte like the 2- and 4-bit codes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------
 * binary16 <-> binary32, written from the IEEE 754 binary16 format (1 sign bit, 5 exponent
 * bits with bias 15, 10 fraction bits; exponent 0 = zero/subnormal, 31 = inf/NaN).
 * ---------------------------------------------------------------------------------- */
float hqo_half_to_float(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    float mag;
    if (expo == 0)
        mag = ldexpf((float)frac, -24);                 /* frac * 2^-24, exact */
    else if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexpf((float)(frac | 0x400), expo - 25); /* 1.frac * 2^(expo-15), exact */
    return sign ? -mag : mag;
}

uint16_t hqo_float_to_half(float f)
{
    /* round-to-nearest-even onto the binary16 grid */
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    float a = fabsf(f);
    if (isnan(f))
        return sign | 0x7e00;
    if (a >= 65520.0f)                     /* halfway above 65504 and beyond: rounds to inf */
        return sign | 0x7c00;
    if (a < ldexpf(1.0f, -14)) {           /* subnormal range: grid step 2^-24 */
        float m = rintf(ldexpf(a, 24));    /* exact scaling, RNE to an integer 0..1024 */
        return sign | (uint16_t)m;         /* m == 1024 is the smallest normal, same bits */
    }
    int e;
    frexpf(a, &e);                         /* a = m * 2^e, m in [0.5, 1) */
    int expo = e - 1;                      /* a in [2^expo, 2^(expo+1)) */
    float m = rintf(ldexpf(a, 10 - expo)); /* significand scaled to [1024, 2048], RNE */
    if (m >= 2048.0f) {                    /* rounded up into the next binade */
        m = 1024.0f;
        expo += 1;
    }
    if (expo > 15)
        return sign | 0x7c00;
    return sign | (uint16_t)(((expo + 15) << 10) | ((int)m - 1024));
}

/* ------------------------------------------------------------------------------------
 * Group view [HQQ 算法解读, "`axis` 不是一个无关紧要的开关"]:
 *   axis = 1: W.reshape([-1, g]) -> group k holds flat elements k*g .. k*g + g - 1;
 *   axis = 0: W.reshape([g, -1]) -> group k is column k of the [g, G] view, i.e. flat
 *             elements j*G + k for j = 0 .. g-1, with G = N / g.
 * ---------------------------------------------------------------------------------- */
static int64_t elem_index(int64_t k, int64_t j, int64_t g, int64_t G, int axis)
{
    return axis == 1 ? k * g + j : j * G + k;
}

/* Min-max initialisation of one group [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"]. */
void hqo_minmax_init(const float *w, int64_t g, int nbits, float eps_tiny, float scale_max,
                     float *s_out, float *z_out)
{
    float mn = w[0], mx = w[0];
    for (int64_t j = 1; j < g; j++) {
        if (w[j] < mn) mn = w[j];
        if (w[j] > mx) mx = w[j];
    }
    float qmax = (float)((1 << nbits) - 1);
    float d = mx - mn;
    float s = (d < eps_tiny) ? 1.0f : qmax / d;
    if (s > scale_max) s = scale_max;
    *s_out = s;
    *z_out = 0.0f - mn * s;
}

/* q = clip(round(t), 0, 2^b - 1) with round-half-to-even [HQQ 算法解读, "量化公式"]. */
static float quant_code(float w, float s, float z, float qmax)
{
    float t = w * s + z;                   /* two roundings: -ffp-contract=off */
    float q = rintf(t);
    if (!(q > 0.0f)) q = 0.0f;
    if (q > qmax) q = qmax;
    return q;
}

/* Generalized lp shrink of a residual (reading of the page's "shrink 算子"). */
float hqo_shrink(float r, double beta, double p)
{
    double a = fabs((double)r);
    if (a == 0.0)
        return 0.0f;
    double m = a - pow(a, p - 1.0) / beta;
    if (!(m > 0.0))
        return 0.0f;
    float mf = (float)m;
    return r < 0.0f ? -mf : mf;
}

/* hqo_shrink over an array (test convenience: one call instead of n). */
void hqo_shrink_n(const float *r, int64_t n, double beta, double p, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = hqo_shrink(r[i], beta, p);
}

/* Pairwise sum of x[lo .. lo+len) with len a power of two; slots at or beyond n are +0. */
static float pairwise(const float *x, int64_t n, int64_t lo, int64_t len)
{
    if (len == 1)
        return lo < n ? x[lo] : 0.0f;
    return pairwise(x, n, lo, len / 2) + pairwise(x, n, lo + len / 2, len / 2);
}

float hqo_pairwise_sum(const float *x, int64_t n)
{
    int64_t len = 1;
    while (len < n) len *= 2;
    return pairwise(x, n, 0, len);
}

/*
 * One pass of the proximal loop over one group [HQQ 算法解读, "第二拍"]:
 *   q = clip(round(W*s + z)); W_hat = (q - z)/s; e = shrink(W - W_hat, beta);
 *   z_new = mean(q - (W - e)*s);  err = sum |W - W_hat|  (both sums pairwise).
 */
void hqo_group_pass(const float *w, int64_t g, int nbits, float s, float z, double beta,
                    double p, uint8_t *q_out, float *err_out, float *znew_out)
{
    float qmax = (float)((1 << nbits) - 1);
    float *term = (float *)malloc(sizeof(float) * (size_t)g);
    float *absr = (float *)malloc(sizeof(float) * (size_t)g);
    for (int64_t j = 0; j < g; j++) {
        float q = quant_code(w[j], s, z, qmax);
        float w_hat = (q - z) / s;
        float r = w[j] - w_hat;
        float e = hqo_shrink(r, beta, p);
        term[j] = q - (w[j] - e) * s;
        absr[j] = fabsf(r);
        if (q_out) q_out[j] = (uint8_t)q;
    }
    *err_out = hqo_pairwise_sum(absr, g);
    *znew_out = hqo_pairwise_sum(term, g) / (float)g;
    free(term);
    free(absr);
}

/* binary32 group error -> integer multiple of 2^-32 (truncation; exact in binary64). */
static uint64_t err_fixed(float err)
{
    return (uint64_t)((double)err * 4294967296.0);
}

int hqo_check_args(int64_t rows, int64_t cols, int nbits, int64_t g, int axis)
{
    if (rows <= 0 || cols <= 0 || g <= 0 || g > 4096) return 1;
    if (nbits < 1 || nbits > 8) return 1;
    if (axis != 0 && axis != 1) return 1;
    if ((rows * cols) % g != 0) return 1;
    return 0;
}

/*
 * The full quantizer.  W: N = rows*cols fp16 values (bit patterns), row-major.
 * Outputs: codes[N] (one code per byte, flat order), s_out[G], z_out[G] (binary32, z_out
 * is the kept zero), iters_run, and per-iteration exact error sums err_trace[2*i] (low
 * 64 bits) / err_trace[2*i+1] (high 64 bits), units of 2^-32, for i < iters_run.
 * mae_trace[i] = that sum / 2^32 / N as a double.  Returns 0, or 1 on bad arguments.
 */
int hqo_quantize(const uint16_t *W, int64_t rows, int64_t cols, int nbits, int64_t g, int axis,
                 int iters, double lp_norm, double beta0, double kappa, float eps_tiny,
                 float scale_max, uint8_t *codes, float *s_out, float *z_out, int *iters_run,
                 uint64_t *err_trace, double *mae_trace)
{
    if (hqo_check_args(rows, cols, nbits, g, axis) || iters < 0) return 1;
    int64_t N = rows * cols, G = N / g;
    float qmax = (float)((1 << nbits) - 1);

    /* binary32 copy of W in group order: wg[k*g + j] = element j of group k */
    float *wg = (float *)malloc(sizeof(float) * (size_t)N);
    float *z = (float *)malloc(sizeof(float) * (size_t)G);
    float *znext = (float *)malloc(sizeof(float) * (size_t)G);
    if (!wg || !z || !znext) { free(wg); free(z); free(znext); return 2; }
    for (int64_t k = 0; k < G; k++)
        for (int64_t j = 0; j < g; j++)
            wg[k * g + j] = hqo_half_to_float(W[elem_index(k, j, g, G, axis)]);

    for (int64_t k = 0; k < G; k++)
        hqo_minmax_init(wg + k * g, g, nbits, eps_tiny, scale_max, &s_out[k], &z[k]);
    memcpy(z_out, z, sizeof(float) * (size_t)G);   /* kept zero before any iteration */

    int have_best = 0, run = 0;
    unsigned __int128 best = 0;
    double beta = beta0;
    for (int i = 0; i < iters; i++) {
        unsigned __int128 total = 0;
#ifdef HQO_PARALLEL
        /* Timing build only (the all-core CPU baseline of the benchmark): the same group
           passes, spread over threads; each thread adds its groups' exact integer errors and
           the partial sums are added afterwards, which gives the same total in any order. */
#pragma omp parallel
        {
            unsigned __int128 part = 0;
#pragma omp for schedule(static)
            for (int64_t k = 0; k < G; k++) {
                float err;
                hqo_group_pass(wg + k * g, g, nbits, s_out[k], z[k], beta, lp_norm, NULL, &err,
                               &znext[k]);
                part += err_fixed(err);
            }
#pragma omp critical
            total += part;
        }
#else
        for (int64_t k = 0; k < G; k++) {
            float err;
            hqo_group_pass(wg + k * g, g, nbits, s_out[k], z[k], beta, lp_norm, NULL, &err,
                           &znext[k]);
            total += err_fixed(err);
        }
#endif
        run = i + 1;
        if (err_trace) {
            err_trace[2 * i] = (uint64_t)total;
            err_trace[2 * i + 1] = (uint64_t)(total >> 64);
        }
        if (mae_trace)
            mae_trace[i] = (double)total / 4294967296.0 / (double)N;
        if (!have_best || total < best) {
            have_best = 1;
            best = total;
            memcpy(z_out, z, sizeof(float) * (size_t)G);   /* z_i measured best so far */
            memcpy(z, znext, sizeof(float) * (size_t)G);   /* move on to z_{i+1} */
        } else {
            break;                                         /* revert to the kept zero */
        }
        beta = beta * kappa;
    }
    if (iters_run) *iters_run = run;

    /* final quantize with the original W and the kept parameters */
    for (int64_t k = 0; k < G; k++)
        for (int64_t j = 0; j < g; j++)
            codes[elem_index(k, j, g, G, axis)] =
                (uint8_t)quant_code(wg[k * g + j], s_out[k], z_out[k], qmax);

    free(wg); free(z); free(znext);
    return 0;
}

/* fp16 metadata [HQQ 算法解读, "量化公式"]: Delta = 1/s and z, each rounded to binary16. */
void hqo_metadata(const float *s, const float *z, int64_t G, uint16_t *scale_h, uint16_t *zero_h)
{
    for (int64_t k = 0; k < G; k++) {
        scale_h[k] = hqo_float_to_half(1.0f / s[k]);
        zero_h[k] = hqo_float_to_half(z[k]);
    }
}

/* Packed size in bytes [HQQ 算法解读, "为什么一定要分组"]: 4 bit two codes per byte, 2 bit four,
 * 3 bit ten per 32-bit word; 5 and 6 bit are stored one code per byte, and so are 7 and 8 bit;
 * 1 bit (which the pages name without a layout) eight codes per byte. */
int64_t hqo_packed_bytes(int64_t n, int nbits)
{
    switch (nbits) {
    case 4: return (n + 1) / 2;
    case 2: return (n + 3) / 4;
    case 1: return (n + 7) / 8;
    case 3: return 4 * ((n + 9) / 10);
    default: return n;                     /* 5..8 bits: one code per byte */
    }
}

/* Bit-packing, codes in flat order, lowest index in the lowest bits. */
void hqo_pack(const uint8_t *codes, int64_t n, int nbits, uint8_t *packed)
{
    int64_t nb = hqo_packed_bytes(n, nbits);
    memset(packed, 0, (size_t)nb);
    if (nbits == 4 || nbits == 2 || nbits == 1) {
        int per = 8 / nbits;
        for (int64_t i = 0; i < n; i++)
            packed[i / per] |= (uint8_t)(codes[i] << (nbits * (i % per)));
    } else if (nbits == 3) {
        for (int64_t i = 0; i < n; i++) {
            int64_t word = i / 10;
            uint32_t v = (uint32_t)codes[i] << (3 * (i % 10));
            for (int b = 0; b < 4; b++)    /* little-endian 32-bit word */
                packed[4 * word + b] |= (uint8_t)(v >> (8 * b));
        }
    } else {
        memcpy(packed, codes, (size_t)n);
    }
}

void hqo_unpack(const uint8_t *packed, int64_t n, int nbits, uint8_t *codes)
{
    if (nbits == 4 || nbits == 2 || nbits == 1) {
        int per = 8 / nbits;
        for (int64_t i = 0; i < n; i++)
            codes[i] = (uint8_t)((packed[i / per] >> (nbits * (i % per))) & ((1 << nbits) - 1));
    } else if (nbits == 3) {
        for (int64_t i = 0; i < n; i++) {
            int64_t word = i / 10;
            uint32_t v = (uint32_t)packed[4 * word] | ((uint32_t)packed[4 * word + 1] << 8) |
                         ((uint32_t)packed[4 * word + 2] << 16) |
                         ((uint32_t)packed[4 * word + 3] << 24);
            codes[i] = (uint8_t)((v >> (3 * (i % 10))) & 7);
        }
    } else {
        memcpy(codes, packed, (size_t)n);
    }
}

/*
 * Dequantize [HQQ 算法解读, "量化公式" and "从压缩文件到一次前向"]:
 * W_hat = (q - z)*Delta with z and Delta read back from fp16, one binary32 subtraction and
 * one binary32 product, rounded once to fp16.  Output in the original row-major layout.
 */
int hqo_dequant(const uint8_t *packed, const uint16_t *scale_h, const uint16_t *zero_h,
                int64_t rows, int64_t cols, int nbits, int64_t g, int axis, uint16_t *W_out)
{
    if (hqo_check_args(rows, cols, nbits, g, axis)) return 1;
    int64_t N = rows * cols, G = N / g;
    uint8_t *codes = (uint8_t *)malloc((size_t)N);
    if (!codes) return 2;
    hqo_unpack(packed, N, nbits, codes);
    for (int64_t n = 0; n < N; n++) {
        int64_t k = axis == 1 ? n / g : n % G;
        float zf = hqo_half_to_float(zero_h[k]);
        float df = hqo_half_to_float(scale_h[k]);
        float v = ((float)codes[n] - zf) * df;
        W_out[n] = hqo_float_to_half(v);
    }
    free(codes);
    return 0;
}

/*
 * The quantized layer's forward product for one input vector [HQQ 算法解读,
 * "从压缩文件到一次前向"]: unpack, (q - z)*Delta, then x @ W_hat.T, i.e.
 *     y[r] = sum_c W_hat[r, c] * x[c]
 * with W_hat exactly the fp16 values hqo_dequant produces and x fp16 [cols].  Every product of
 * two fp16 values is exact in binary64, and the sum runs in binary64 in column order, so y
 * carries only the rounding of that sum (the reading: the pages fix no summation order or
 * precision for this step).  absum[r] = sum_c |W_hat[r, c] * x[c]| bounds any other
 * summation order's error.  Both outputs [rows] binary64.
 */
int hqo_gemv(const uint8_t *packed, const uint16_t *scale_h, const uint16_t *zero_h,
             int64_t rows, int64_t cols, int nbits, int64_t g, int axis, const uint16_t *x_h,
             double *y, double *absum)
{
    if (hqo_check_args(rows, cols, nbits, g, axis)) return 1;
    int64_t N = rows * cols;
    uint16_t *w = (uint16_t *)malloc((size_t)N * sizeof(uint16_t));
    if (!w) return 2;
    int rc = hqo_dequant(packed, scale_h, zero_h, rows, cols, nbits, g, axis, w);
    if (rc) { free(w); return rc; }
    for (int64_t r = 0; r < rows; r++) {
        double acc = 0.0, mag = 0.0;
        for (int64_t c = 0; c < cols; c++) {
            double p = (double)hqo_half_to_float(w[r * cols + c]) * (double)hqo_half_to_float(x_h[c]);
            acc += p;
            mag += fabs(p);
        }
        y[r] = acc;
        absum[r] = mag;
    }
    free(w);
    return 0;
}
