/*
 * hqq_b200.h -- C ABI of the B200 (sm_100a) HQQ group-wise weight quantizer.
 *
 * The method is the one described on the page "HQQ 算法解读：不用校准数据，怎样把大模型权重压到
 * 4 bit" (ludovicoyin.github.io/blog/posts/hqq-half-quadratic-quantization), cited as
 * [HQQ 算法解读, <section>].  Its Python interface there is BaseQuantizeConfig(nbits,
 * group_size, axis) plus HQQLinear(...) and .dequantize() (section "一个最小可复现实验"); this
 * header restates quantize and dequantize as two calls on caller-owned device buffers.
 *
 * Conventions for every call below:
 *   - all data pointers are DEVICE pointers owned by the caller; the library allocates
 *     nothing and keeps no pointer after the call returns;
 *   - calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream);
 *     the return value reports argument checks and launch errors only;
 *   - W is fp16, row-major [rows, cols], never modified; N = rows * cols, G = N / group_size;
 *   - group view [HQQ 算法解读, "`axis` 不是一个无关紧要的开关"]: axis = 1 takes groups of
 *     group_size consecutive elements (W.reshape([-1, g])); axis = 0 takes the columns of
 *     the [g, G] row-major view (W.reshape([g, -1])), i.e. group k = elements j*G + k;
 *   - packed codes are in flat row-major element order for both axes, lowest index in the
 *     lowest bits [HQQ 算法解读, "为什么一定要分组"]: 4 bit = two codes per byte, 2 bit = four
 *     codes per byte, 3 bit = ten codes per little-endian 32-bit word (bits 30-31 zero),
 *     5 and 6 bit = one code per byte (unpacked); this library stores 7- and 8-bit codes one
 *     per byte as well and packs 1-bit codes eight per byte (the pages name 1 bit without a
 *     layout); the tail of the last byte or word is zero;
 *   - metadata [HQQ 算法解读, "量化公式：把尺子写出来"]: scale[G] = fp16(1/s) (the page's
 *     Delta) and zero[G] = fp16(z), in group order.
 *   - W should hold finite values: a group with a NaN or an infinity gets unspecified codes and
 *     metadata (the call still completes and touches no memory outside its buffers).
 */
#ifndef HQQ_B200_H
#define HQQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define HQQ_OK 0
#define HQQ_ERR_ARG 1          /* a size, bit width, axis, option or required pointer is invalid */
#define HQQ_ERR_ALIGN 2        /* a pointer is not aligned as documented */
#define HQQ_ERR_WORKSPACE 3    /* workspace null or smaller than hqq_quantize_workspace_bytes() */
#define HQQ_ERR_CUDA 4         /* a CUDA runtime call or kernel launch failed */
#define HQQ_ERR_UNSUPPORTED 5  /* valid for the method, outside this library's limits (below) */

/* limits of this library */
#define HQQ_MAX_GROUP_SIZE 256 /* group_size 1 .. 256 */
#define HQQ_MAX_ITERS 64       /* iters 0 .. 64 (the page's default is 20) */

/*
 * Options of the proximal loop [HQQ 算法解读, "第一拍" and "第二拍"].
 *   iters      at most this many rounds (page: 20)
 *   lp_norm    p of the lp shrink, 0 < p < 2 (page: 0.7)
 *   beta       beta of the first round, > 0 (page: 10)
 *   kappa      beta is multiplied by kappa after each round, > 0 (page: 1.01)
 *   eps_tiny   a group whose max - min is below this gets s = 1 (the page only says "too
 *              small"; 1e-4 is this library's reading), >= 0
 *   scale_max  s is clamped to at most this value (page: 2e4), > 0
 */
typedef struct hqq_opt {
    int32_t iters;
    double lp_norm;
    double beta;
    double kappa;
    float eps_tiny;
    float scale_max;
} hqq_opt_t;

/* Fills *opt with the page's defaults: 20, 0.7, 10, 1.01, 1e-4, 2e4. */
void hqq_default_opt(hqq_opt_t *opt);

/* Exact size in bytes of the packed codes of n weights [HQQ 算法解读, "为什么一定要分组"]:
 * n/8 (1 bit), n/4 (2 bit), 4*ceil(n/10) (3 bit), n/2 (4 bit), rounded up, or n (5 to 8 bit).
 * Returns -1 for nbits outside 1..8 or n < 0. */
int64_t hqq_packed_bytes(int64_t n, int nbits);

/* Device workspace, in bytes, that hqq_quantize needs for these arguments (0 if invalid). */
size_t hqq_quantize_workspace_bytes(int64_t rows, int64_t cols, int nbits, int64_t group_size,
                                    int axis, int iters);

/*
 * HQQ quantize + pack [HQQ 算法解读, "第一拍", "第二拍", "为什么一定要分组"]:
 * per group s0 = (2^b-1)/(max-min) (s = 1 when max-min < eps_tiny, then s <= scale_max),
 * z0 = -min*s0; then up to `iters` rounds of q = clip(round(W*s+z), 0, 2^b-1),
 * W_hat = (q-z)/s, e = shrink_lp(W - W_hat, beta_i), z <- mean(q - (W-e)*s), with
 * beta_i = beta*kappa^i; the loop stops at the first round whose tensor-wide MAE
 * mean|W - W_hat| is not strictly below the best so far and keeps the zero of the best
 * round; a final quantize with the original W gives the codes.
 *
 * Arguments
 *   W            [rows*cols] fp16, 16-byte aligned
 *   nbits        1 to 8;  group_size 1..256 dividing rows*cols;  axis 0 or 1.  2- and 4-bit
 *                axis-1 layouts with a power-of-two group of 16..128 run the one-group-per-lane
 *                engine; every other layout the tile engine, which for 5 to 8 bits computes
 *                W_hat by one IEEE division per element instead of a table of the 2^b values
 *   opt          options (host pointer); NULL = hqq_default_opt()
 *   packed       [hqq_packed_bytes(N, nbits)] bytes, 16-byte aligned (output)
 *   scale, zero  [G] fp16 each, 2-byte aligned (outputs): fp16(1/s) and fp16(z)
 *   iters_run    device int32, nullable (output): rounds whose MAE was computed
 *   s_f32, z_f32 [G] float each, nullable (outputs): s and the kept z in binary32
 *   err_trace    [2*iters] uint64, nullable (output): entry i < iters_run is the exact sum
 *                over groups of floor(2^32 * sum_group |W - W_hat|) at round i, as
 *                (low 64 bits, high 64 bits); MAE_i = that / 2^32 / N.  Entries at or past
 *                iters_run are unspecified.
 *   group_rounds [G] uint8, nullable (output): rounds each group ran.  A group stops once
 *                its zero stops moving and every later round provably repeats the last one,
 *                or after iters rounds; 0 when iters = 0.  Diagnostic: the work the loop
 *                did.
 *   workspace    >= hqq_quantize_workspace_bytes(...) bytes, 16-byte aligned; contents on
 *                entry do not matter; must not be used by anything else until the work
 *                queued on `stream` by this call has finished
 *   stream       cudaStream_t
 * Returns HQQ_OK or an HQQ_ERR_* code; on an error nothing is launched.
 */
int hqq_quantize(const void *W, int64_t rows, int64_t cols, int nbits, int64_t group_size,
                 int axis, const hqq_opt_t *opt, void *packed, void *scale, void *zero,
                 int32_t *iters_run, float *s_f32, float *z_f32, uint64_t *err_trace,
                 uint8_t *group_rounds, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Unpack + dequantize [HQQ 算法解读, "量化公式" and "从压缩文件到一次前向"]:
 * W_out = fp16((q - f32(zero)) * f32(scale)) in binary32, rounded once to fp16, written in
 * the original [rows, cols] row-major layout.
 *   packed   as written by hqq_quantize, 16-byte aligned
 *   scale, zero [G] fp16, 2-byte aligned
 *   W_out    [rows*cols] fp16, 16-byte aligned (output)
 * Returns HQQ_OK or an HQQ_ERR_* code; on an error nothing is launched.
 */
int hqq_dequantize(const void *packed, const void *scale, const void *zero, int64_t rows,
                   int64_t cols, int nbits, int64_t group_size, int axis, void *W_out,
                   void *stream);

/*
 * hqq_gemv: the quantized layer's forward product for one input vector, with dequantization
 * fused in [HQQ 算法解读, "从压缩文件到一次前向"]: unpack -> (q - zero) * scale -> x @ W_hat.T,
 * without writing W_hat to memory.
 *     y[r] = sum_c W_hat[r, c] * x[c]
 * W_hat[r, c] is exactly the fp16 value hqq_dequantize writes. Each product of two fp16 values
 * is exact in binary32, and the row sum runs in binary32 in an order of the kernel's choosing,
 * so y[r] is within cols * 2^-23 * sum_c |W_hat[r, c] * x[c]| of the exact sum.
 *   packed, scale, zero  as written by hqq_quantize for the same rows, cols, nbits, group_size
 *                        and axis (packed 16-byte aligned, scale and zero 2-byte aligned)
 *   x       [cols] fp16, 2-byte aligned. 16-byte alignment enables the fast path.
 *   y       [rows] binary32, 4-byte aligned (output)
 *   stream  cudaStream_t, or NULL for the default stream
 * Every layout is accepted.  Fast paths (x 16-byte aligned):
 *   - axis 1, 2- or 4-bit codes, group_size a multiple of 32 dividing cols: one warp per row,
 *     32-code pieces (from 16 MiB of codes on, with scale and zero 16-byte aligned, rows move
 *     in bulk copies through shared memory);
 *   - axis 1, 2- or 4-bit codes, cols and group_size multiples of the codes per 32-bit word (8
 *     at 4 bit, 16 at 2 bit), group_size dividing cols: one warp per row, one word per load;
 *   - axis 0, 4-bit codes, group_size dividing rows, cols a multiple of 32, scale and zero
 *     16-byte aligned: one warp per row with per-code metadata;
 *   - axis 1, 3-bit codes, group_size >= 10, cols even and at most 24576, x 4-byte aligned
 *     suffices: x staged in shared memory.
 * Other layouts read their codes one at a time.
 * Returns HQQ_OK, HQQ_ERR_ARG (shape or null pointer), HQQ_ERR_ALIGN, or HQQ_ERR_CUDA.
 */
int hqq_gemv(const void *packed, const void *scale, const void *zero, int64_t rows, int64_t cols,
             int nbits, int64_t group_size, int axis, const void *x, float *y, void *stream);

/*
 * hqq_gemm: the quantized layer's forward product for a batch of input vectors, with
 * dequantization fused in [HQQ 算法解读, "从压缩文件到一次前向"; the `axis` table's row for low-batch
 * inference throughput]:
 *     Y[b, r] = sum_c W_hat[r, c] * X[b, c]        for b < batch
 * W_hat[r, c] is exactly the fp16 value hqq_dequantize writes.  Each product of two fp16 values is
 * exact in binary32 and the sums run in binary32 in an order of the library's choosing, so
 * Y[b, r] is within cols * 2^-23 * sum_c |W_hat[r, c] * X[b, c]| of the exact sum.
 *   packed, scale, zero  as written by hqq_quantize (packed 16-byte aligned, scale and zero
 *                        2-byte aligned)
 *   X       [batch, cols] fp16 row-major, 2-byte aligned
 *   batch   >= 0 (0: nothing is launched)
 *   Y       [batch, rows] binary32 row-major, 4-byte aligned (output)
 *   stream  cudaStream_t, or NULL for the default stream
 * Axis-1 layouts with 2- or 4-bit codes, group_size a multiple of 8 that divides cols, cols a
 * multiple of 64 and a 16-byte aligned X run on the tensor cores (tcgen05.mma, fp16 operands, binary32 accumulators in
 * tensor memory; up to 256 batch entries per launch) when batch >= 2.  A batch of one, and
 * every other layout, runs the one-vector product (hqq_gemv) once per batch entry.
 * Returns HQQ_OK, HQQ_ERR_ARG (shape, batch or null pointer), HQQ_ERR_ALIGN, or HQQ_ERR_CUDA.
 */
int hqq_gemm(const void *packed, const void *scale, const void *zero, int64_t rows, int64_t cols,
             int nbits, int64_t group_size, int axis, const void *X, int64_t batch, float *Y,
             void *stream);

/*
 * hqq_quantize without a workspace argument.  The pages have no counterpart to this call: it
 * exists for callers that cannot allocate device memory, such as plugins running inside a
 * framework whose pool owns all of the GPU's memory, or loops that must never call cudaMalloc
 * (it may synchronize the device).  Its scratch is a fixed 4 MiB buffer compiled into this
 * library (HQQ_NOALLOC_SCRATCH_BYTES): every GPU that loads the library keeps it until the
 * process exits.  Arguments, outputs and results are those of hqq_quantize; additionally it
 * returns HQQ_ERR_WORKSPACE, launching nothing, when hqq_quantize_workspace_bytes() for these
 * arguments exceeds that buffer.  It allocates nothing.  The buffer used is the one of the
 * calling thread's current device, in that device's primary context (the CUDA runtime's
 * default; a context made with the driver API is not supported): W, the outputs and the stream
 * must belong to that device.  The first call on each device looks up the buffer's device
 * address (make it before any stream capture).  All calls share the one buffer: calls whose GPU
 * work overlaps (other streams, other host threads) race on it.
 */
#define HQQ_NOALLOC_SCRATCH_BYTES (4u << 20)
int hqq_quantize_noalloc(const void *W, int64_t rows, int64_t cols, int nbits, int64_t group_size,
                         int axis, const hqq_opt_t *opt, void *packed, void *scale, void *zero,
                         int32_t *iters_run, float *s_f32, float *z_f32, uint64_t *err_trace,
                         uint8_t *group_rounds, void *stream);

/*
 * The generalized lp shrink operator of the proximal step [HQQ 算法解读, "shrink 不是删除极值"],
 * element by element, exactly as hqq_quantize evaluates it inside its rounds:
 *     out[i] = sign(r[i]) * max(|r[i]| - |r[i]|^(p - 1) / beta, 0)
 * computed in binary64 from the binary32 r[i] and rounded once to binary32 (0 for r[i] = 0).
 * r and out: device pointers to n binary32 values (4-byte aligned; out may equal r).  It lets a
 * caller check the operator against another implementation (the power function is CUDA's).
 * Returns HQQ_OK (n = 0: nothing launched), HQQ_ERR_ARG (n < 0, beta <= 0, p <= 0, null
 * pointer), HQQ_ERR_ALIGN or HQQ_ERR_CUDA.
 */
int hqq_shrink_lp(const float *r, int64_t n, double beta, double p, float *out, void *stream);

/* Text for a return code (static storage). */
const char *hqq_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* HQQ_B200_H */
