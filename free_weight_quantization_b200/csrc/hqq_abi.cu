// hqq_abi.cu -- the C ABI of the B200 HQQ library (include/hqq_b200.h): argument checks, the
// launch plan (which engine, tile sizes, workspace layout) and the entry points.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "hqq_common.cuh"

namespace {

// groups up to which a stream-engine tensor keeps its zeros per round (G x iters binary32)
constexpr int64_t kZringMaxGroups = 16384;

struct Plan {
    int64_t N, G;
    int g, P, L, stride, tile;  // stride: floats per tile row
    int64_t ntiles;
    bool aligned;  // packed words can be written per tile
    bool stream;   // axis 1, 2- or 4-bit, power-of-two groups of 16 .. 128 (the stream engine)
    size_t ws_acc, ws_fk, ws_tile, ws_stale, ws_codes, ws_zring, ws_total;
};

int64_t gcd64(int64_t a, int64_t b) {
    while (b) { int64_t t = a % b; a = b; b = t; }
    return a;
}

// codes per 32-bit word of the packed layout (the Pack<NB> of the kernels)
int cpw_of(int nbits) { return nbits == 3 ? 10 : nbits == 1 ? 32 : nbits == 2 ? 16 : nbits == 4 ? 8 : 4; }

int make_plan(int64_t rows, int64_t cols, int nbits, int64_t group_size, int axis, int iters,
              Plan *pl) {
    if (rows <= 0 || cols <= 0 || group_size <= 0) return HQQ_ERR_ARG;
    if (nbits < 1 || nbits > 8) return HQQ_ERR_ARG;
    if (axis != 0 && axis != 1) return HQQ_ERR_ARG;
    if (rows > (int64_t(1) << 40) / cols) return HQQ_ERR_UNSUPPORTED;
    const int64_t N = rows * cols;
    if (N % group_size) return HQQ_ERR_ARG;
    if (group_size > HQQ_MAX_GROUP_SIZE) return HQQ_ERR_UNSUPPORTED;
    if (iters < 0) return HQQ_ERR_ARG;
    if (iters > HQQ_MAX_ITERS) return HQQ_ERR_UNSUPPORTED;
    pl->N = N;
    pl->G = N / group_size;
    pl->g = (int)group_size;
    int P = 16;
    while (P < pl->g) P *= 2;
    pl->P = P;
    pl->L = P / kE;
    pl->stride = P + (P >= 64 ? 8 : 0);  // halves per tile row (the padding staggers banks)
    const int target = 40960;            // halves of W per tile
    const int cap = std::max(1, target / pl->stride);
    // tiles that start on a packed word: axis 1, tiles of 320k elements (a multiple of 4, 8, 10,
    // 16 and 32 codes, and 16-byte aligned); axis 0, a multiple of 80 columns (lcm of 4, 8, 10,
    // 16), or of 160 for 1-bit codes (32 per word)
    const int unit = axis == 1 ? (int)(320 / gcd64(pl->g, 320)) : (nbits == 1 ? 160 : 80);
    pl->tile = unit * std::max(1, cap / unit);
    // two CTAs per SM: keep the whole shared-memory layout within 110 KB
    while (pl->tile > unit &&
           smem_layout(pl->tile, pl->stride, nbits <= 4 ? 1 << nbits : 0, pl->L, iters).total > 110 * 1024)
        pl->tile -= unit;
    // spread the groups evenly over whole waves of resident CTAs (two per SM)
    {
        const int64_t slots = 2 * 148;  // B200: 148 SMs
        const int64_t want = (pl->G + pl->tile - 1) / pl->tile;
        const int64_t waves = (want + slots - 1) / slots;
        const int64_t per = (pl->G + waves * slots - 1) / (waves * slots);
        const int64_t even = (per + unit - 1) / unit * unit;
        if (even < pl->tile) pl->tile = (int)even;
    }
    pl->ntiles = (pl->G + pl->tile - 1) / pl->tile;
    pl->aligned = axis == 1 || (pl->G % cpw_of(nbits) == 0);
    // the stream engine: axis 1, 2- and 4-bit codes, groups of 16 .. 128 that are whole 32-bit
    // words of the output (its codes are stored straight from registers)
    pl->stream = axis == 1 && (nbits == 2 || nbits == 4) && P <= 128 && pl->g == P && (pl->g * nbits) % 32 == 0;
    const int K = iters > 0 ? iters : 1;
    pl->ws_acc = (size_t)4 * K * sizeof(u64) + 64;  // per-round sums + control words (zeroed)
    pl->ws_fk = (size_t)((pl->G + 15) / 16 * 16);
    pl->ws_tile = (size_t)((pl->ntiles + 15) / 16 * 16);
    pl->ws_stale = (size_t)(4 * pl->ntiles + 15) / 16 * 16;
    pl->ws_codes = pl->aligned ? 0 : (size_t)((N + 15) / 16 * 16);
    // a small stream-engine tensor keeps every group's zero after each update, so that the
    // fixup of a stale group reads the kept zero instead of replaying the rounds up to it
    pl->ws_zring = pl->stream && iters > 0 && pl->G <= kZringMaxGroups ? (size_t)pl->G * iters * 4 : 0;
    pl->ws_total = pl->ws_acc + pl->ws_fk + pl->ws_tile + pl->ws_stale + pl->ws_codes + pl->ws_zring;
    return HQQ_OK;
}

bool aligned_to(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

}  // namespace


// ==========================================================================================
// C ABI
// ==========================================================================================
extern "C" void hqq_default_opt(hqq_opt_t *opt) {
    if (!opt) return;
    opt->iters = 20;
    opt->lp_norm = 0.7;
    opt->beta = 10.0;
    opt->kappa = 1.01;
    opt->eps_tiny = 1e-4f;
    opt->scale_max = 2e4f;
}

extern "C" int64_t hqq_packed_bytes(int64_t n, int nbits) {
    if (n < 0) return -1;
    switch (nbits) {
    case 1: return (n + 7) / 8;
    case 2: return (n + 3) / 4;
    case 3: return 4 * ((n + 9) / 10);
    case 4: return (n + 1) / 2;
    case 5: case 6: case 7: case 8: return n;
    default: return -1;
    }
}

extern "C" size_t hqq_quantize_workspace_bytes(int64_t rows, int64_t cols, int nbits,
                                               int64_t group_size, int axis, int iters) {
    Plan pl;
    if (make_plan(rows, cols, nbits, group_size, axis, iters, &pl) != HQQ_OK) return 0;
    return pl.ws_total;
}

extern "C" int hqq_quantize(const void *W, int64_t rows, int64_t cols, int nbits,
                            int64_t group_size, int axis, const hqq_opt_t *opt, void *packed,
                            void *scale, void *zero, int32_t *iters_run, float *s_f32,
                            float *z_f32, uint64_t *err_trace, uint8_t *group_rounds,
                            void *workspace, size_t workspace_bytes, void *stream) {
    hqq_opt_t o;
    if (opt) o = *opt; else hqq_default_opt(&o);
    Plan pl;
    int rc = make_plan(rows, cols, nbits, group_size, axis, o.iters, &pl);
    if (rc != HQQ_OK) return rc;
    if (!W || !packed || !scale || !zero) return HQQ_ERR_ARG;
    if (!(o.lp_norm > 0.0 && o.lp_norm < 2.0) || !(o.beta > 0.0) || !(o.kappa > 0.0) ||
        !(o.eps_tiny >= 0.0f) || !(o.scale_max > 0.0f) || !std::isfinite(o.beta) ||
        !std::isfinite(o.kappa) || !std::isfinite(o.scale_max))
        return HQQ_ERR_ARG;
    if (!aligned_to(W, 16) || !aligned_to(packed, 16) || !aligned_to(scale, 2) ||
        !aligned_to(zero, 2) || !aligned_to(iters_run, 4) || !aligned_to(s_f32, 4) ||
        !aligned_to(z_f32, 4) || !aligned_to(err_trace, 8))
        return HQQ_ERR_ALIGN;
    if (!workspace || workspace_bytes < pl.ws_total) return HQQ_ERR_WORKSPACE;
    if (!aligned_to(workspace, 16)) return HQQ_ERR_ALIGN;

    QParams P;
    memset(&P, 0, sizeof(P));
    P.W = (const __half *)W;
    P.N = pl.N;
    P.G = pl.G;
    P.g = pl.g;
    P.axis = axis;
    P.K = o.iters;
    P.stride = pl.stride;
    P.tile = pl.tile;
    P.packed = (uint8_t *)packed;
    P.packed_bytes = hqq_packed_bytes(pl.N, nbits);
    P.scale = (__half *)scale;
    P.zero = (__half *)zero;
    P.s_out = s_f32;
    P.z_out = z_f32;
    P.acc = (u64 *)workspace;
    uint8_t *wsp = (uint8_t *)workspace;
    P.fk = wsp + pl.ws_acc;
    uint8_t *wtile = wsp + pl.ws_acc + pl.ws_fk;
    P.tile_maxf = wtile;
    P.stale = (int *)(wtile + pl.ws_tile);
    P.codes_u8 = pl.aligned ? nullptr : wtile + pl.ws_tile + pl.ws_stale;
    P.zring = pl.ws_zring ? (float *)(wtile + pl.ws_tile + pl.ws_stale + pl.ws_codes) : nullptr;
    P.iters_run = iters_run;
    P.err_trace = (u64 *)err_trace;
    P.group_rounds = group_rounds;
    P.eps_tiny = o.eps_tiny;
    P.scale_max = o.scale_max;
    P.p = o.lp_norm;
    // beta_i = beta * kappa^i by repeated binary64 multiplication; the safe threshold keeps a
    // 0.1% margin below the exact zero set |r| <= beta^(-1/(2-p)) of the shrink
    double beta = o.beta;
    for (int i = 0; i < o.iters; ++i) {
        P.beta[i] = beta;
        P.thr[i] = (float)(0.999 * std::pow(beta, -1.0 / (2.0 - o.lp_norm)));
        beta = beta * o.kappa;
    }
    cudaStream_t st = (cudaStream_t)stream;
    P.acc_words = (int64_t)(pl.ws_acc / sizeof(u64));
    cudaError_t e;
    if (pl.stream) {
        e = hqq_impl::launch_stream_engine(P, nbits, pl.g, st);
    } else {
        const bool direct = axis == 1 && pl.g % 16 == 0 && (nbits == 2 || nbits == 4);
        e = hqq_impl::launch_tile_engine(P, nbits, pl.L, pl.g == pl.P, direct, pl.ntiles, st);
    }
    return e == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int hqq_dequantize(const void *packed, const void *scale, const void *zero,
                              int64_t rows, int64_t cols, int nbits, int64_t group_size, int axis,
                              void *W_out, void *stream) {
    Plan pl;
    int rc = make_plan(rows, cols, nbits, group_size, axis, 0, &pl);
    if (rc != HQQ_OK) return rc;
    if (!packed || !scale || !zero || !W_out) return HQQ_ERR_ARG;
    if (!aligned_to(packed, 16) || !aligned_to(W_out, 16) || !aligned_to(scale, 2) ||
        !aligned_to(zero, 2))
        return HQQ_ERR_ALIGN;
    const int64_t pb = hqq_packed_bytes(pl.N, nbits);
    cudaStream_t st = (cudaStream_t)stream;
    const uint8_t *pk = (const uint8_t *)packed;
    const __half *sc = (const __half *)scale, *ze = (const __half *)zero;
    __half *out = (__half *)W_out;
    const cudaError_t e = hqq_impl::launch_dequantize(nbits, pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st);
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int hqq_gemv(const void *packed, const void *scale, const void *zero, int64_t rows,
                        int64_t cols, int nbits, int64_t group_size, int axis, const void *x,
                        float *y, void *stream) {
    Plan pl;
    int rc = make_plan(rows, cols, nbits, group_size, axis, 0, &pl);
    if (rc != HQQ_OK) return rc;
    if (!packed || !scale || !zero || !x || !y) return HQQ_ERR_ARG;
    if (!aligned_to(packed, 16) || !aligned_to(scale, 2) || !aligned_to(zero, 2) ||
        !aligned_to(x, 2) || !aligned_to(y, 4))
        return HQQ_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const uint8_t *pk = (const uint8_t *)packed;
    const __half *sc = (const __half *)scale, *ze = (const __half *)zero, *xh = (const __half *)x;
    const cudaError_t e = hqq_impl::launch_gemv(nbits, pk, sc, ze, rows, cols, pl.g, pl.G, axis, xh, y, st);
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" int hqq_gemm(const void *packed, const void *scale, const void *zero, int64_t rows,
                        int64_t cols, int nbits, int64_t group_size, int axis, const void *X,
                        int64_t batch, float *Y, void *stream) {
    Plan pl;
    int rc = make_plan(rows, cols, nbits, group_size, axis, 0, &pl);
    if (rc != HQQ_OK) return rc;
    if (batch < 0) return HQQ_ERR_ARG;
    if (batch == 0) return HQQ_OK;
    if (!packed || !scale || !zero || !X || !Y) return HQQ_ERR_ARG;
    if (!aligned_to(packed, 16) || !aligned_to(scale, 2) || !aligned_to(zero, 2) ||
        !aligned_to(X, 2) || !aligned_to(Y, 4))
        return HQQ_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const uint8_t *pk = (const uint8_t *)packed;
    const __half *sc = (const __half *)scale, *ze = (const __half *)zero, *xh = (const __half *)X;
    cudaError_t e;
    // one input vector: the SIMT product is faster than four N = 16 MMAs per tile
    if (batch >= 2 && hqq_impl::gemm_tc_layout(nbits, rows, cols, pl.g, axis, X)) {
        e = hqq_impl::launch_gemm_tc(nbits, pk, sc, ze, rows, cols, pl.g, xh, batch, Y, st);
    } else {  // a single vector, or any other layout: the one-vector product per batch entry
        e = cudaSuccess;
        for (int64_t b = 0; b < batch && e == cudaSuccess; ++b)
            e = hqq_impl::launch_gemv(nbits, pk, sc, ze, rows, cols, pl.g, pl.G, axis, xh + b * cols,
                                      Y + b * rows, st);
    }
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

namespace {
__global__ void __launch_bounds__(256) hqq_shrink_kernel(const float *__restrict__ r, int64_t n, double beta,
                                                         double p, float *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = shrink_lp(r[i], beta, p);
}
}  // namespace

extern "C" int hqq_shrink_lp(const float *r, int64_t n, double beta, double p, float *out, void *stream) {
    if (n < 0 || !(beta > 0.0) || !(p > 0.0)) return HQQ_ERR_ARG;
    if (n == 0) return HQQ_OK;
    if (!r || !out) return HQQ_ERR_ARG;
    if (!aligned_to(r, 4) || !aligned_to(out, 4)) return HQQ_ERR_ALIGN;
    const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 32);
    hqq_shrink_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(r, n, beta, p, out);
    return cudaGetLastError() == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
}

extern "C" const char *hqq_strerror(int code) {
    switch (code) {
    case HQQ_OK: return "ok";
    case HQQ_ERR_ARG: return "invalid argument";
    case HQQ_ERR_ALIGN: return "misaligned pointer";
    case HQQ_ERR_WORKSPACE: return "workspace missing or too small";
    case HQQ_ERR_CUDA: return "CUDA launch or runtime error";
    case HQQ_ERR_UNSUPPORTED: return "outside this library's limits (group_size <= 256, iters <= 64)";
    default: return "unknown error";
    }
}

// ==========================================================================================
// No-allocation variant of hqq_quantize
//
// Some callers cannot hand this library a workspace: code running under a host framework
// that owns all device memory through its own pool, plugins that may not call cudaMalloc
// (it can synchronize the device and fail once a pool has reserved the memory), or tight
// loops that must never allocate.  For them the scratch of hqq_quantize lives in a fixed
// buffer compiled into this library: every GPU that loads the library holds it until the
// process exits.  Host code cannot pass the array's name to a kernel (in host code it is a
// stand-in, not a device address), so the device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and that address is what the kernels
// receive.  The first call on each device does this look-up, so make that first call before
// any stream capture.  All calls share the one buffer and it keeps the previous call's data:
// hqq_quantize clears the part that must start at zero on every call, and two calls whose
// work overlaps on the GPU (different streams, or different host threads) race on it.
// ==========================================================================================
namespace {

constexpr size_t kNoAllocScratchBytes = HQQ_NOALLOC_SCRATCH_BYTES;  // 4 MiB, from the header
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device

int noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HQQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HQQ_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return HQQ_OK;
}

}  // namespace

extern "C" int hqq_quantize_noalloc(const void *W, int64_t rows, int64_t cols, int nbits,
                                    int64_t group_size, int axis, const hqq_opt_t *opt,
                                    void *packed, void *scale, void *zero, int32_t *iters_run,
                                    float *s_f32, float *z_f32, uint64_t *err_trace,
                                    uint8_t *group_rounds, void *stream) {
    hqq_opt_t o;
    if (opt) o = *opt; else hqq_default_opt(&o);
    Plan pl;
    const int rc = make_plan(rows, cols, nbits, group_size, axis, o.iters, &pl);
    if (rc != HQQ_OK) return rc;
    if (pl.ws_total > kNoAllocScratchBytes) return HQQ_ERR_WORKSPACE;  // beyond the fixed buffer
    void *scratch = nullptr;
    const int sr = noalloc_scratch(&scratch);
    if (sr != HQQ_OK) return sr;
    return hqq_quantize(W, rows, cols, nbits, group_size, axis, &o, packed, scale, zero, iters_run,
                        s_f32, z_f32, err_trace, group_rounds, scratch, kNoAllocScratchBytes, stream);
}
