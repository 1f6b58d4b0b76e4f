// hqq_common.cuh -- declarations and device helpers shared by the translation units of the
// B200 (sm_100a) HQQ library: parameters of a quantize call, the exact fixed-point error sums
// and the stop rule, the correctly rounded table of reconstructions, the residual bound of the
// shrink's dead zone, and programmatic-dependent-launch helpers.
//
// Method: the page "HQQ 算法解读：不用校准数据，怎样把大模型权重压到 4 bit"
// (ludovicoyin.github.io/blog/posts/hqq-half-quadratic-quantization), cited as
// [HQQ 算法解读, <section>].  The arithmetic reproduces, operation for operation, the binary32
// definition stated in include/hqq_b200.h: every product and sum rounded separately
// (__fmul_rn/__fadd_rn and their packed .f32x2 forms, no contraction), W_hat = (q - z)/s
// correctly rounded, round half to even, pairwise (recursive-halving) group sums, the lp shrink
// in binary64, and an exact fixed-point (2^-32) 128-bit tensor-wide error sum for the stop
// rule.  No tensor cores: nothing on this path is a dense contraction.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "hqq_b200.h"

namespace hqq_impl {

typedef unsigned long long u64;

struct QParams {
    const __half *W;
    int64_t N, G;
    int g;          // group size
    int axis;
    int K;          // iteration cap
    int stride;     // floats per group row of the shared tile
    int tile;       // groups per tile
    int stream_warps;  // warps of each stream-engine CTA that take groups (the rest idle)
    int stream_lanes;  // lanes of such a warp that take groups (32, or 4 for a small tensor)
    int64_t acc_words; // 64-bit words of round sums and control words zeroed before each call
    uint8_t *packed;
    int64_t packed_bytes;
    __half *scale, *zero;
    float *s_out, *z_out;
    u64 *acc;       // [K][2] direct round sums, [K][2] difference array, then control words
    uint8_t *fk;    // [G] last round run by each group
    uint8_t *tile_maxf;  // [ntiles] largest f of each tile
    int *stale;     // [ntiles] tiles holding a group whose last round lies past the kept one
    uint8_t *codes_u8;  // [N] byte-per-code staging when the packed layout is not tile aligned
    float *zring;       // [G][K] zero after each update (small stream-engine tensors), or null
    int32_t *iters_run;
    u64 *err_trace;
    uint8_t *group_rounds;  // [G] nullable: rounds run by each group in the search kernel
    float eps_tiny, scale_max;
    double p;
    double beta[HQQ_MAX_ITERS];
    float thr[HQQ_MAX_ITERS];  // |r| <= thr[i] guarantees shrink(r, beta_i) == 0
};

}  // namespace hqq_impl

namespace {

using hqq_impl::QParams;
using hqq_impl::u64;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kE = 16;  // elements per lane
constexpr unsigned kFull = 0xffffffffu;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer (RNE)



// ------------------------------------------------------------------------------------------
// small device helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ u64 err_fixed(float err) {
    // floor(err * 2^32): the scaling is exact in binary32; truncation toward zero
    return __float2ull_rz(__fmul_rn(err, 4294967296.0f));
}

__device__ __forceinline__ void add_fixed(unsigned *row, u64 v) {
    // 64-bit fixed-point value into four 16-bit-chunk counters (exact; no counter overflows)
    atomicAdd(row, (unsigned)(v & 0xffffu));
    atomicAdd(row + 1, (unsigned)((v >> 16) & 0xffffu));
    atomicAdd(row + 2, (unsigned)((v >> 32) & 0xffffu));
    atomicAdd(row + 3, (unsigned)(v >> 48));
}

// e = sign(r) * max(|r| - |r|^(p-1)/beta, 0) in binary64, rounded once to binary32
// [HQQ 算法解读, "第二拍" and "shrink 不是删除极值"; the formula is the HQQ paper's lp shrink]
__device__ __noinline__ float shrink_lp(float r, double beta, double p) {
    double a = fabs((double)r);
    if (a == 0.0) return 0.0f;
    double m = a - pow(a, p - 1.0) / beta;
    if (!(m > 0.0)) return 0.0f;
    float mf = (float)m;
    return r < 0.0f ? -mf : mf;
}

// pairwise (recursive halving) sum of 16 values
__device__ __forceinline__ float tree16(const float *x) {
    float a0 = __fadd_rn(x[0], x[1]), a1 = __fadd_rn(x[2], x[3]);
    float a2 = __fadd_rn(x[4], x[5]), a3 = __fadd_rn(x[6], x[7]);
    float a4 = __fadd_rn(x[8], x[9]), a5 = __fadd_rn(x[10], x[11]);
    float a6 = __fadd_rn(x[12], x[13]), a7 = __fadd_rn(x[14], x[15]);
    float b0 = __fadd_rn(a0, a1), b1 = __fadd_rn(a2, a3);
    float b2 = __fadd_rn(a4, a5), b3 = __fadd_rn(a6, a7);
    return __fadd_rn(__fadd_rn(b0, b1), __fadd_rn(b2, b3));
}

// upper levels of the pairwise tree across the L lanes of a segment (lane l holds the sum
// of elements [16 l, 16 l + 16)); a + b == b + a exactly, so every lane gets the same value
template <int L>
__device__ __forceinline__ float seg_sum(float v) {
#pragma unroll
    for (int off = 1; off < L; off <<= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, off));
    return v;
}

// the packed layout of b-bit codes [HQQ 算法解读, "为什么一定要分组"]: cpw codes per 32-bit word,
// each in a slot of `slot` bits, the lowest index in the lowest bits.  4 bit two per byte, 2 bit
// four per byte, 3 bit ten per word; 5- and 6-bit codes one per byte (unpacked), and so 7 and 8
// bit; 1-bit codes eight per byte.
template <int NB>
struct Pack {
    static_assert(NB >= 1 && NB <= 8, "1- to 8-bit codes");
    static constexpr int slot = NB == 3 ? 3 : NB <= 4 ? NB : 8;
    static constexpr int cpw = NB == 3 ? 10 : 32 / slot;
};
// the tile engine reads W_hat = (k - z)/s from a table of the 2^b code values up to 4 bits; wider
// codes divide per element (a 32..256-entry table per group and round would cost more)
template <int NB>
struct TileTab {
    static constexpr bool on = NB <= 4;
    static constexpr int nq = on ? (1 << NB) : 0;
};


// workspace words after the per-round sums: CTAs finished, kept round, rounds measured,
// number of stale tiles; then the per-tile largest f and the list of stale tiles
struct Ctl {
    unsigned done;      // tiles (or CTAs, stream engine) finished
    int b;              // kept round
    int run;            // rounds whose MAE was computed
    int nstale;         // stale tiles (tile engine)
    unsigned long long work;  // next group to hand out (stream engine)
    unsigned long long pad[5];
};
static_assert(sizeof(Ctl) == 64, "control words: 64 bytes after the round sums");

// Programmatic dependent launch: a kernel launched with programmatic stream serialization may
// become resident while its predecessor still runs; wait_prerequisite() returns once the
// predecessor grid has completed and its writes are visible, and allow_dependents() lets the
// next grid be scheduled once every CTA of this one has called it (or exited).
__device__ __forceinline__ void wait_prerequisite() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// zeroes the per-call round sums and control words of the workspace (n 64-bit words)
__global__ void __launch_bounds__(256) hqq_zero_kernel(u64 *acc, int n) {
    allow_dependents();
    for (int i = threadIdx.x; i < n; i += blockDim.x) acc[i] = 0ull;
}

__device__ __forceinline__ Ctl *ctl_of(const QParams &P) {
    return reinterpret_cast<Ctl *>(P.acc + 4 * (P.K > 0 ? P.K : 1));
}

// The stop rule [HQQ 算法解读, "第二拍"]: round i's tensor error is direct[i] + sum_{j<=i} D[j];
// the loop keeps going while it is strictly below the best so far.  b = the kept round.
__device__ void stop_rule(const QParams &P) {
    const int K = P.K;
    unsigned __int128 cum = 0, best = 0;
    int b = 0, run = 0;
    bool stopped = false;
    for (int i = 0; i < K; ++i) {
        const u64 dlo = __ldcg(P.acc + 2 * (K + i)), dhi = __ldcg(P.acc + 2 * (K + i) + 1);
        const u64 lo = __ldcg(P.acc + 2 * i), hi = __ldcg(P.acc + 2 * i + 1);
        cum += ((unsigned __int128)dhi << 64) | dlo;
        const unsigned __int128 tot = (((unsigned __int128)hi << 64) | lo) + cum;
        if (P.err_trace) {
            P.err_trace[2 * i] = (u64)tot;
            P.err_trace[2 * i + 1] = (u64)(tot >> 64);
        }
        if (!stopped) {
            run = i + 1;
            if (i == 0 || tot < best) {
                best = tot;
                b = i;
            } else {
                stopped = true;
            }
        }
    }
    Ctl *c = ctl_of(P);
    c->b = b;
    c->run = run;
    if (P.iters_run) *P.iters_run = run;
}

// shared-memory layout of a tile-engine CTA (also used on the host to size tiles)
struct SmemLayout {
    int wh, s_t, z_t, lo_t, hi_t, f_t, tab, acc, thr, beta, total;
};

__host__ __device__ inline SmemLayout smem_layout(int tile, int rs, int nq, int L, int K) {
    SmemLayout s;
    const int Kc = K > 0 ? K : 1;
    int o = 0;
    s.wh = o; o += (tile * rs * 2 + 15) / 16 * 16;
    s.s_t = o; o += tile * 4;
    s.z_t = o; o += tile * 4;
    s.lo_t = o; o += tile * 4;
    s.hi_t = o; o += tile * 4;
    s.f_t = o; o += (tile + 15) / 16 * 16;
    s.tab = o; o += kWarps * nq * (32 / L) * 4;
    s.acc = o; o += kWarps * 2 * Kc * 4 * 4;  // per warp: [2][K] x 4 chunks
    s.thr = o; o += (Kc * 4 + 15) / 16 * 16;
    s.beta = o; o += Kc * 8;
    s.total = o;
    return s;
}

// ------------------------------------------------------------------------------------------
// pairwise sums, shared-memory access, the table of reconstructions and the residual bound
// ------------------------------------------------------------------------------------------

// push a chunk's sum onto a pairwise stack: after chunk ch, level l holds the sum of the last
// 2^l chunks whenever bit l of ch + 1 is set; the final entry is the whole pairwise sum
template <int LOGN>
__device__ __forceinline__ void pw_push(float (&stk)[LOGN + 1], int ch, float v) {
#pragma unroll
    for (int lvl = 0; lvl <= LOGN; ++lvl) {
        if ((ch >> lvl) & 1) {
            v = __fadd_rn(stk[lvl], v);
        } else {
            stk[lvl] = v;
            return;
        }
    }
}

__device__ __forceinline__ float tree8(const float *x) {
    return __fadd_rn(__fadd_rn(__fadd_rn(x[0], x[1]), __fadd_rn(x[2], x[3])),
                     __fadd_rn(__fadd_rn(x[4], x[5]), __fadd_rn(x[6], x[7])));
}

// the 8-element pairwise trees of two chunks at once (x[m] = element m of each chunk)
__device__ __forceinline__ float2 tree8x2(const float2 *x) {
    return __fadd2_rn(__fadd2_rn(__fadd2_rn(x[0], x[1]), __fadd2_rn(x[2], x[3])),
                      __fadd2_rn(__fadd2_rn(x[4], x[5]), __fadd2_rn(x[6], x[7])));
}

// the same for |x|: the first level in scalar adds, which take |.| for free
__device__ __forceinline__ float2 abs_tree8x2(const float2 *x) {
    float2 l1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        l1[i] = make_float2(__fadd_rn(fabsf(x[2 * i].x), fabsf(x[2 * i + 1].x)),
                            __fadd_rn(fabsf(x[2 * i].y), fabsf(x[2 * i + 1].y)));
    return __fadd2_rn(__fadd2_rn(l1[0], l1[1]), __fadd2_rn(l1[2], l1[3]));
}

__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v));
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// The reconstructions W_hat_k = (k - z)/s of every code k [HQQ 算法解读, "第二拍"], correctly
// rounded, into this lane's table column (entry k at col + 128 k).  Each quotient is
// (k - z) * y with y = RN(1/s), refined by two remainder corrections q + RN(a - s q) * y
// (Markstein, IBM J. Res. Dev. 34(1), 1990: with y = RN(1/s) and q within one ulp of a/s,
// the correction rounds to RN(a/s)).  The first correction brings the product within one
// ulp; the second then rounds it.  The quotients and remainders must stay in the normal
// range: every nonzero |k - z| is at least min(|z|, 2^-25), so |z| >= 2^-60 (or z = 0) with
// 2^-60 <= s <= 2^30 keeps each nonzero quotient above 2^-90 and each nonzero remainder
// above 2^-110.  Outside that the lane divides.
// the reconstructions by IEEE division, for the groups outside the Markstein conditions (rare:
// kept out of line so that the common path stays short)
template <int NQ>
__device__ __noinline__ void build_table_div(uint32_t col, float s, float z) {
    for (int k = 0; k < NQ; ++k) sts_f32(col + 128u * k, __fdiv_rn(__fsub_rn((float)k, z), s));
}

template <int NQ>
__device__ __forceinline__ void build_table(uint32_t col, float s, float y, float z) {
    if ((z == 0.0f || fabsf(z) >= 0x1p-60f) && s >= 0x1p-60f && s <= 0x1p30f) {
        const float2 y2 = make_float2(y, y), ns2 = make_float2(-s, -s), nz2 = make_float2(-z, -z);
#pragma unroll
        for (int k = 0; k < NQ; k += 2) {
            const float2 a = __fadd2_rn(make_float2((float)k, (float)(k + 1)), nz2);  // k - z
            const float2 q0 = __fmul2_rn(a, y2);
            const float2 q1 = __ffma2_rn(__ffma2_rn(q0, ns2, a), y2, q0);
            const float2 q2 = __ffma2_rn(__ffma2_rn(q1, ns2, a), y2, q1);
            sts_f32(col + 128u * k, q2.x);
            sts_f32(col + 128u * (k + 1), q2.y);
        }
    } else {
        build_table_div<NQ>(col, s, z);
    }
}

// An upper bound on every |RN(W - W_hat)| of the round, from the group's state alone:
// lz = RN(lo + z) and hz = RN(hi + z) are the smallest and largest W s + z of the group, so
// |t - q| <= max(1/2, -lz, hz - qmax).  The rounding of W s, of + z, of the table and of the
// difference adds less than (3A + 4|z| + 3 qmax) 2^-24 with A = max(|lo|, |hi|), and the
// bound is taken twice that wide and scaled by 1 + 2^-20 to cover its own rounding.
__device__ __forceinline__ float resid_bound(float lz, float hz, float A, float z, float y,
                                             float qmax) {
    const float M = fmaxf(0.5f, fmaxf(-lz, __fsub_rn(hz, qmax)));
    const float slack = __fmul_rn(__fadd_rn(__fmul_rn(8.0f, __fadd_rn(A, fabsf(z))), 4.0f * qmax), 0x1p-23f);
    return __fmul_rn(__fmul_rn(__fadd_rn(M, slack), y), 1.0f + 0x1p-20f);
}


// The rare paths read the group's row back from global memory (it is cached), so the
// unrolled register copy stays out of them.
//
// The zero-update sum with the exact lp shrink e = shrink(W - W_hat) for every element:
// pairwise in the same order as stream_round (8-element chunks, then a stack over chunks).
template <int NB>
__device__ __noinline__ float group_zsum_shrink(const __half *wrow, int g, int P, float s,
                                                float z, uint32_t tab_adj, double beta,
                                                double p) {
    constexpr float kQmax = (float)((1 << NB) - 1);
    float stk[6];
    const int nch = P / 8;
    for (int ch = 0; ch < nch; ++ch) {
        float tm[8];
        for (int m = 0; m < 8; ++m) {
            const int j = 8 * ch + m;
            float term = 0.0f;
            if (j < g) {
                const float w = __half2float(wrow[j]);
                const float t = fminf(fmaxf(__fadd_rn(__fmul_rn(w, s), z), 0.0f), kQmax);
                const float u = __fadd_rn(t, kMagic);
                const float qf = __fsub_rn(u, kMagic);
                const float what = lds_f32(tab_adj + (__float_as_uint(u) << 7));
                const float e = shrink_lp(__fsub_rn(w, what), beta, p);
                term = __fsub_rn(qf, __fmul_rn(__fsub_rn(w, e), s));
            }
            tm[m] = term;
        }
        float v = tree8(tm);
        int lvl = 0;
        for (; (ch >> lvl) & 1; ++lvl) v = __fadd_rn(stk[lvl], v);
        stk[lvl] = v;
    }
    int top = 0;
    while ((1 << top) < nch) ++top;
    return stk[top];
}

__device__ __forceinline__ void prefetch_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// the slot swizzle of a lane: the P/8 chunks of lanes l .. l+7 (one quarter warp of 16-byte
// accesses) must land in 8 different 16-byte bank groups
// (a slot of one chunk needs none: consecutive lanes' chunks are already consecutive)
template <int P>
__device__ __forceinline__ int slot_swizzle(int lane) {
    constexpr int C = P / 8;  // chunks per slot: 1, 2, 4, 8 or 16
    static_assert(C >= 1 && (C & (C - 1)) == 0, "slots hold a power of two of 16-byte chunks");
    return C >= 8 ? (lane & 7) : C == 4 ? ((lane >> 1) & 3) : C == 2 ? ((lane >> 2) & 1) : 0;
}

// position of the k-th (from 0) set bit of mask, or -1
__device__ __forceinline__ int nth_set_bit(unsigned mask, int k) {
    for (int i = 0; i < k; ++i) mask &= mask - 1u;
    return __ffs(mask) - 1;
}

// one table entry (k - z)/s, correctly rounded, under the same conditions as build_table
__device__ __forceinline__ float table_entry(float k, float s, float y, float z) {
    if ((z == 0.0f || fabsf(z) >= 0x1p-60f) && s >= 0x1p-60f && s <= 0x1p30f) {
        const float a = __fsub_rn(k, z);
        const float q0 = __fmul_rn(a, y);
        const float q1 = __fmaf_rn(__fmaf_rn(-q0, s, a), y, q0);
        return __fmaf_rn(__fmaf_rn(-q1, s, a), y, q1);
    }
    return __fdiv_rn(__fsub_rn(k, z), s);
}

// launches kernel<<<grid, block, smem, st>>>(args...) with programmatic stream serialization:
// the launch overlaps the kernel before it, which the kernel waits for in wait_prerequisite()
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, int smem,
                       cudaStream_t st, Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// the sum over a warp of a 64-bit value per lane, exact (each value below 2^63; the sum must
// fit in 64 bits): three 21-bit slices, each summed by redux.sync without overflow
__device__ __forceinline__ u64 warp_sum64(u64 v) {
    const unsigned a = __reduce_add_sync(kFull, (unsigned)(v & 0x1fffffu));
    const unsigned b = __reduce_add_sync(kFull, (unsigned)((v >> 21) & 0x1fffffu));
    const unsigned c = __reduce_add_sync(kFull, (unsigned)(v >> 42));
    return (u64)a + ((u64)b << 21) + ((u64)c << 42);
}

}  // namespace

// ------------------------------------------------------------------------------------------
// host side: the launchers each translation unit exports to the C ABI
// ------------------------------------------------------------------------------------------
namespace hqq_impl {

// the tile engine (axis 0, 3-bit and the 1-, 5- to 8-bit codes, group sizes that are not whole
// power-of-two rows); one launcher per code width, in two translation units
cudaError_t launch_tile_engine(const QParams &P, int nbits, int L, bool full, bool direct,
                               int64_t ntiles, cudaStream_t st);
template <int NB>
cudaError_t launch_tile_nb(const QParams &P, int L, bool full, bool direct, int64_t ntiles,
                           cudaStream_t st);
// the stream engine (axis 1, 2- or 4-bit codes, group size 16, 32, 64 or 128)
cudaError_t launch_stream_engine(const QParams &P, int nbits, int group_size, cudaStream_t st);
cudaError_t launch_dequantize(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                              int64_t N, int g, int64_t G, int axis, int64_t pb, __half *out,
                              cudaStream_t st);
// the tensor-core product of a batch (axis 1, 2- or 4-bit codes, group size a multiple of 8,
// cols a multiple of 64, X 16-byte aligned)
bool gemm_tc_layout(int nbits, int64_t rows, int64_t cols, int64_t g, int axis, const void *X);
cudaError_t launch_gemm_tc(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                           int64_t rows, int64_t cols, int64_t g, const __half *X, int64_t batch,
                           float *Y, cudaStream_t st);
cudaError_t launch_gemv(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                        int64_t rows, int64_t cols, int64_t g, int64_t G, int axis,
                        const __half *x, float *y, cudaStream_t st);

}  // namespace hqq_impl
