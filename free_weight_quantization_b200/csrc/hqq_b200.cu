// hqq_b200.cu -- HQQ group-wise weight quantization for B200 (sm_100a): kernels + C ABI.
//
// Method: the page "HQQ 算法解读：不用校准数据，怎样把大模型权重压到 4 bit"
// (ludovicoyin.github.io/blog/posts/hqq-half-quadratic-quantization), cited as
// [HQQ 算法解读, <section>].  The arithmetic reproduces, operation for operation, the binary32
// definition stated in include/hqq_b200.h: every product and sum rounded separately
// (__fmul_rn/__fadd_rn, no contraction), IEEE division for W_hat = (q - z)/s, round half to
// even, pairwise (recursive-halving) group sums, the lp shrink in binary64, and an exact
// fixed-point (2^-32) 128-bit tensor-wide error sum for the stop rule.
//
// Design (no tensor cores: nothing here is a dense contraction; the loop is ALU-bound):
//   search kernel  one CTA per tile of ~10k weights.  The tile is read from HBM once with
//                  16-byte loads and kept in shared memory as binary32, one padded row per
//                  group.  Warps are split into segments of L = P/16 lanes (P = group size
//                  rounded up to a power of two >= 16); each lane holds 16 consecutive
//                  elements of its group in registers, so a group's pairwise sums are a
//                  16-element in-lane tree plus log2(L) xor-shuffle levels.  A segment runs
//                  its group round after round until the zero stops moving (z_{i+1} == z_i
//                  with every residual below the last round's shrink threshold: every later
//                  round would repeat it exactly) or `iters` rounds are done, then takes the
//                  next group of the tile from a shared counter, so finished groups free
//                  their lanes.  Each round's per-group error goes to exact per-round
//                  accumulators (a frozen group's error is carried to all later rounds with a
//                  difference array).  The group's codes for its last round are packed with
//                  the rest of the tile and written once.
//   fixup kernel   evaluates the stop rule from the accumulators.  A group whose own last
//                  round lies beyond the global stopping point is stale; only tiles holding a
//                  stale group are recomputed (replaying exactly min(b, f) zero updates).
//   dequant kernel one thread per 16 packed bytes, 16-byte loads and stores.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>

#include "hqq_b200.h"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kE = 16;  // elements per lane
constexpr unsigned kFull = 0xffffffffu;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: x + kMagic rounds x to an integer (RNE)

typedef unsigned long long u64;

struct QParams {
    const __half *W;
    int64_t N, G;
    int g;          // group size
    int axis;
    int K;          // iteration cap
    int stride;     // floats per group row in shared memory (P + 4)
    int tile;       // groups per tile
    uint8_t *packed;
    int64_t packed_bytes;
    __half *scale, *zero;
    float *s_out, *z_out;
    u64 *acc;       // [K][2] direct round sums, then [K][2] difference array
    uint8_t *fk;    // [G] last round run by each group in the search kernel
    uint8_t *codes_u8;  // [N] byte-per-code staging when the packed layout is not tile aligned
    int32_t *iters_run;
    u64 *err_trace;
    float eps_tiny, scale_max;
    double p;
    double beta[HQQ_MAX_ITERS];
    float thr[HQQ_MAX_ITERS];  // |r| <= thr[i] guarantees shrink(r, beta_i) == 0
};

// ------------------------------------------------------------------------------------------
// small device helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ u64 err_fixed(float err) {
    // floor(err * 2^32): the scaling is exact in binary32; truncation toward zero
    return __float2ull_rz(__fmul_rn(err, 4294967296.0f));
}

__device__ __forceinline__ void acc_add(u64 *lohi, u64 v) {
    // 128-bit accumulate (low, high) with exact carry; works on shared or global memory
    u64 old = atomicAdd(lohi, v);
    if (old + v < old) atomicAdd(lohi + 1, 1ull);
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

template <int L>
__device__ __forceinline__ float seg_max(float v) {
#pragma unroll
    for (int off = 1; off < L; off <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
    return v;
}

template <int L>
__device__ __forceinline__ float seg_min(float v) {
#pragma unroll
    for (int off = 1; off < L; off <<= 1) v = fminf(v, __shfl_xor_sync(kFull, v, off));
    return v;
}

template <int NB>
struct Pack;  // codes per 32-bit output word
template <> struct Pack<4> { static constexpr int cpw = 8; };
template <> struct Pack<2> { static constexpr int cpw = 16; };
template <> struct Pack<3> { static constexpr int cpw = 10; };

// ------------------------------------------------------------------------------------------
// tile staging: fp16 W -> binary32 rows of the shared tile, one row of `stride` floats per
// group [HQQ 算法解读, "`axis` 不是一个无关紧要的开关"]
// ------------------------------------------------------------------------------------------
__device__ void stage_tile(const QParams &P, float *wt, int64_t t0, int tg) {
    const int g = P.g, stride = P.stride;
    if (P.axis == 1) {
        const int ne = tg * g;
        const __half *src = P.W + t0 * (int64_t)g;  // 16-byte aligned: tiles hold 320k elements
        const int nvec = ne >> 3;
        for (int v = threadIdx.x; v < nvec; v += kThreads) {
            uint4 x = __ldg(reinterpret_cast<const uint4 *>(src) + v);
            const __half *h = reinterpret_cast<const __half *>(&x);
            int e0 = v << 3;
            int grp = e0 / g, j = e0 - grp * g;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                wt[grp * stride + j] = __half2float(h[c]);
                if (++j == g) { j = 0; ++grp; }
            }
        }
        for (int e = (nvec << 3) + threadIdx.x; e < ne; e += kThreads) {
            int grp = e / g;
            wt[grp * stride + (e - grp * g)] = __half2float(src[e]);
        }
    } else {
        // group c of the tile is column t0 + c of the [g, G] view: elements j*G + t0 + c
        const int64_t G = P.G;
        if ((G & 7) == 0) {
            const int nv = (tg + 7) >> 3;  // tg % 8 == 0 except possibly at the end (G % 8 == 0)
            for (int v = threadIdx.x; v < g * nv; v += kThreads) {
                int j = v / nv, cv = v - j * nv;
                uint4 x = __ldg(reinterpret_cast<const uint4 *>(P.W + j * G + t0) + cv);
                const __half *h = reinterpret_cast<const __half *>(&x);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    int col = cv * 8 + c;
                    if (col < tg) wt[col * stride + j] = __half2float(h[c]);
                }
            }
        } else {
            for (int v = threadIdx.x; v < g * tg; v += kThreads) {
                int j = v / tg, col = v - j * tg;
                wt[col * stride + j] = __half2float(P.W[j * G + t0 + col]);
            }
        }
    }
}

// min-max init of every group of the tile [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"]
template <int NB>
__device__ void init_tile(const QParams &P, const float *wt, float *s_t, float *z_t, int tg) {
    constexpr float kQmax = (float)((1 << NB) - 1);
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        const float *row = wt + i * P.stride;
        float mn = row[0], mx = row[0];
        for (int j = 1; j < P.g; ++j) {
            mn = fminf(mn, row[j]);
            mx = fmaxf(mx, row[j]);
        }
        float d = __fsub_rn(mx, mn);
        float s = (d < P.eps_tiny) ? 1.0f : __fdiv_rn(kQmax, d);
        s = fminf(s, P.scale_max);
        s_t[i] = s;
        z_t[i] = __fsub_rn(0.0f, __fmul_rn(mn, s));
    }
}

// ------------------------------------------------------------------------------------------
// the proximal loop [HQQ 算法解读, "第二拍：half-quadratic 迭代修正零点"]
//
// REPLAY = false (search): each group runs until frozen or K rounds; per-round errors go to
//   acc_d (direct) and acc_f (difference array); codes of the group's last round are left
//   in its tile row; f_tile[grp] = last round index.
// REPLAY = true (fixup): each group runs exactly n = min(b, f_tile[grp]) zero updates, then
//   its codes for z_n are left in its tile row.
// ------------------------------------------------------------------------------------------
template <int NB, int L, bool REPLAY>
__device__ void run_segments(const QParams &P, float *wt, float *s_t, float *z_t,
                             uint8_t *f_tile, float *tab, u64 *acc_d, u64 *acc_f, int *counter,
                             int tg, int b_stop) {
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    constexpr int NSEG = 32 / L;
    const int lane = threadIdx.x & 31;
    const int sg = lane / L, l = lane - sg * L, seg_base = sg * L;
    const unsigned seg_mask = (L == 32) ? kFull : (((1u << L) - 1u) << seg_base);
    const int K = P.K, g = P.g, stride = P.stride;
    const int nvalid = min(max(g - l * kE, 0), kE);
    const float g_f = (float)g;
    const float thr_last = K > 0 ? P.thr[K - 1] : 0.0f;

    float w[kE], ws[kE];
    float s = 1.0f, z = 0.0f;
    int grp = -1, it = 0, nupd = 0;
    bool exhausted = false;

    while (true) {
        // ---- refill idle segments with the next group of the tile
        const bool need = (grp < 0) && !exhausted;
        if (__any_sync(kFull, need)) {
            int cand = 0;
            if (need && l == 0) cand = atomicAdd(counter, 1);
            cand = __shfl_sync(kFull, cand, seg_base);
            if (need) {
                if (cand < tg) {
                    grp = cand;
                    const float4 *src = reinterpret_cast<const float4 *>(wt + grp * stride + l * kE);
#pragma unroll
                    for (int v = 0; v < kE / 4; ++v) {
                        float4 x = src[v];
                        w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
                    }
                    s = s_t[grp];
                    z = z_t[grp];
#pragma unroll
                    for (int m = 0; m < kE; ++m) ws[m] = __fmul_rn(w[m], s);
                    it = 0;
                    if (REPLAY) nupd = min(b_stop, (int)f_tile[grp]);
                } else {
                    exhausted = true;
                }
            }
        }
        const bool active = grp >= 0;
        if (!__any_sync(kFull, active)) break;

        const bool do_iter = active && (REPLAY ? (it < nupd) : (K > 0));
        bool done = active && (REPLAY ? (it >= nupd) : (K == 0));
        if (__any_sync(kFull, do_iter)) {
            const int ii = min(it, K - 1);
            // table of reconstructions W_hat = (k - z)/s for every code k of this group:
            // the same IEEE division the method performs per element, done once per code
            __syncwarp();
#pragma unroll
            for (int kk = 0; kk < (NQ + L - 1) / L; ++kk) {
                const int k = l + kk * L;
                if (k < NQ) tab[k * NSEG + sg] = __fdiv_rn(__fsub_rn((float)k, z), s);
            }
            __syncwarp();
            float absr[kE], term[kE];
            float maxr = 0.0f;
#pragma unroll
            for (int m = 0; m < kE; ++m) {
                float t = __fadd_rn(ws[m], z);
                t = fminf(fmaxf(t, 0.0f), kQmax);           // clip then round == round then clip
                const float u = __fadd_rn(t, kMagic);
                const float qf = __fsub_rn(u, kMagic);      // round half to even
                const float what = tab[(__float_as_int(u) & (NQ - 1)) * NSEG + sg];
                const float ar = fabsf(__fsub_rn(w[m], what));
                const bool valid = m < nvalid;
                absr[m] = valid ? ar : 0.0f;
                term[m] = valid ? __fsub_rn(qf, ws[m]) : 0.0f;  // q - (W - 0)*s
                maxr = fmaxf(maxr, absr[m]);
            }
            const float esum = seg_sum<L>(tree16(absr));
            float zsum = seg_sum<L>(tree16(term));
            // lp shrink: any residual above this round's safe threshold -> exact path
            const bool over = do_iter && (maxr > P.thr[ii]);
            const bool slow = (__ballot_sync(kFull, over) & seg_mask) != 0;
            if (__any_sync(kFull, slow)) {
                const double beta = P.beta[ii];
#pragma unroll
                for (int m = 0; m < kE; ++m) {
                    float t = __fadd_rn(ws[m], z);
                    t = fminf(fmaxf(t, 0.0f), kQmax);
                    const float u = __fadd_rn(t, kMagic);
                    const float qf = __fsub_rn(u, kMagic);
                    const float what = tab[(__float_as_int(u) & (NQ - 1)) * NSEG + sg];
                    const float r = __fsub_rn(w[m], what);
                    const float e = (slow && m < nvalid) ? shrink_lp(r, beta, P.p) : 0.0f;
                    term[m] = (m < nvalid) ? __fsub_rn(qf, __fmul_rn(__fsub_rn(w[m], e), s)) : 0.0f;
                }
                const float zs2 = seg_sum<L>(tree16(term));
                if (slow) zsum = zs2;
            }
            const float znew = __fdiv_rn(zsum, g_f);
            if (do_iter) {
                if (!REPLAY) {
                    const u64 fx = err_fixed(esum);
                    if (l == 0) acc_add(acc_d + 2 * it, fx);
                    const bool big = maxr > thr_last;
                    const bool seg_big = (__ballot_sync(seg_mask, big) & seg_mask) != 0;
                    const bool frozen = !slow && !seg_big && (znew == z);
                    if (frozen || it == K - 1) {
                        done = true;
                        if (it + 1 < K && l == 0) acc_add(acc_f + 2 * (it + 1), fx);
                    } else {
                        z = znew;
                        ++it;
                    }
                } else {
                    z = znew;
                    ++it;
                    done = it >= nupd;
                }
            }
        }
        // ---- a finished group leaves its codes for z in its own tile row
        if (done) {
            uint8_t *crow = reinterpret_cast<uint8_t *>(wt + grp * stride);
#pragma unroll
            for (int m = 0; m < kE; ++m) {
                if (m < nvalid) {
                    float t = __fadd_rn(ws[m], z);
                    t = fminf(fmaxf(t, 0.0f), kQmax);
                    crow[l * kE + m] = (uint8_t)(__float_as_int(__fadd_rn(t, kMagic)) & (NQ - 1));
                }
            }
            if (l == 0) {
                z_t[grp] = z;
                if (!REPLAY) f_tile[grp] = (uint8_t)it;
            }
            grp = -1;
        }
    }
}

// ------------------------------------------------------------------------------------------
// tile output: metadata [HQQ 算法解读, "量化公式"] and packed codes [HQQ 算法解读, "为什么一定要分组"]
// ------------------------------------------------------------------------------------------
template <int NB>
__device__ void write_tile(const QParams &P, const float *wt, const float *s_t, const float *z_t,
                           int64_t t0, int tg) {
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        const int64_t k = t0 + i;
        const float s = s_t[i], z = z_t[i];
        P.scale[k] = __float2half_rn(__fdiv_rn(1.0f, s));
        P.zero[k] = __float2half_rn(z);
        if (P.s_out) P.s_out[k] = s;
        if (P.z_out) P.z_out[k] = z;
    }
    const int g = P.g, stride = P.stride;
    const uint8_t *cb = reinterpret_cast<const uint8_t *>(wt);
    const int rowb = stride * 4;  // bytes per tile row
    if (P.codes_u8) {
        // byte-per-code staging, packed afterwards by pack_codes_kernel
        if (P.axis == 1) {
            for (int e = threadIdx.x; e < tg * g; e += kThreads) {
                const int grp = e / g;
                P.codes_u8[t0 * g + e] = cb[grp * rowb + (e - grp * g)];
            }
        } else {
            for (int v = threadIdx.x; v < tg * g; v += kThreads) {
                const int j = v / tg, col = v - j * tg;
                P.codes_u8[j * P.G + t0 + col] = cb[col * rowb + j];
            }
        }
        return;
    }
    constexpr int CPW = Pack<NB>::cpw;
    auto store_word = [&](int64_t widx, uint32_t word) {
        const int64_t off = widx * 4;
        if (off + 4 <= P.packed_bytes) {
            reinterpret_cast<uint32_t *>(P.packed)[widx] = word;
        } else {
            for (int b = 0; b < 4; ++b)
                if (off + b < P.packed_bytes) P.packed[off + b] = (uint8_t)(word >> (8 * b));
        }
    };
    if (P.axis == 1) {
        const int ne = tg * g;
        const int nw = (ne + CPW - 1) / CPW;
        const int64_t w0 = t0 * g / CPW;  // tiles start on a word boundary
        for (int wi = threadIdx.x; wi < nw; wi += kThreads) {
            const int e0 = wi * CPW;
            int grp = e0 / g, j = e0 - grp * g;
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                if (e0 + c < ne) {
                    word |= (uint32_t)cb[grp * rowb + j] << (NB * c);
                    if (++j == g) { j = 0; ++grp; }
                }
            }
            store_word(w0 + wi, word);
        }
    } else {
        // row j of the [g, G] view holds the tile's codes at flat j*G + t0 + col;
        // G % CPW == 0 and t0 % CPW == 0 here, so each row segment starts on a word
        const int nwr = (tg + CPW - 1) / CPW;
        for (int v = threadIdx.x; v < g * nwr; v += kThreads) {
            const int j = v / nwr, wr = v - j * nwr;
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                const int col = wr * CPW + c;
                if (col < tg) word |= (uint32_t)cb[col * rowb + j] << (NB * c);
            }
            store_word((j * P.G + t0) / CPW + wr, word);
        }
    }
}

struct SmemLayout {
    int wt, s_t, z_t, f_t, tab, acc, counter, total;
};

__host__ __device__ inline SmemLayout smem_layout(int tile, int stride, int nq, int L, int K) {
    SmemLayout s;
    int o = 0;
    s.wt = o; o += tile * stride * 4;
    s.s_t = o; o += tile * 4;
    s.z_t = o; o += tile * 4;
    s.f_t = o; o += (tile + 15) / 16 * 16;
    s.tab = o; o += kWarps * nq * (32 / L) * 4;
    s.acc = o; o += 2 * (K > 0 ? K : 1) * 16;
    s.counter = o; o += 16;
    s.total = o;
    return s;
}

template <int NB, int L>
__global__ void __launch_bounds__(kThreads) hqq_search_kernel(const __grid_constant__ QParams P) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
    float *wt = reinterpret_cast<float *>(smem + lay.wt);
    float *s_t = reinterpret_cast<float *>(smem + lay.s_t);
    float *z_t = reinterpret_cast<float *>(smem + lay.z_t);
    uint8_t *f_t = smem + lay.f_t;
    float *tab = reinterpret_cast<float *>(smem + lay.tab) + (threadIdx.x >> 5) * (1 << NB) * (32 / L);
    u64 *acc = reinterpret_cast<u64 *>(smem + lay.acc);
    int *counter = reinterpret_cast<int *>(smem + lay.counter);
    const int K = P.K;

    const int64_t t0 = (int64_t)blockIdx.x * P.tile;
    const int tg = (int)min((int64_t)P.tile, P.G - t0);
    for (int i = threadIdx.x; i < 4 * K; i += kThreads) acc[i] = 0;
    if (threadIdx.x == 0) *counter = 0;
    stage_tile(P, wt, t0, tg);
    __syncthreads();
    init_tile<NB>(P, wt, s_t, z_t, tg);
    __syncthreads();
    run_segments<NB, L, false>(P, wt, s_t, z_t, f_t, tab, acc, acc + 2 * K, counter, tg, 0);
    __syncthreads();
    write_tile<NB>(P, wt, s_t, z_t, t0, tg);
    for (int i = threadIdx.x; i < tg; i += kThreads) P.fk[t0 + i] = f_t[i];
    for (int i = threadIdx.x; i < 2 * K; i += kThreads) {
        const u64 v = acc[2 * i], hi = acc[2 * i + 1];
        if (v | hi) {
            acc_add(P.acc + 2 * i, v);
            if (hi) atomicAdd(P.acc + 2 * i + 1, hi);
        }
    }
}

// global stop rule from the accumulated round errors: returns the index of the kept round
// (z of that round is kept) and the number of rounds whose MAE was computed
__device__ void stop_rule(const QParams &P, int *b_out, int *run_out, bool write) {
    const int K = P.K;
    unsigned __int128 cum = 0, best = 0;
    bool have = false;
    int b = 0, run = 0;
    for (int i = 0; i < K; ++i) {
        cum += ((unsigned __int128)P.acc[2 * (K + i) + 1] << 64) | P.acc[2 * (K + i)];
        const unsigned __int128 tot =
            (((unsigned __int128)P.acc[2 * i + 1] << 64) | P.acc[2 * i]) + cum;
        if (write && P.err_trace) {
            P.err_trace[2 * i] = (u64)tot;
            P.err_trace[2 * i + 1] = (u64)(tot >> 64);
        }
        if (run == i) {  // still inside the loop
            run = i + 1;
            if (!have || tot < best) {
                have = true;
                best = tot;
                b = i;
            } else {
                if (!write) break;
                run = -run;  // stopped; keep writing the trace
            }
        }
    }
    if (run < 0) run = -run;
    *b_out = b;
    *run_out = run;
}

template <int NB, int L>
__global__ void __launch_bounds__(kThreads) hqq_fixup_kernel(const __grid_constant__ QParams P) {
    extern __shared__ __align__(16) unsigned char smem[];
    const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
    float *wt = reinterpret_cast<float *>(smem + lay.wt);
    float *s_t = reinterpret_cast<float *>(smem + lay.s_t);
    float *z_t = reinterpret_cast<float *>(smem + lay.z_t);
    uint8_t *f_t = smem + lay.f_t;
    float *tab = reinterpret_cast<float *>(smem + lay.tab) + (threadIdx.x >> 5) * (1 << NB) * (32 / L);
    int *counter = reinterpret_cast<int *>(smem + lay.counter);
    __shared__ int sh_b, sh_stale;

    if (threadIdx.x == 0) {
        int b = 0, run = 0;
        stop_rule(P, &b, &run, blockIdx.x == 0);
        if (blockIdx.x == 0 && P.iters_run) *P.iters_run = run;
        sh_b = b;
        sh_stale = 0;
        *counter = 0;
    }
    __syncthreads();
    const int b = sh_b;
    const int64_t t0 = (int64_t)blockIdx.x * P.tile;
    const int tg = (int)min((int64_t)P.tile, P.G - t0);
    int stale = 0;
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        const uint8_t f = P.fk[t0 + i];
        f_t[i] = f;
        stale |= (int)f > b;
    }
    if (__syncthreads_or(stale) == 0) return;
    stage_tile(P, wt, t0, tg);
    __syncthreads();
    init_tile<NB>(P, wt, s_t, z_t, tg);
    __syncthreads();
    run_segments<NB, L, true>(P, wt, s_t, z_t, f_t, tab, nullptr, nullptr, counter, tg, b);
    __syncthreads();
    write_tile<NB>(P, wt, s_t, z_t, t0, tg);
}

// byte-per-code staging -> packed words (only for axis = 0 layouts that tiles cannot pack)
template <int NB>
__global__ void pack_codes_kernel(const uint8_t *codes, int64_t N, uint8_t *packed,
                                  int64_t packed_bytes) {
    constexpr int CPW = Pack<NB>::cpw;
    const int64_t nw = (N + CPW - 1) / CPW;
    for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi < nw;
         wi += (int64_t)gridDim.x * blockDim.x) {
        uint32_t word = 0;
        for (int c = 0; c < CPW; ++c) {
            const int64_t n = wi * CPW + c;
            if (n < N) word |= (uint32_t)codes[n] << (NB * c);
        }
        const int64_t off = wi * 4;
        if (off + 4 <= packed_bytes) {
            reinterpret_cast<uint32_t *>(packed)[wi] = word;
        } else {
            for (int b = 0; b < 4; ++b)
                if (off + b < packed_bytes) packed[off + b] = (uint8_t)(word >> (8 * b));
        }
    }
}

// ------------------------------------------------------------------------------------------
// dequantize [HQQ 算法解读, "量化公式" and "从压缩文件到一次前向"]: W = (q - z) * Delta
// Each thread expands 16 packed bytes (4 words): 32, 64 or 40 codes.
// ------------------------------------------------------------------------------------------
template <int NB>
__global__ void __launch_bounds__(256) hqq_dequant_kernel(const uint8_t *__restrict__ packed,
                                                          const __half *__restrict__ scale,
                                                          const __half *__restrict__ zero,
                                                          int64_t N, int g, int64_t G, int axis,
                                                          int64_t packed_bytes,
                                                          __half *__restrict__ out) {
    constexpr int CPW = Pack<NB>::cpw;
    constexpr int CPT = 4 * CPW;  // codes per thread
    constexpr uint32_t MASK = (1u << NB) - 1u;
    const int64_t nchunks = (N + CPT - 1) / CPT;
    for (int64_t ch = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ch < nchunks;
         ch += (int64_t)gridDim.x * blockDim.x) {
        uint32_t wd[4];
        const int64_t boff = ch * 16;
        if (boff + 16 <= packed_bytes) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(packed) + ch);
            wd[0] = x.x; wd[1] = x.y; wd[2] = x.z; wd[3] = x.w;
        } else {
            for (int i = 0; i < 4; ++i) {
                uint32_t v = 0;
                for (int b = 0; b < 4; ++b) {
                    const int64_t o = boff + 4 * i + b;
                    if (o < packed_bytes) v |= (uint32_t)packed[o] << (8 * b);
                }
                wd[i] = v;
            }
        }
        const int64_t n0 = ch * CPT;
        int64_t k;
        int j = 0;
        if (axis == 1) {
            k = n0 / g;
            j = (int)(n0 - k * g);
        } else {
            k = n0 % G;
        }
        float zf = __half2float(zero[k]), df = __half2float(scale[k]);
        uint32_t res[CPT / 2];  // fp16 pairs, low half = lower index
#pragma unroll
        for (int c = 0; c < CPT; c += 2) {
            float v[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int cc = c + h;
                const uint32_t q = (wd[cc / CPW] >> (NB * (cc % CPW))) & MASK;
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)q), 8388608.0f);
                v[h] = __fmul_rn(__fsub_rn(qf, zf), df);
                // advance to the group of the next element
                if (axis == 1) {
                    if (++j == g) {
                        j = 0;
                        ++k;
                        if (k < G) { zf = __half2float(zero[k]); df = __half2float(scale[k]); }
                    }
                } else {
                    if (++k == G) k = 0;
                    if (n0 + cc + 1 < N) { zf = __half2float(zero[k]); df = __half2float(scale[k]); }
                }
            }
            const __half2 h2 = __floats2half2_rn(v[0], v[1]);
            uint32_t bits;
            memcpy(&bits, &h2, 4);
            res[c / 2] = bits;
        }
        if (n0 + CPT <= N) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + n0);
#pragma unroll
            for (int i = 0; i < CPT / 8; ++i)
                dst[i] = make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]);
        } else {
            unsigned short *o16 = reinterpret_cast<unsigned short *>(out + n0);
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                if (n0 + c < N) o16[c] = (unsigned short)(res[c / 2] >> (16 * (c % 2)));
        }
    }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
struct Plan {
    int64_t N, G;
    int g, P, L, stride, tile;
    int64_t ntiles;
    bool aligned;  // packed words can be written per tile
    size_t ws_acc, ws_fk, ws_codes, ws_total;
};

int64_t gcd64(int64_t a, int64_t b) {
    while (b) { int64_t t = a % b; a = b; b = t; }
    return a;
}

int cpw_of(int nbits) { return nbits == 4 ? 8 : nbits == 2 ? 16 : 10; }

int make_plan(int64_t rows, int64_t cols, int nbits, int64_t group_size, int axis, int iters,
              Plan *pl) {
    if (rows <= 0 || cols <= 0 || group_size <= 0) return HQQ_ERR_ARG;
    if (nbits != 2 && nbits != 3 && nbits != 4) return HQQ_ERR_ARG;
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
    pl->stride = P + 4;
    const int budget = 16384;  // floats of tile rows per CTA (64 KB)
    const int cap = (int)std::min<int64_t>(10240 / pl->g, budget / pl->stride);
    if (axis == 1) {
        // tiles of a multiple of 320 elements: word (8, 16, 10 codes) and 16-byte aligned
        const int unit = (int)(320 / gcd64(pl->g, 320));
        pl->tile = unit * std::max(1, cap / unit);
    } else {
        pl->tile = 80 * std::max(1, cap / 80);  // columns; 80 = lcm(8, 16, 10)
    }
    pl->ntiles = (pl->G + pl->tile - 1) / pl->tile;
    pl->aligned = axis == 1 || (pl->G % cpw_of(nbits) == 0);
    const int K = iters > 0 ? iters : 1;
    pl->ws_acc = (size_t)4 * K * sizeof(u64);
    pl->ws_fk = (size_t)((pl->G + 15) / 16 * 16);
    pl->ws_codes = pl->aligned ? 0 : (size_t)((N + 15) / 16 * 16);
    pl->ws_total = pl->ws_acc + pl->ws_fk + pl->ws_codes;
    return HQQ_OK;
}

bool aligned_to(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

template <int NB, int L>
cudaError_t launch_quant(const QParams &P, int64_t ntiles, cudaStream_t st) {
    const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
    cudaError_t e = cudaFuncSetAttribute(hqq_search_kernel<NB, L>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(hqq_fixup_kernel<NB, L>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lay.total);
    if (e != cudaSuccess) return e;
    hqq_search_kernel<NB, L><<<(unsigned)ntiles, kThreads, lay.total, st>>>(P);
    hqq_fixup_kernel<NB, L><<<(unsigned)ntiles, kThreads, lay.total, st>>>(P);
    if (P.codes_u8) {
        const int64_t nw = (P.N + Pack<NB>::cpw - 1) / Pack<NB>::cpw;
        const unsigned blocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 16);
        pack_codes_kernel<NB><<<blocks, 256, 0, st>>>(P.codes_u8, P.N, P.packed, P.packed_bytes);
    }
    return cudaGetLastError();
}

template <int NB>
cudaError_t launch_quant_l(const QParams &P, int L, int64_t ntiles, cudaStream_t st) {
    switch (L) {
    case 1: return launch_quant<NB, 1>(P, ntiles, st);
    case 2: return launch_quant<NB, 2>(P, ntiles, st);
    case 4: return launch_quant<NB, 4>(P, ntiles, st);
    case 8: return launch_quant<NB, 8>(P, ntiles, st);
    default: return launch_quant<NB, 16>(P, ntiles, st);
    }
}

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
    case 4: return (n + 1) / 2;
    case 2: return (n + 3) / 4;
    case 3: return 4 * ((n + 9) / 10);
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
                            float *z_f32, uint64_t *err_trace, void *workspace,
                            size_t workspace_bytes, void *stream) {
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
    P.fk = (uint8_t *)workspace + pl.ws_acc;
    P.codes_u8 = pl.aligned ? nullptr : (uint8_t *)workspace + pl.ws_acc + pl.ws_fk;
    P.iters_run = iters_run;
    P.err_trace = (u64 *)err_trace;
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
    if (cudaMemsetAsync(workspace, 0, pl.ws_acc, st) != cudaSuccess) return HQQ_ERR_CUDA;
    cudaError_t e;
    switch (nbits) {
    case 4: e = launch_quant_l<4>(P, pl.L, pl.ntiles, st); break;
    case 3: e = launch_quant_l<3>(P, pl.L, pl.ntiles, st); break;
    default: e = launch_quant_l<2>(P, pl.L, pl.ntiles, st); break;
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
    const int cpt = 4 * cpw_of(nbits);
    const int64_t nchunks = (pl.N + cpt - 1) / cpt;
    const unsigned blocks = (unsigned)std::min<int64_t>((nchunks + 255) / 256, (int64_t)1 << 30);
    const int64_t pb = hqq_packed_bytes(pl.N, nbits);
    cudaStream_t st = (cudaStream_t)stream;
    const uint8_t *pk = (const uint8_t *)packed;
    const __half *sc = (const __half *)scale, *ze = (const __half *)zero;
    __half *out = (__half *)W_out;
    switch (nbits) {
    case 4: hqq_dequant_kernel<4><<<blocks, 256, 0, st>>>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out); break;
    case 3: hqq_dequant_kernel<3><<<blocks, 256, 0, st>>>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out); break;
    default: hqq_dequant_kernel<2><<<blocks, 256, 0, st>>>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out); break;
    }
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
