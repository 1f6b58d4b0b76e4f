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
#include <mutex>

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
    u64 *acc;       // [K][2] direct round sums, [K][2] difference array, then control words
    uint8_t *fk;    // [G] last round run by each group in the search kernel
    uint8_t *codes_u8;  // [N] byte-per-code staging when the packed layout is not tile aligned
    int32_t *iters_run;
    u64 *err_trace;
    uint8_t *group_rounds;  // [G] nullable: rounds run by each group in the search kernel
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

// min-max init of every group of the tile [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"].
// Also keeps W*s of the group's min and max element: every element's W*s lies between them
// (rounding is monotonic), which bounds W*s + z without visiting the elements.
template <int NB>
__device__ void init_tile(const QParams &P, const float *wt, float *s_t, float *z_t, float *lo_t,
                          float *hi_t, int tg) {
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
        lo_t[i] = __fmul_rn(mn, s);
        hi_t[i] = __fmul_rn(mx, s);
    }
}

// ------------------------------------------------------------------------------------------
// the proximal loop [HQQ 算法解读, "第二拍：half-quadratic 迭代修正零点"]
//
// The CTA advances its tile round by round.  A list in shared memory holds the groups that
// are still active; each pass of a warp takes NSEG of them (one per segment of L lanes), so
// finished groups drop out and the remaining ones are packed onto as few warps as possible.
// Within a round every contribution goes to the same round index, which lets a warp add its
// segments' errors with native 32-bit reductions (16-bit chunks of the 64-bit fixed-point
// value) before one shared-memory add.
//
// REPLAY = false (search): a group leaves the list once frozen (z_{r+1} == z_r, no residual
//   above the last round's shrink threshold: every later round repeats round r exactly) or
//   after round K-1; its codes for z_r stay in its tile row and f_t = r.  Per-round error
//   sums go to acc_c[0][r]; a group frozen at r also adds its error to acc_c[1][r+1] (a
//   difference array: that error repeats in every later round).
// REPLAY = true (fixup): a group makes exactly n = min(b, f_t) zero updates and leaves its
//   codes for z_n in its tile row.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void warp_add_fixed(unsigned *dst, u64 v) {
    // exact sum over the warp of 64-bit values, as four 16-bit chunks (each chunk sum < 2^21)
    const unsigned c0 = __reduce_add_sync(kFull, (unsigned)(v & 0xffffu));
    const unsigned c1 = __reduce_add_sync(kFull, (unsigned)((v >> 16) & 0xffffu));
    const unsigned c2 = __reduce_add_sync(kFull, (unsigned)((v >> 32) & 0xffffu));
    const unsigned c3 = __reduce_add_sync(kFull, (unsigned)(v >> 48));
    if ((threadIdx.x & 31) == 0) {  // the row belongs to this warp alone
        dst[0] += c0;
        dst[1] += c1;
        dst[2] += c2;
        dst[3] += c3;
    }
}

// One round over the 16 elements a lane holds: t = W*s + z, q = round(clip(t)), W_hat from
// the code table, |W - W_hat| and q - W*s (the zero-update term with e = 0).  CLIP = false
// is used only when every t of the warp's groups is known to round inside [0, 2^b - 1].
template <int NB, int NSEG, bool CLIP, bool FULL>
__device__ __forceinline__ void round_elems(const float (&w)[kE], float s, float z,
                                            const float *tab, int sg, int nvalid,
                                            float (&absr)[kE], float (&term)[kE]) {
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
#pragma unroll
    for (int m = 0; m < kE; ++m) {
        const float wsm = __fmul_rn(w[m], s);
        float t = __fadd_rn(wsm, z);
        if (CLIP) t = fminf(fmaxf(t, 0.0f), kQmax);  // clip then round == round then clip
        const float u = __fadd_rn(t, kMagic);
        const float qf = __fsub_rn(u, kMagic);        // round half to even
        const float what = tab[(__float_as_int(u) & (NQ - 1)) * NSEG + sg];
        const float ar = fabsf(__fsub_rn(w[m], what));
        const float tm = __fsub_rn(qf, wsm);          // q - (W - 0)*s
        if (FULL) {
            absr[m] = ar;
            term[m] = tm;
        } else {
            absr[m] = m < nvalid ? ar : 0.0f;
            term[m] = m < nvalid ? tm : 0.0f;
        }
    }
}

// Each warp owns a contiguous slice of at most 64 groups of the tile and runs its rounds on
// its own (no block-wide barrier inside the loop).  The slice's active groups are the set
// bits of a 64-bit mask, listed in shared memory at the start of each round; a pass hands
// the next NSEG of them to the warp's segments.
template <int NB, int L, bool REPLAY, bool FULL>
__device__ void run_rounds(const QParams &P, const float *wt, const float *s_t, float *z_t,
                           const float *lo_t, const float *hi_t, uint8_t *f_t, float *tab,
                           uint8_t *list, unsigned *acc_w, int tg, int b_stop) {
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    constexpr int NSEG = 32 / L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sg = lane / L, l = lane - sg * L;
    const unsigned seg_mask = (L == 32) ? kFull : (((1u << L) - 1u) << (sg * L));
    const int K = P.K, stride = P.stride;
    const int nvalid = FULL ? kE : min(max(P.g - l * kE, 0), kE);
    const float g_f = (float)P.g, inv_g = 1.0f / (float)P.g;  // exact for FULL (g = 2^k)
    const float thr_last = K > 0 ? P.thr[K - 1] : 0.0f;
    const int rounds = REPLAY ? b_stop : K;
    const int gpw = (P.tile + kWarps - 1) / kWarps;  // <= 64 (host plan)
    const int g0 = warp * gpw;
    const int ng = max(0, min(gpw, tg - g0));

    u64 mask = 0;
    for (int gi = lane; gi < ng; gi += 32) {
        const bool go = REPLAY ? (min(b_stop, (int)f_t[g0 + gi]) > 0) : (K > 0);
        if (go) mask |= 1ull << gi;
        else if (!REPLAY) f_t[g0 + gi] = 0;
    }
    mask = ((u64)__reduce_or_sync(kFull, (unsigned)(mask >> 32)) << 32) |
           __reduce_or_sync(kFull, (unsigned)mask);

    for (int r = 0; r < rounds && mask; ++r) {
        const int n_act = __popcll(mask);
        __syncwarp();
        for (int i = lane; i < 64; i += 32)
            if ((mask >> i) & 1ull) list[__popcll(mask & ((1ull << i) - 1ull))] = (uint8_t)i;
        __syncwarp();
        const float thr_r = P.thr[r];
        u64 fx_acc = 0, fd_acc = 0, dmask = 0;
        for (int base = 0; base < n_act; base += NSEG) {
            const int idx = base + sg;
            const bool active = idx < n_act;
            const int gi = list[active ? idx : base];
            const int grp = g0 + gi;
            float w[kE];
            const float4 *src = reinterpret_cast<const float4 *>(wt + grp * stride + l * kE);
#pragma unroll
            for (int v = 0; v < kE / 4; ++v) {
                const float4 x = src[v];
                w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
            }
            const float s = s_t[grp];
            const float z = z_t[grp];
            // t of every element of the group lies in [lo + z, hi + z]: no clip is needed when
            // that range rounds inside [0, 2^b - 1]
            const bool inside = __fadd_rn(lo_t[grp], z) >= -0.5f && __fadd_rn(hi_t[grp], z) < kQmax + 0.5f;
            const bool noclip = __all_sync(kFull, inside);

            // reconstructions W_hat = (k - z)/s for every code k: the IEEE division of the
            // method, done once per code value instead of once per element
            __syncwarp();
#pragma unroll
            for (int kk = 0; kk < (NQ + L - 1) / L; ++kk) {
                const int k = l + kk * L;
                if (k < NQ) tab[k * NSEG + sg] = __fdiv_rn(__fsub_rn((float)k, z), s);
            }
            __syncwarp();
            float absr[kE], term[kE];
            if (noclip) round_elems<NB, NSEG, false, FULL>(w, s, z, tab, sg, nvalid, absr, term);
            else round_elems<NB, NSEG, true, FULL>(w, s, z, tab, sg, nvalid, absr, term);
            const float esum_l = tree16(absr);
            // the lane's largest residual is at most its partial sum; only when that bound
            // fails is the maximum taken
            float maxr = esum_l;
            if (__any_sync(kFull, esum_l > thr_last)) {
                maxr = 0.0f;
#pragma unroll
                for (int m = 0; m < kE; ++m) maxr = fmaxf(maxr, absr[m]);
            }
            const float esum = seg_sum<L>(esum_l);
            float zsum = seg_sum<L>(tree16(term));
            // lp shrink: a residual above the round's safe threshold -> exact binary64 path
            const bool slow = (__ballot_sync(kFull, active && maxr > thr_r) & seg_mask) != 0;
            if (__any_sync(kFull, slow)) {
                const double beta = P.beta[r];
#pragma unroll
                for (int m = 0; m < kE; ++m) {
                    float t = __fadd_rn(__fmul_rn(w[m], s), z);
                    t = fminf(fmaxf(t, 0.0f), kQmax);
                    const float u = __fadd_rn(t, kMagic);
                    const float qf = __fsub_rn(u, kMagic);
                    const float what = tab[(__float_as_int(u) & (NQ - 1)) * NSEG + sg];
                    const float rr = __fsub_rn(w[m], what);
                    const float e = (slow && m < nvalid) ? shrink_lp(rr, beta, P.p) : 0.0f;
                    term[m] = (m < nvalid) ? __fsub_rn(qf, __fmul_rn(__fsub_rn(w[m], e), s)) : 0.0f;
                }
                const float zs2 = seg_sum<L>(tree16(term));
                if (slow) zsum = zs2;
            }
            const float znew = FULL ? __fmul_rn(zsum, inv_g) : __fdiv_rn(zsum, g_f);

            bool done;
            float zfin;
            if (!REPLAY) {
                const bool big = (__ballot_sync(kFull, maxr > thr_last) & seg_mask) != 0;
                const bool frozen = !slow && !big && (znew == z);
                done = frozen || r == K - 1;
                zfin = z;
                if (active && l == 0) {
                    const u64 fx = err_fixed(esum);
                    fx_acc += fx;
                    if (done && r + 1 < K) fd_acc += fx;
                }
            } else {
                done = r + 1 >= min(b_stop, (int)f_t[grp]);
                zfin = znew;
            }
            if (active && l == 0) {
                z_t[grp] = done ? zfin : znew;
                if (done) {
                    if (!REPLAY) f_t[grp] = (uint8_t)r;
                    dmask |= 1ull << gi;
                }
            }
        }
        if (!REPLAY) {
            warp_add_fixed(acc_w + 4 * r, fx_acc);
            if (r + 1 < K) warp_add_fixed(acc_w + 4 * (K + r + 1), fd_acc);
        }
        dmask = ((u64)__reduce_or_sync(kFull, (unsigned)(dmask >> 32)) << 32) |
                __reduce_or_sync(kFull, (unsigned)dmask);
        mask &= ~dmask;
    }
}

// ------------------------------------------------------------------------------------------
// tile output: metadata [HQQ 算法解读, "量化公式"] and packed codes [HQQ 算法解读, "为什么一定要分组"]
// The final quantize with the original W and the kept z (section "第二拍") happens here: step 1
// turns each 16-element run of a group row into codes in a byte buffer laid out in flat
// tensor order for the tile; step 2 packs that buffer into 32-bit words.
// ------------------------------------------------------------------------------------------
template <int NB>
__device__ void write_tile(const QParams &P, const float *wt, const float *s_t, const float *z_t,
                           uint8_t *cbuf, int64_t t0, int tg) {
    constexpr float kQmax = (float)((1 << NB) - 1);
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        const int64_t k = t0 + i;
        const float s = s_t[i], z = z_t[i];
        P.scale[k] = __float2half_rn(__fdiv_rn(1.0f, s));
        P.zero[k] = __float2half_rn(z);
        if (P.s_out) P.s_out[k] = s;
        if (P.z_out) P.z_out[k] = z;
    }
    const int g = P.g, stride = P.stride;
    const int L = (P.stride - 4) / kE;  // lanes per group row (P / 16)
    // step 1: codes
    for (int it = threadIdx.x; it < tg * L; it += kThreads) {
        const int grp = it / L, l = it - grp * L;
        const int j0 = l * kE;
        if (j0 >= g) continue;
        const float s = s_t[grp], z = z_t[grp];
        const float4 *src = reinterpret_cast<const float4 *>(wt + grp * stride + j0);
        uint32_t qw[kE / 4];  // codes, four per word, lowest index in the lowest byte
#pragma unroll
        for (int v = 0; v < kE / 4; ++v) {
            const float4 x = src[v];
            const float xs[4] = {x.x, x.y, x.z, x.w};
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float t = fminf(fmaxf(__fadd_rn(__fmul_rn(xs[c], s), z), 0.0f), kQmax);
                word |= (uint32_t)(__float_as_int(__fadd_rn(t, kMagic)) & ((1 << NB) - 1)) << (8 * c);
            }
            qw[v] = word;
        }
        const int n = min(kE, g - j0);
        if (P.axis == 1) {
            uint8_t *dst = cbuf + grp * g + j0;
            if (n == kE && ((grp * g + j0) & 15) == 0) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(qw[0], qw[1], qw[2], qw[3]);
            } else {
#pragma unroll
                for (int m = 0; m < kE; ++m)
                    if (m < n) dst[m] = (uint8_t)(qw[m / 4] >> (8 * (m % 4)));
            }
        } else {
#pragma unroll
            for (int m = 0; m < kE; ++m)
                if (m < n) cbuf[(j0 + m) * tg + grp] = (uint8_t)(qw[m / 4] >> (8 * (m % 4)));
        }
    }
    __syncthreads();
    if (P.codes_u8) {  // byte-per-code staging, packed afterwards by pack_codes_kernel
        if (P.axis == 1) {
            for (int e = threadIdx.x; e < tg * g; e += kThreads) P.codes_u8[t0 * g + e] = cbuf[e];
        } else {
            for (int v = threadIdx.x; v < tg * g; v += kThreads) {
                const int j = v / tg, col = v - j * tg;
                P.codes_u8[j * P.G + t0 + col] = cbuf[v];
            }
        }
        return;
    }
    // step 2: words of CPW codes from the flat code buffer
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
    auto pack_word = [&](const uint8_t *c, int n) -> uint32_t {
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < CPW; ++k)
            if (k < n) word |= (uint32_t)c[k] << (NB * k);
        return word;
    };
    if (P.axis == 1) {
        const int ne = tg * g;
        const int nw = (ne + CPW - 1) / CPW;
        const int64_t w0 = t0 * g / CPW;  // tiles start on a word boundary
        for (int wi = threadIdx.x; wi < nw; wi += kThreads)
            store_word(w0 + wi, pack_word(cbuf + wi * CPW, min(CPW, ne - wi * CPW)));
    } else {
        // row j of the [g, G] view holds the tile's codes at flat j*G + t0 + col; here
        // G % CPW == 0 and t0 % CPW == 0, so each row segment starts on a word boundary
        const int nwr = (tg + CPW - 1) / CPW;
        for (int v = threadIdx.x; v < g * nwr; v += kThreads) {
            const int j = v / nwr, wr = v - j * nwr;
            store_word((j * P.G + t0) / CPW + wr,
                       pack_word(cbuf + j * tg + wr * CPW, min(CPW, tg - wr * CPW)));
        }
    }
}

struct SmemLayout {
    int wt, s_t, z_t, lo_t, hi_t, f_t, tab, list, acc, cbuf, total;
};

__host__ __device__ inline SmemLayout smem_layout(int tile, int stride, int nq, int L, int K) {
    SmemLayout s;
    int o = 0;
    s.wt = o; o += tile * stride * 4;
    s.s_t = o; o += tile * 4;
    s.z_t = o; o += tile * 4;
    s.lo_t = o; o += tile * 4;
    s.hi_t = o; o += tile * 4;
    s.f_t = o; o += (tile + 15) / 16 * 16;
    s.tab = o; o += kWarps * nq * (32 / L) * 4;
    s.list = o; o += kWarps * 64;
    s.acc = o; o += kWarps * 2 * (K > 0 ? K : 1) * 4 * 4;  // per warp: [2][K] x 4 chunks
    s.cbuf = o; o += (tile * (stride - 4) + 15) / 16 * 16;  // codes of the tile, one byte each
    s.total = o;
    return s;
}

template <int NB, int L>
struct Smem {
    float *wt, *s_t, *z_t, *lo_t, *hi_t, *tab;
    uint8_t *f_t, *list, *cbuf;
    unsigned *acc;  // all warps' rows
    unsigned *acc_w;  // this warp's row
    __device__ Smem(unsigned char *base, const QParams &P) {
        const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
        wt = reinterpret_cast<float *>(base + lay.wt);
        s_t = reinterpret_cast<float *>(base + lay.s_t);
        z_t = reinterpret_cast<float *>(base + lay.z_t);
        lo_t = reinterpret_cast<float *>(base + lay.lo_t);
        hi_t = reinterpret_cast<float *>(base + lay.hi_t);
        f_t = base + lay.f_t;
        list = base + lay.list + (threadIdx.x >> 5) * 64;
        cbuf = base + lay.cbuf;
        tab = reinterpret_cast<float *>(base + lay.tab) + (threadIdx.x >> 5) * (1 << NB) * (32 / L);
        acc = reinterpret_cast<unsigned *>(base + lay.acc);
        acc_w = acc + (threadIdx.x >> 5) * 8 * (P.K > 0 ? P.K : 1);
    }
};

// workspace words after the per-round sums: tiles finished, kept round, rounds measured
struct Ctl {
    unsigned done;
    int b;
    int run;
    int pad;
};

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

template <int NB, int L, bool FULL>
__global__ void __launch_bounds__(kThreads) hqq_search_kernel(const __grid_constant__ QParams P) {
    extern __shared__ __align__(16) unsigned char smem[];
    Smem<NB, L> S(smem, P);
    __shared__ bool last;
    const int K = P.K;
    const int64_t t0 = (int64_t)blockIdx.x * P.tile;
    const int tg = (int)min((int64_t)P.tile, P.G - t0);
    for (int i = threadIdx.x; i < kWarps * 8 * K; i += kThreads) S.acc[i] = 0;
    stage_tile(P, S.wt, t0, tg);
    __syncthreads();
    init_tile<NB>(P, S.wt, S.s_t, S.z_t, S.lo_t, S.hi_t, tg);
    __syncthreads();
    run_rounds<NB, L, false, FULL>(P, S.wt, S.s_t, S.z_t, S.lo_t, S.hi_t, S.f_t, S.tab, S.list,
                                   S.acc_w, tg, 0);
    __syncthreads();
    write_tile<NB>(P, S.wt, S.s_t, S.z_t, S.cbuf, t0, tg);
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        P.fk[t0 + i] = S.f_t[i];
        if (P.group_rounds) P.group_rounds[t0 + i] = K > 0 ? (uint8_t)(S.f_t[i] + 1) : 0;
    }
    // this tile's per-round sums (16-bit chunks) -> 128-bit global sums
    for (int i = threadIdx.x; i < 2 * K; i += kThreads) {
        unsigned __int128 v = 0;
        for (int wp = 0; wp < kWarps; ++wp) {
            const unsigned *c = S.acc + wp * 8 * K + 4 * i;
            v += (unsigned __int128)c[0] + ((unsigned __int128)c[1] << 16) +
                 ((unsigned __int128)c[2] << 32) + ((unsigned __int128)c[3] << 48);
        }
        const u64 lo = (u64)v, hi = (u64)(v >> 64);
        if (lo | hi) {
            const u64 old = atomicAdd(P.acc + 2 * i, lo);
            const u64 carry = (old + lo < old) ? 1ull : 0ull;
            if (hi + carry) atomicAdd(P.acc + 2 * i + 1, hi + carry);
        }
    }
    // the last tile to finish applies the stop rule once for the whole tensor
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&ctl_of(P)->done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (last && threadIdx.x == 0) {
        __threadfence();
        stop_rule(P);
    }
}

// Recomputes the tiles that hold a group whose own last round lies past the kept round b.
template <int NB, int L, bool FULL>
__global__ void __launch_bounds__(kThreads) hqq_fixup_kernel(const __grid_constant__ QParams P,
                                                              int64_t ntiles) {
    extern __shared__ __align__(16) unsigned char smem[];
    Smem<NB, L> S(smem, P);
    const int b = __ldcg(&ctl_of(P)->b);
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t t0 = tile * P.tile;
        const int tg = (int)min((int64_t)P.tile, P.G - t0);
        int stale = 0;
        for (int i = threadIdx.x; i < tg; i += kThreads) {
            const uint8_t f = P.fk[t0 + i];
            S.f_t[i] = f;
            stale |= (int)f > b;
        }
        if (__syncthreads_or(stale) == 0) continue;
        stage_tile(P, S.wt, t0, tg);
        __syncthreads();
        init_tile<NB>(P, S.wt, S.s_t, S.z_t, S.lo_t, S.hi_t, tg);
        __syncthreads();
        run_rounds<NB, L, true, FULL>(P, S.wt, S.s_t, S.z_t, S.lo_t, S.hi_t, S.f_t, S.tab, S.list,
                                      nullptr, tg, b);
        __syncthreads();
        write_tile<NB>(P, S.wt, S.s_t, S.z_t, S.cbuf, t0, tg);
        __syncthreads();
    }
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
// One packed 32-bit word (8, 16 or 10 codes) per lane and step, so that a warp's loads cover
// 128 contiguous bytes and its stores 512 contiguous bytes (4 bit).  A thread handles kDqU
// words spaced a block apart, all loaded before any is expanded.
//   MODE 0: axis 1, group_size a multiple of the codes per word: one group per word
//   MODE 1: axis 1, any group size
//   MODE 2: axis 0 (element n belongs to group n % G)
// ------------------------------------------------------------------------------------------
constexpr int kDqU = 4;
constexpr int kDqThreads = 256;

template <int NB, int MODE>
__global__ void __launch_bounds__(kDqThreads) hqq_dequant_kernel(
    const uint32_t *__restrict__ packed, const __half *__restrict__ scale,
    const __half *__restrict__ zero, int64_t N, int g, int64_t G, int64_t packed_bytes,
    int wpg_shift, bool vec_meta, __half *__restrict__ out) {
    constexpr int CPW = Pack<NB>::cpw;
    constexpr uint32_t MASK = (1u << NB) - 1u;
    const int64_t nwords = (N + CPW - 1) / CPW;
    const int64_t wbase = (int64_t)blockIdx.x * (kDqThreads * kDqU) + threadIdx.x;
    uint32_t wd[kDqU];
#pragma unroll
    for (int u = 0; u < kDqU; ++u) {
        const int64_t wi = wbase + u * kDqThreads;
        wd[u] = 0;
        if (wi < nwords) {
            if (wi * 4 + 4 <= packed_bytes) {
                wd[u] = __ldcs(packed + wi);
            } else {  // the last word of a byte-sized packing may be short
                const uint8_t *pb = reinterpret_cast<const uint8_t *>(packed);
                for (int b = 0; b < 4 && wi * 4 + b < packed_bytes; ++b)
                    wd[u] |= (uint32_t)pb[wi * 4 + b] << (8 * b);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kDqU; ++u) {
        const int64_t wi = wbase + u * kDqThreads;
        if (wi >= nwords) break;
        const int64_t n0 = wi * CPW;
        uint32_t res[(CPW + 1) / 2];
        float v[CPW];
        if (MODE == 0) {
            const int64_t k = wpg_shift >= 0 ? (wi >> wpg_shift) : (n0 / g);
            const float zf = __half2float(zero[k]), df = __half2float(scale[k]);
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (NB * c)) & MASK)), 8388608.0f);
                v[c] = __fmul_rn(__fsub_rn(qf, zf), df);
            }
        } else if (MODE == 2 && vec_meta) {
            // CPW consecutive groups starting at a multiple of 8: 16-byte metadata loads
            const int64_t k0 = n0 % G;
#pragma unroll
            for (int c8 = 0; c8 < CPW; c8 += 8) {
                const uint4 zv = __ldg(reinterpret_cast<const uint4 *>(zero + k0 + c8));
                const uint4 dv = __ldg(reinterpret_cast<const uint4 *>(scale + k0 + c8));
                const __half *zh = reinterpret_cast<const __half *>(&zv);
                const __half *dh = reinterpret_cast<const __half *>(&dv);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (NB * (c8 + c))) & MASK)), 8388608.0f);
                    v[c8 + c] = __fmul_rn(__fsub_rn(qf, __half2float(zh[c])), __half2float(dh[c]));
                }
            }
        } else {
            int64_t k;
            int j = 0;
            if (MODE == 1) {
                k = n0 / g;
                j = (int)(n0 - k * g);
            } else {
                k = n0 % G;
            }
            float zf = __half2float(zero[k]), df = __half2float(scale[k]);
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (NB * c)) & MASK)), 8388608.0f);
                v[c] = __fmul_rn(__fsub_rn(qf, zf), df);
                if (c + 1 < CPW && n0 + c + 1 < N) {  // move to the group of the next element
                    if (MODE == 1) {
                        if (++j == g) {
                            j = 0;
                            ++k;
                            zf = __half2float(zero[k]);
                            df = __half2float(scale[k]);
                        }
                    } else {
                        if (++k == G) k = 0;
                        zf = __half2float(zero[k]);
                        df = __half2float(scale[k]);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPW; c += 2) {
            const __half2 h2 = __floats2half2_rn(v[c], c + 1 < CPW ? v[c + 1] : 0.0f);
            memcpy(&res[c / 2], &h2, 4);
        }
        if (n0 + CPW <= N) {
            if (CPW % 8 == 0) {  // 16 or 32 bytes per word, 16-byte aligned
                uint4 *dst = reinterpret_cast<uint4 *>(out + n0);
#pragma unroll
                for (int i = 0; i < CPW / 8; ++i)
                    __stcs(dst + i, make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]));
            } else {  // 10 codes: 20 bytes, 4-byte aligned
                uint32_t *dst = reinterpret_cast<uint32_t *>(out + n0);
#pragma unroll
                for (int i = 0; i < CPW / 2; ++i) __stcs(dst + i, res[i]);
            }
        } else {
            unsigned short *o16 = reinterpret_cast<unsigned short *>(out + n0);
#pragma unroll
            for (int c = 0; c < CPW; ++c)
                if (n0 + c < N) o16[c] = (unsigned short)(res[c / 2] >> (16 * (c % 2)));
        }
    }
}

template <int NB>
void launch_dequant(const uint8_t *pk, const __half *sc, const __half *ze, int64_t N, int g,
                    int64_t G, int axis, int64_t pb, __half *out, cudaStream_t st) {
    constexpr int CPW = Pack<NB>::cpw;
    const int64_t nwords = (N + CPW - 1) / CPW;
    const unsigned blocks = (unsigned)((nwords + kDqThreads * kDqU - 1) / (kDqThreads * kDqU));
    const uint32_t *pw = reinterpret_cast<const uint32_t *>(pk);
    int shift = -1;
    if (g % CPW == 0) {
        const int wpg = g / CPW;
        if ((wpg & (wpg - 1)) == 0) { shift = 0; while ((1 << shift) < wpg) ++shift; }
    }
    const bool vec_meta = CPW % 8 == 0 && G % 8 == 0 && (((uintptr_t)sc | (uintptr_t)ze) & 15) == 0;
    if (axis == 1 && g % CPW == 0)
        hqq_dequant_kernel<NB, 0><<<blocks, kDqThreads, 0, st>>>(pw, sc, ze, N, g, G, pb, shift, false, out);
    else if (axis == 1)
        hqq_dequant_kernel<NB, 1><<<blocks, kDqThreads, 0, st>>>(pw, sc, ze, N, g, G, pb, -1, false, out);
    else
        hqq_dequant_kernel<NB, 2><<<blocks, kDqThreads, 0, st>>>(pw, sc, ze, N, g, G, pb, -1, vec_meta, out);
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
    const int cap2 = std::min(cap, kWarps * 64);  // each warp owns at most 64 groups
    if (axis == 1) {
        // tiles of a multiple of 320 elements: word (8, 16, 10 codes) and 16-byte aligned
        const int unit = (int)(320 / gcd64(pl->g, 320));
        pl->tile = unit * std::max(1, cap2 / unit);
    } else {
        pl->tile = 80 * std::max(1, cap2 / 80);  // columns; 80 = lcm(8, 16, 10)
    }
    if (pl->tile > kWarps * 64) return HQQ_ERR_UNSUPPORTED;
    pl->ntiles = (pl->G + pl->tile - 1) / pl->tile;
    pl->aligned = axis == 1 || (pl->G % cpw_of(nbits) == 0);
    const int K = iters > 0 ? iters : 1;
    pl->ws_acc = (size_t)4 * K * sizeof(u64) + 16;  // per-round sums + control words
    pl->ws_fk = (size_t)((pl->G + 15) / 16 * 16);
    pl->ws_codes = pl->aligned ? 0 : (size_t)((N + 15) / 16 * 16);
    pl->ws_total = pl->ws_acc + pl->ws_fk + pl->ws_codes;
    return HQQ_OK;
}

bool aligned_to(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

template <int NB, int L, bool FULL>
cudaError_t launch_quant(const QParams &P, int64_t ntiles, cudaStream_t st) {
    const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
    cudaError_t e = cudaFuncSetAttribute(hqq_search_kernel<NB, L, FULL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(hqq_fixup_kernel<NB, L, FULL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    hqq_search_kernel<NB, L, FULL><<<(unsigned)ntiles, kThreads, lay.total, st>>>(P);
    const unsigned fix_blocks = (unsigned)std::min<int64_t>(ntiles, 148 * 4);
    hqq_fixup_kernel<NB, L, FULL><<<fix_blocks, kThreads, lay.total, st>>>(P, ntiles);
    if (P.codes_u8) {
        const int64_t nw = (P.N + Pack<NB>::cpw - 1) / Pack<NB>::cpw;
        const unsigned blocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 16);
        pack_codes_kernel<NB><<<blocks, 256, 0, st>>>(P.codes_u8, P.N, P.packed, P.packed_bytes);
    }
    return cudaGetLastError();
}

template <int NB>
cudaError_t launch_quant_l(const QParams &P, int L, bool full, int64_t ntiles, cudaStream_t st) {
    if (full) {  // group size a power of two >= 16: every slot of a lane holds an element
        switch (L) {
        case 1: return launch_quant<NB, 1, true>(P, ntiles, st);
        case 2: return launch_quant<NB, 2, true>(P, ntiles, st);
        case 4: return launch_quant<NB, 4, true>(P, ntiles, st);
        case 8: return launch_quant<NB, 8, true>(P, ntiles, st);
        default: return launch_quant<NB, 16, true>(P, ntiles, st);
        }
    }
    switch (L) {
    case 1: return launch_quant<NB, 1, false>(P, ntiles, st);
    case 2: return launch_quant<NB, 2, false>(P, ntiles, st);
    case 4: return launch_quant<NB, 4, false>(P, ntiles, st);
    case 8: return launch_quant<NB, 8, false>(P, ntiles, st);
    default: return launch_quant<NB, 16, false>(P, ntiles, st);
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
    P.fk = (uint8_t *)workspace + pl.ws_acc;
    P.codes_u8 = pl.aligned ? nullptr : (uint8_t *)workspace + pl.ws_acc + pl.ws_fk;
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
    if (cudaMemsetAsync(workspace, 0, pl.ws_acc, st) != cudaSuccess) return HQQ_ERR_CUDA;
    cudaError_t e;
    switch (nbits) {
    case 4: e = launch_quant_l<4>(P, pl.L, pl.g == pl.P, pl.ntiles, st); break;
    case 3: e = launch_quant_l<3>(P, pl.L, pl.g == pl.P, pl.ntiles, st); break;
    default: e = launch_quant_l<2>(P, pl.L, pl.g == pl.P, pl.ntiles, st); break;
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
    switch (nbits) {
    case 4: launch_dequant<4>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
    case 3: launch_dequant<3>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
    default: launch_dequant<2>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
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

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
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
