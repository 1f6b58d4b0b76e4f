// hqq_b200.cu -- HQQ group-wise weight quantization for B200 (sm_100a): kernels + C ABI.
//
// Method: the page "HQQ 算法解读：不用校准数据，怎样把大模型权重压到 4 bit"
// (ludovicoyin.github.io/blog/posts/hqq-half-quadratic-quantization), cited as
// [HQQ 算法解读, <section>].  The arithmetic reproduces, operation for operation, the binary32
// definition stated in include/hqq_b200.h: every product and sum rounded separately
// (__fmul_rn/__fadd_rn and their packed .f32x2 forms, no contraction), W_hat = (q - z)/s
// correctly rounded (a reciprocal product with Markstein's remainder corrections gives the
// same bits as IEEE division), round half to even, pairwise (recursive-halving) group sums,
// the lp shrink in binary64, and an exact fixed-point (2^-32) 128-bit tensor-wide error sum
// for the stop rule.
//
// Design (no tensor cores: nothing here is a dense contraction; the loop is ALU-bound):
//   A quantize call launches a one-block zero kernel for the round sums, then one of two
//   engines and a fixup kernel, each later kernel with programmatic stream serialization so
//   that its launch overlaps the kernel before it (griddepcontrol.wait orders the data).
//   stream engine  axis 1, 2- or 4-bit codes, power-of-two groups of 16..128 that fill whole
//                  32-bit words: a persistent kernel with one group per lane.  The lane
//                  keeps the group's fp16 row in registers for all its rounds, its table of
//                  the 2^b reconstructions in its own shared-memory column, and the next
//                  group's row in a swizzled shared-memory slot (cp.async, one group ahead).
//                  Groups come from a global counter; once it is empty, idle lanes take the
//                  queued groups of busy ones, and a warp's last few groups are split over
//                  segments of lanes.
//   tile engine    everything else (axis 0, 3-bit, other group sizes): one CTA per tile of
//                  groups staged in shared memory, segments of L = P/16 lanes per group.
//   Both engines run a group round after round until its zero stops moving (z_{i+1} == z_i
//   with every residual provably below the last round's shrink threshold: every later round
//   would repeat it exactly) or `iters` rounds are done; a group's error goes to exact
//   per-round counters (a frozen group's error is carried to later rounds by a difference
//   array), and its last round's codes are its final codes.  The last CTA to finish applies
//   the stop rule; the fixup kernel recomputes the few groups whose own last round lies past
//   the kept one, replaying exactly min(b, f) zero updates.
//   dequant        one packed 32-bit word per lane per step, coalesced loads and stores.
//   gemv           dequantize fused into y = W_hat @ x for one input vector.
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
    int stride;     // floats per group row of the shared tile
    int tile;       // groups per tile
    int stream_warps;  // warps of each streaming-engine CTA that take groups (the rest idle)
    int64_t acc_words; // 64-bit words of round sums and control words zeroed before each call
    uint8_t *packed;
    int64_t packed_bytes;
    __half *scale, *zero;
    float *s_out, *z_out;
    u64 *acc;       // [K][2] direct round sums, [K][2] difference array, then control words
    uint8_t *fk;    // [G] last round run by each group in the search kernel
    uint8_t *tile_maxf;  // [ntiles] largest f of each tile
    int *stale;     // [ntiles] tiles holding a group whose last round lies past the kept one
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

template <int NB>
struct Pack;  // codes per 32-bit output word
template <> struct Pack<4> { static constexpr int cpw = 8; };
template <> struct Pack<2> { static constexpr int cpw = 16; };
template <> struct Pack<3> { static constexpr int cpw = 10; };

// ------------------------------------------------------------------------------------------
// tile staging: the tile's groups as fp16 rows of `rs` halves in shared memory
// [HQQ 算法解读, "`axis` 不是一个无关紧要的开关"].  Each thread issues up to four 16-byte
// loads before storing them, to keep enough bytes in flight.
// ------------------------------------------------------------------------------------------
__device__ void stage_tile(const QParams &P, __half *wh, int64_t t0, int tg) {
    const int g = P.g, rs = P.stride;
    if (P.axis == 1) {
        const int ne = tg * g;
        const __half *src = P.W + t0 * (int64_t)g;  // 16-byte aligned: tiles hold 320k elements
        if ((g & 7) == 0) {  // 8-element vectors never cross a row
            const int nvec = ne >> 3;
            for (int v0 = threadIdx.x; v0 < nvec; v0 += 4 * kThreads) {
                uint4 x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = v0 + u * kThreads;
                    if (v < nvec) x[u] = __ldcs(reinterpret_cast<const uint4 *>(src) + v);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = v0 + u * kThreads;
                    if (v < nvec) {
                        const int e0 = v << 3, grp = e0 / g;
                        *reinterpret_cast<uint4 *>(wh + grp * rs + (e0 - grp * g)) = x[u];
                    }
                }
            }
        } else {
            for (int e = threadIdx.x; e < ne; e += kThreads) {
                const int grp = e / g;
                wh[grp * rs + (e - grp * g)] = src[e];
            }
        }
    } else {
        // group c of the tile is column t0 + c of the [g, G] view: elements j*G + t0 + c
        const int64_t G = P.G;
        if ((G & 7) == 0) {
            const int nv = (tg + 7) >> 3;  // tg % 8 == 0 except possibly at the end (G % 8 == 0)
            for (int v0 = threadIdx.x; v0 < g * nv; v0 += 4 * kThreads) {
                uint4 x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = v0 + u * kThreads;
                    if (v < g * nv) {
                        const int j = v / nv, cv = v - j * nv;
                        x[u] = __ldcs(reinterpret_cast<const uint4 *>(P.W + j * G + t0) + cv);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = v0 + u * kThreads;
                    if (v < g * nv) {
                        const int j = v / nv, cv = v - j * nv;
                        const __half *h = reinterpret_cast<const __half *>(&x[u]);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int col = cv * 8 + c;
                            if (col < tg) wh[col * rs + j] = h[c];
                        }
                    }
                }
            }
        } else {
            for (int v = threadIdx.x; v < g * tg; v += kThreads) {
                const int j = v / tg, col = v - j * tg;
                wh[col * rs + j] = P.W[j * G + t0 + col];
            }
        }
    }
}

// min-max init of every group of the tile [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"].
// Also keeps W*s of the group's min and max element: every element's W*s lies between them
// (rounding is monotonic), which bounds W*s + z without visiting the elements.
template <int NB>
__device__ void init_tile(const QParams &P, const __half *wh, float *s_t, float *z_t, float *lo_t,
                          float *hi_t, int tg) {
    constexpr float kQmax = (float)((1 << NB) - 1);
    const int g = P.g;
    for (int i = threadIdx.x; i < tg; i += kThreads) {
        const __half *row = wh + i * P.stride;
        float mn[4], mx[4];
        bool nan = false;
#pragma unroll
        for (int c = 0; c < 4; ++c) { mn[c] = INFINITY; mx[c] = -INFINITY; }
        int j = 0;
        for (; j + 4 <= g; j += 4) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = __half2float(row[j + c]);
                mn[c] = fminf(mn[c], v);
                mx[c] = fmaxf(mx[c], v);
                nan |= v != v;
            }
        }
        for (; j < g; ++j) {
            const float v = __half2float(row[j]);
            mn[0] = fminf(mn[0], v);
            mx[0] = fmaxf(mx[0], v);
            nan |= v != v;
        }
        const float lo_w = fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3]));
        const float hi_w = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        const float d = __fsub_rn(hi_w, lo_w);
        float s = (d < P.eps_tiny) ? 1.0f : __fdiv_rn(kQmax, d);
        s = fminf(s, P.scale_max);
        s_t[i] = s;
        z_t[i] = __fsub_rn(0.0f, __fmul_rn(lo_w, s));
        // a NaN in the group sends its warp down the clamped path (fmaxf(NaN, 0) = 0), so
        // table addresses stay in range whatever W holds
        lo_t[i] = nan ? __int_as_float(0x7fc00000) : __fmul_rn(lo_w, s);
        hi_t[i] = __fmul_rn(hi_w, s);
    }
}

// Code storage of a lane's 16 codes while the group iterates.  DIRECT: already in the packed
// format of the output (4 bit: two words of eight nibbles; 2 bit: one word), written straight
// to global memory when the group is done.  Otherwise one byte per code, left in the tile row
// and packed when the tile is written out.
template <int NB, bool DIRECT>
struct Codes {
    static constexpr int kWords = DIRECT ? (NB == 4 ? 2 : 1) : 4;
    static constexpr int kBits = DIRECT ? NB : 8;
    uint32_t w[kWords];
    __device__ __forceinline__ void put(int m, uint32_t bits) {
        // insert the low NB bits of `bits` at the code's position
        constexpr int per = 32 / kBits;
        uint32_t d;
        asm("bfi.b32 %0, %1, %2, %3, %4;" : "=r"(d)
            : "r"(bits), "r"(m % per == 0 ? 0u : w[m / per]), "r"(kBits * (m % per)), "r"(NB));
        w[m / per] = d;
    }
};

// One round over the 16 elements a lane holds: t = W*s + z, q = round(clip(t)), W_hat from
// the code table, |W - W_hat| and q - W*s (the zero-update term with e = 0); the codes are
// kept.  CLIP = false only when every t of the warp's groups rounds inside [0, 2^b - 1].
template <int NB, int NSEG, bool CLIP, bool FULL, bool DIRECT>
__device__ __forceinline__ void round_elems(const float (&w)[kE], const float (&ws)[kE], float z,
                                            uint32_t tab_adj, int nvalid, float (&absr)[kE],
                                            float (&term)[kE], Codes<NB, DIRECT> &codes) {
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    constexpr int kShift = NSEG == 32 ? 7 : NSEG == 16 ? 6 : NSEG == 8 ? 5 : NSEG == 4 ? 4 : 3;
#pragma unroll
    for (int m = 0; m < kE; ++m) {
        float t = __fadd_rn(ws[m], z);
        if (CLIP) t = fminf(fmaxf(t, 0.0f), kQmax);  // clip then round == round then clip
        const float u = __fadd_rn(t, kMagic);
        const float qf = __fsub_rn(u, kMagic);        // round half to even
        // u's bit pattern is 0x4B400000 + q: the table entry of code q sits at
        // tab_adj + (bits << kShift) (mod 2^32), tab_adj having absorbed the constant part
        const uint32_t bits = __float_as_uint(u);
        float what;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(what) : "r"(tab_adj + (bits << kShift)));
        codes.put(m, bits);
        const float ar = fabsf(__fsub_rn(w[m], what));
        const float tm = __fsub_rn(qf, ws[m]);        // q - (W - 0)*s
        if (FULL) {
            absr[m] = ar;
            term[m] = tm;
        } else {
            absr[m] = m < nvalid ? ar : 0.0f;
            term[m] = m < nvalid ? tm : 0.0f;
        }
    }
}

__device__ __forceinline__ void add_fixed(unsigned *row, u64 v) {
    // 64-bit fixed-point value into four 16-bit-chunk counters (exact; no counter overflows)
    atomicAdd(row, (unsigned)(v & 0xffffu));
    atomicAdd(row + 1, (unsigned)((v >> 16) & 0xffffu));
    atomicAdd(row + 2, (unsigned)((v >> 32) & 0xffffu));
    atomicAdd(row + 3, (unsigned)(v >> 48));
}

// metadata of one group [HQQ 算法解读, "量化公式"]: Delta = 1/s and z, rounded to fp16
__device__ __forceinline__ void write_meta(const QParams &P, int64_t k, float s, float z, int f) {
    P.scale[k] = __float2half_rn(__fdiv_rn(1.0f, s));
    P.zero[k] = __float2half_rn(z);
    if (P.s_out) P.s_out[k] = s;
    if (P.z_out) P.z_out[k] = z;
    if (f >= 0) {
        P.fk[k] = (uint8_t)f;
        if (P.group_rounds) P.group_rounds[k] = P.K > 0 ? (uint8_t)(f + 1) : 0;
    }
}

// ------------------------------------------------------------------------------------------
// the proximal loop [HQQ 算法解读, "第二拍：half-quadratic 迭代修正零点"]
//
// Each warp owns a contiguous slice of the tile's groups.  A segment of L lanes takes the
// slice's next group, keeps its 16-element runs in registers (binary32) and runs round after
// round until the group is done, then takes the next one, so lanes never idle while the
// slice has work left.  Segments of a warp may be at different rounds.
//   search (REPLAY = false): a group is done once frozen (z_{r+1} == z_r and no residual
//     above the last round's shrink threshold: every later round repeats round r exactly) or
//     after round K-1.  Round r's error is added to counters acc_w[r]; a group frozen at r
//     also adds it to acc_w[K + r + 1] (a difference array: it repeats in every later round).
//   fixup (REPLAY = true): a group makes exactly n = min(b, f) zero updates.
// The codes of a group's last round are its final codes (the final quantize with the
// original W and the kept zero, section "第二拍"): a done group writes them, with its
// metadata, straight to global memory (DIRECT) or leaves them in its tile row.
// ------------------------------------------------------------------------------------------
template <int NB, int L, bool REPLAY, bool FULL, bool DIRECT>
__device__ void run_groups(const QParams &P, __half *wh, const float *s_t, float *z_t,
                           const float *lo_t, const float *hi_t, uint8_t *f_t, float *tab,
                           unsigned *acc_w, const float *thr_s, const double *beta_s, int64_t t0,
                           int tg, int b_stop) {
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    constexpr int NSEG = 32 / L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sg = lane / L, l = lane - sg * L;
    const unsigned seg_mask = (L == 32) ? kFull : (((1u << L) - 1u) << (sg * L));
    const int K = P.K, rs = P.stride;
    const int nvalid = FULL ? kE : min(max(P.g - l * kE, 0), kE);
    const float g_f = (float)P.g, inv_g = 1.0f / (float)P.g;  // exact for FULL (g = 2^k)
    const float thr_last = K > 0 ? thr_s[K - 1] : 0.0f;
    const int gpw = (P.tile + kWarps - 1) / kWarps;
    const int g0 = warp * gpw;
    const int ng = max(0, min(gpw, tg - g0));
    const float lf = (float)l;  // code k = l + kk*L of the table, as an exact float
    // shared-space address of this segment's table column, minus the contribution of the
    // constant high bits of a rounded value (see round_elems); wraps modulo 2^32 on purpose
    constexpr int kShift = NSEG == 32 ? 7 : NSEG == 16 ? 6 : NSEG == 8 ? 5 : NSEG == 4 ? 4 : 3;
    const uint32_t tab_adj = (uint32_t)__cvta_generic_to_shared(tab + sg) - (0x4B400000u << kShift);

    // Every lane's state stays in range even with no group: the table address of round_elems
    // assumes W*s + z rounds inside [0, 2^b - 1] whenever the clip is skipped
    float w[kE], ws[kE];
#pragma unroll
    for (int m = 0; m < kE; ++m) { w[m] = 0.0f; ws[m] = 0.0f; }
    float s = 1.0f, z = 0.0f, lo = 0.0f, hi = 0.0f;
    int grp = -1, it = 0, nupd = 0, next = 0;
    bool exhausted = false;
    Codes<NB, DIRECT> codes;
#pragma unroll
    for (int i = 0; i < Codes<NB, DIRECT>::kWords; ++i) codes.w[i] = 0;
    while (true) {
        // ---- refill: segments without a group take the slice's next ones in lane order
        const bool need = grp < 0 && !exhausted;
        if (__any_sync(kFull, need)) {
            const unsigned nm = __ballot_sync(kFull, need && l == 0);
            int cand = next + __popc(nm & ((1u << lane) - 1u));
            cand = __shfl_sync(kFull, cand, sg * L);
            next += __popc(nm);
            if (need) {
                if (cand < ng) {
                    grp = g0 + cand;
                    const uint4 *src = reinterpret_cast<const uint4 *>(wh + grp * rs + l * kE);
                    const uint4 a = src[0], b = src[1];
                    const __half2 *ha = reinterpret_cast<const __half2 *>(&a);
                    const __half2 *hb = reinterpret_cast<const __half2 *>(&b);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 x = __half22float2(ha[i]), y = __half22float2(hb[i]);
                        w[2 * i] = x.x; w[2 * i + 1] = x.y; w[8 + 2 * i] = y.x; w[9 + 2 * i] = y.y;
                    }
                    s = s_t[grp];
                    z = z_t[grp];
                    lo = lo_t[grp];
                    hi = hi_t[grp];
#pragma unroll
                    for (int m = 0; m < kE; ++m) ws[m] = __fmul_rn(w[m], s);
                    if (!FULL) {  // slots past the group's end: W*s at the group's minimum
#pragma unroll
                        for (int m = 0; m < kE; ++m)
                            if (m >= nvalid) { w[m] = 0.0f; ws[m] = lo; }
                    }
                    it = 0;
                    if (REPLAY) nupd = min(b_stop, (int)f_t[grp]);
                } else {
                    exhausted = true;
                }
            }
        }
        const bool active = grp >= 0;
        if (!__any_sync(kFull, active)) break;

        const bool do_iter = active && (REPLAY ? (it < nupd) : (K > 0));
        bool done = active && !do_iter;
        if (__any_sync(kFull, do_iter)) {
            const int ri = min(it, max(K - 1, 0));
            // no clip is needed when [lo + z, hi + z] rounds inside [0, 2^b - 1]; lanes
            // without a group keep their last group's (or zero) state, so they are tested too
            const bool inside = __fadd_rn(lo, z) >= -0.5f && __fadd_rn(hi, z) < kQmax + 0.5f;
            const bool noclip = __all_sync(kFull, inside);
            // reconstructions W_hat = (k - z)/s for every code k: the IEEE division of the
            // method, done once per code value instead of once per element
            __syncwarp();
#pragma unroll
            for (int kk = 0; kk < (NQ + L - 1) / L; ++kk) {
                const int k = l + kk * L;
                if (k < NQ) tab[k * NSEG + sg] = __fdiv_rn(__fsub_rn(lf + (float)(kk * L), z), s);
            }
            __syncwarp();
            float absr[kE], term[kE];
            if (noclip) round_elems<NB, NSEG, false, FULL, DIRECT>(w, ws, z, tab_adj, nvalid, absr, term, codes);
            else round_elems<NB, NSEG, true, FULL, DIRECT>(w, ws, z, tab_adj, nvalid, absr, term, codes);
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
            const bool slow = (__ballot_sync(kFull, do_iter && maxr > thr_s[ri]) & seg_mask) != 0;
            if (__any_sync(kFull, slow)) {
                const double beta = beta_s[ri];
#pragma unroll
                for (int m = 0; m < kE; ++m) {
                    float t = __fadd_rn(ws[m], z);
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
            const bool big = (__ballot_sync(kFull, maxr > thr_last) & seg_mask) != 0;
            if (do_iter) {
                if (!REPLAY) {
                    const bool frozen = !slow && !big && (znew == z);
                    done = frozen || it == K - 1;
                    if (l == 0) {
                        const u64 fx = err_fixed(esum);
                        add_fixed(acc_w + 4 * it, fx);
                        if (done && it + 1 < K) add_fixed(acc_w + 4 * (K + it + 1), fx);
                    }
                    if (!done) {
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
        if (done) {
            if (REPLAY || K == 0) {
                // replay: the last round's codes were for z_{n-1}, the kept zero is z_n; no
                // round at all: codes for z0.  Either way quantize once more here.
#pragma unroll
                for (int m = 0; m < kE; ++m) {
                    const float t = fminf(fmaxf(__fadd_rn(ws[m], z), 0.0f), kQmax);
                    codes.put(m, __float_as_uint(__fadd_rn(t, kMagic)));
                }
            }
            const int64_t kg = t0 + grp;
            if (DIRECT) {
                if (nvalid > 0) {
                    const int64_t e = kg * P.g + l * kE;  // flat index of the lane's first code
                    if (NB == 4)
                        *reinterpret_cast<uint2 *>(P.packed + e / 2) = make_uint2(codes.w[0], codes.w[1]);
                    else
                        *reinterpret_cast<uint32_t *>(P.packed + e / 4) = codes.w[0];
                }
                if (l == 0) write_meta(P, kg, s, z, REPLAY ? -1 : it);
            } else {
                // the row's halves are dead (the group lives in registers): its bytes take the codes
                *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(wh + grp * rs) + l * kE) =
                    make_uint4(codes.w[0], codes.w[1 % Codes<NB, DIRECT>::kWords],
                               codes.w[2 % Codes<NB, DIRECT>::kWords],
                               codes.w[3 % Codes<NB, DIRECT>::kWords]);
                if (l == 0) {
                    z_t[grp] = z;
                    if (!REPLAY) f_t[grp] = (uint8_t)it;
                }
            }
            grp = -1;
        }
    }
}

// ------------------------------------------------------------------------------------------
// tile output when codes are not written directly: metadata [HQQ 算法解读, "量化公式"] and
// packed codes [HQQ 算法解读, "为什么一定要分组"] from the code bytes at the start of each row
// ------------------------------------------------------------------------------------------
template <int NB>
__device__ void write_tile(const QParams &P, const __half *wh, const float *s_t,
                           const float *z_t, const uint8_t *f_t, bool search, int64_t t0, int tg) {
    for (int i = threadIdx.x; i < tg; i += kThreads)
        write_meta(P, t0 + i, s_t[i], z_t[i], search ? (int)f_t[i] : -1);
    const int g = P.g;
    const int rowb = 2 * P.stride;  // bytes per tile row
    const uint8_t *cb = reinterpret_cast<const uint8_t *>(wh);
    if (P.codes_u8) {  // byte-per-code staging, packed afterwards by pack_codes_kernel
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
            for (int k = 0; k < CPW; ++k) {
                if (e0 + k < ne) {
                    word |= (uint32_t)cb[grp * rowb + j] << (NB * k);
                    if (++j == g) { j = 0; ++grp; }
                }
            }
            store_word(w0 + wi, word);
        }
    } else {
        // row j of the [g, G] view holds the tile's codes at flat j*G + t0 + col; here
        // G % CPW == 0 and t0 % CPW == 0, so each row segment starts on a word boundary
        const int nwr = (tg + CPW - 1) / CPW;
        for (int v = threadIdx.x; v < g * nwr; v += kThreads) {
            const int j = v / nwr, wr = v - j * nwr;
            uint32_t word = 0;
#pragma unroll
            for (int k = 0; k < CPW; ++k) {
                const int col = wr * CPW + k;
                if (col < tg) word |= (uint32_t)cb[col * rowb + j] << (NB * k);
            }
            store_word((j * P.G + t0) / CPW + wr, word);
        }
    }
}

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

template <int NB, int L>
struct Smem {
    __half *wh;
    float *s_t, *z_t, *lo_t, *hi_t, *tab, *thr;
    double *beta;
    uint8_t *f_t;
    unsigned *acc;    // all warps' counters
    unsigned *acc_w;  // this warp's counters
    __device__ Smem(unsigned char *base, const QParams &P) {
        const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
        wh = reinterpret_cast<__half *>(base + lay.wh);
        s_t = reinterpret_cast<float *>(base + lay.s_t);
        z_t = reinterpret_cast<float *>(base + lay.z_t);
        lo_t = reinterpret_cast<float *>(base + lay.lo_t);
        hi_t = reinterpret_cast<float *>(base + lay.hi_t);
        f_t = base + lay.f_t;
        tab = reinterpret_cast<float *>(base + lay.tab) + (threadIdx.x >> 5) * (1 << NB) * (32 / L);
        acc = reinterpret_cast<unsigned *>(base + lay.acc);
        acc_w = acc + (threadIdx.x >> 5) * 8 * (P.K > 0 ? P.K : 1);
        thr = reinterpret_cast<float *>(base + lay.thr);
        beta = reinterpret_cast<double *>(base + lay.beta);
    }
};

// workspace words after the per-round sums: tiles finished, kept round, rounds measured,
// number of stale tiles; then the per-tile largest f and the list of stale tiles
struct Ctl {
    unsigned done;      // tiles (or warps, streaming engine) finished
    int b;              // kept round
    int run;            // rounds whose MAE was computed
    int nstale;         // stale tiles (tile engine)
    unsigned long long work;  // next group to hand out (streaming engine)
    unsigned long long pad;
};

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

template <int NB, int L>
__device__ void load_constants(const QParams &P, Smem<NB, L> &S) {
    for (int i = threadIdx.x; i < P.K; i += kThreads) {
        S.thr[i] = P.thr[i];
        S.beta[i] = P.beta[i];
    }
}

template <int NB, int L, bool FULL, bool DIRECT>
__global__ void __launch_bounds__(kThreads, 2) hqq_search_kernel(const __grid_constant__ QParams P) {
    extern __shared__ __align__(16) unsigned char smem[];
    Smem<NB, L> S(smem, P);
    __shared__ bool last;
    __shared__ int maxf;
    const int K = P.K;
    const int64_t t0 = (int64_t)blockIdx.x * P.tile;
    const int tg = (int)min((int64_t)P.tile, P.G - t0);
    for (int i = threadIdx.x; i < kWarps * 8 * K; i += kThreads) S.acc[i] = 0;
    if (threadIdx.x == 0) maxf = 0;
    load_constants(P, S);
    stage_tile(P, S.wh, t0, tg);
    __syncthreads();
    init_tile<NB>(P, S.wh, S.s_t, S.z_t, S.lo_t, S.hi_t, tg);
    __syncthreads();
    run_groups<NB, L, false, FULL, DIRECT>(P, S.wh, S.s_t, S.z_t, S.lo_t, S.hi_t, S.f_t, S.tab,
                                           S.acc_w, S.thr, S.beta, t0, tg, 0);
    __syncthreads();
    if (!DIRECT) write_tile<NB>(P, S.wh, S.s_t, S.z_t, S.f_t, true, t0, tg);
    // the largest f of the tile (for the fixup's staleness test)
    int mf = 0;
    for (int i = threadIdx.x; i < tg; i += kThreads) mf = max(mf, DIRECT ? (int)__ldcg(P.fk + t0 + i) : (int)S.f_t[i]);
    atomicMax(&maxf, mf);
    // the global round sums were zeroed by the kernel launched before this one
    wait_prerequisite();
    allow_dependents();
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
    __syncthreads();
    if (threadIdx.x == 0) P.tile_maxf[blockIdx.x] = (uint8_t)maxf;
    // the last tile to finish applies the stop rule once for the whole tensor and lists the
    // tiles that hold a group whose own last round lies past the kept round
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&ctl_of(P)->done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (last) {
        __threadfence();
        if (threadIdx.x == 0) stop_rule(P);
        __syncthreads();
        Ctl *c = ctl_of(P);
        const int b = *(volatile int *)&c->b;
        for (int t = threadIdx.x; t < (int)gridDim.x; t += kThreads)
            if ((int)__ldcg(P.tile_maxf + t) > b) P.stale[atomicAdd(&c->nstale, 1)] = t;
    }
}

// Recomputes the stale tiles listed by the search kernel.
template <int NB, int L, bool FULL, bool DIRECT>
__global__ void __launch_bounds__(kThreads, 2) hqq_fixup_kernel(const __grid_constant__ QParams P) {
    extern __shared__ __align__(16) unsigned char smem[];
    wait_prerequisite();  // the search kernel has finished and listed the stale tiles
    allow_dependents();
    Ctl *c = ctl_of(P);
    const int nstale = __ldcg(&c->nstale);
    if ((int)blockIdx.x >= nstale) return;
    Smem<NB, L> S(smem, P);
    const int b = __ldcg(&c->b);
    load_constants(P, S);
    for (int si = blockIdx.x; si < nstale; si += gridDim.x) {
        const int64_t t0 = (int64_t)__ldcg(P.stale + si) * P.tile;
        const int tg = (int)min((int64_t)P.tile, P.G - t0);
        for (int i = threadIdx.x; i < tg; i += kThreads) S.f_t[i] = __ldcg(P.fk + t0 + i);
        stage_tile(P, S.wh, t0, tg);
        __syncthreads();
        init_tile<NB>(P, S.wh, S.s_t, S.z_t, S.lo_t, S.hi_t, tg);
        __syncthreads();
        run_groups<NB, L, true, FULL, DIRECT>(P, S.wh, S.s_t, S.z_t, S.lo_t, S.hi_t, S.f_t, S.tab,
                                              nullptr, S.thr, S.beta, t0, tg, b);
        __syncthreads();
        if (!DIRECT) write_tile<NB>(P, S.wh, S.s_t, S.z_t, S.f_t, false, t0, tg);
        __syncthreads();
    }
}

// ==========================================================================================
// Streaming engine (axis 1; 2- or 4-bit codes; power-of-two groups of 16 .. 128 elements that
// fill whole 32-bit words of the output): one lane per group
//
// Each lane holds one whole group: its fp16 row in registers (P/2 words), its own table of the
// 2^b reconstructions in a private shared-memory column, and its running state.  Lanes take
// groups from a global counter (one atomic per warp and refill), so the work stays balanced
// to the end, and each lane copies its next group's row into a shared-memory slot with
// cp.async one group ahead.
//
// The arithmetic runs on packed binary32 pairs (add/mul/fma.rn.f32x2: two IEEE operations per
// instruction, each rounded exactly as its scalar form).  A register word pairs element j with
// element j + 8 of the same 16-element block, so the two halves of every pair fall in two
// consecutive 8-element chunks.  The pairwise tree of each chunk then runs on both chunks at
// once, and the group sums keep the oracle's order: an 8-element tree per chunk, then
// recursive halving over the chunks.
// ==========================================================================================
template <int P>
struct SRow {
    uint32_t h[P / 2];  // word 8c + m: element 16c + m (low half) and 16c + 8 + m (high half)
};

__device__ __forceinline__ float half_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xffffu))); }
__device__ __forceinline__ float half_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

// element j of a row held in the paired layout
template <int P>
__device__ __forceinline__ float row_elem(const SRow<P> &row, int j) {
    const uint32_t w = row.h[(j >> 4) * 8 + (j & 7)];
    return (j & 8) ? half_hi(w) : half_lo(w);
}

// one 16-element block from its natural fp16 words n[i] = (x[2i], x[2i+1]) to the paired layout
__device__ __forceinline__ void pair_block(uint32_t *dst, uint32_t n0, uint32_t n1, uint32_t n2,
                                           uint32_t n3, uint32_t n4, uint32_t n5, uint32_t n6,
                                           uint32_t n7) {
    const uint32_t lo[4] = {n0, n1, n2, n3}, hi[4] = {n4, n5, n6, n7};
#pragma unroll
    for (int m = 0; m < 8; ++m) dst[m] = __byte_perm(lo[m >> 1], hi[m >> 1], (m & 1) ? 0x7632 : 0x5410);
}

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
#pragma unroll
        for (int k = 0; k < NQ; ++k) sts_f32(col + 128u * k, __fdiv_rn(__fsub_rn((float)k, z), s));
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

template <int NB, int P, bool DIRECT>
struct SCodes {  // a lane's codes of the current round, in the output's packed format
    static constexpr int kWords = DIRECT ? P * NB / 32 : 1;
    uint32_t w[kWords];
    __device__ __forceinline__ void put(int j, uint32_t bits) {  // code j: low NB bits of bits
        constexpr int CPW = 32 / NB;
        uint32_t d;
        asm("bfi.b32 %0, %1, %2, %3, %4;" : "=r"(d)
            : "r"(bits), "r"(j % CPW == 0 ? 0u : w[j / CPW]), "r"(NB * (j % CPW)), "r"(NB));
        w[j / CPW] = d;
    }
};

// One proximal round over a lane's group [HQQ 算法解读, "第二拍"] with e = 0 for every element.
// Returns the group's error sum, the zero-update sum (z_new times g) and (DIRECT) the round's
// codes.  CLIP: clamp W s + z to [0, 2^b - 1] before rounding.
template <int NB, int P, bool CLIP, bool DIRECT>
__device__ __forceinline__ void stream_round(const SRow<P> &row, float s, float z,
                                             uint32_t tab_adj, float &esum, float &zsum,
                                             SCodes<NB, P, DIRECT> &codes) {
    constexpr int NCH = P / 8;
    constexpr int LOGN = NCH == 2 ? 1 : NCH == 4 ? 2 : NCH == 8 ? 3 : 4;
    constexpr float kQmax = (float)((1 << NB) - 1);
    const float2 s2 = make_float2(s, s), z2 = make_float2(z, z);
    const float2 mg2 = make_float2(kMagic, kMagic), nmg2 = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    float sa[LOGN + 1], st[LOGN + 1];
#pragma unroll
    for (int c = 0; c < P / 16; ++c) {
        float2 d[8], tm[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float2 w = __half22float2(*reinterpret_cast<const __half2 *>(&row.h[8 * c + m]));
            const float2 ws = __fmul2_rn(w, s2);
            float2 t = __fadd2_rn(ws, z2);
            if (CLIP) {
                t.x = fminf(fmaxf(t.x, 0.0f), kQmax);
                t.y = fminf(fmaxf(t.y, 0.0f), kQmax);
            }
            const float2 u = __fadd2_rn(t, mg2);     // round half to even: the integer in the
            const float2 qf = __fadd2_rn(u, nmg2);   // low mantissa bits of u
            const uint32_t ba = __float_as_uint(u.x), bb = __float_as_uint(u.y);
            const float2 what = make_float2(lds_f32(tab_adj + (ba << 7)), lds_f32(tab_adj + (bb << 7)));
            if (DIRECT) {
                codes.put(16 * c + m, ba);
                codes.put(16 * c + 8 + m, bb);
            }
            d[m] = __ffma2_rn(what, neg1, w);   // W - W_hat
            tm[m] = __ffma2_rn(ws, neg1, qf);   // q - (W - 0) s
        }
        const float2 ea = abs_tree8x2(d), ta = tree8x2(tm);
        pw_push<LOGN>(sa, 2 * c, ea.x);
        pw_push<LOGN>(sa, 2 * c + 1, ea.y);
        pw_push<LOGN>(st, 2 * c, ta.x);
        pw_push<LOGN>(st, 2 * c + 1, ta.y);
    }
    esum = sa[LOGN];
    zsum = st[LOGN];
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

// final codes of a lane's group with the kept zero, written to the packed output
// [HQQ 算法解读, "第二拍" and "为什么一定要分组"].  The group covers whole 32-bit words of the
// output, stored as they are.
template <int NB, int P>
__device__ __forceinline__ void group_store_codes(const QParams &Pm, const SRow<P> &row,
                                                  int64_t grp, float s, float z) {
    constexpr int CPW = 32 / NB;  // NB in {2, 4}; g = P and P*NB % 32 == 0
    constexpr float kQmax = (float)((1 << NB) - 1);
    uint32_t *dst = reinterpret_cast<uint32_t *>(Pm.packed) + grp * (P / CPW);
#pragma unroll
    for (int wi = 0; wi < P / CPW; ++wi) {
        uint32_t word = 0;
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
            const float w = row_elem<P>(row, wi * CPW + c);
            const float t = fminf(fmaxf(__fadd_rn(__fmul_rn(w, s), z), 0.0f), kQmax);
            word |= (__float_as_uint(__fadd_rn(t, kMagic)) & ((1u << NB) - 1u)) << (NB * c);
        }
        dst[wi] = word;
    }
}

// the group's metadata [HQQ 算法解读, "量化公式"]: Delta = 1/s (y = RN(1/s)) and z in fp16
__device__ __forceinline__ void stream_meta(const QParams &Pm, int64_t k, float s, float y,
                                            float z, int f) {
    Pm.scale[k] = __float2half_rn(y);
    Pm.zero[k] = __float2half_rn(z);
    if (Pm.s_out) Pm.s_out[k] = s;
    if (Pm.z_out) Pm.z_out[k] = z;
    if (f >= 0) {
        Pm.fk[k] = (uint8_t)f;
        if (Pm.group_rounds) Pm.group_rounds[k] = Pm.K > 0 ? (uint8_t)(f + 1) : 0;
    }
}

// per-group state of the streaming engine
struct SGroup {
    float s, y, z, lo, hi, A;  // scale, RN(1/s), zero, min*s, max*s, max(|lo|, |hi|)
    __device__ __forceinline__ void idle() { s = 1.0f; y = 1.0f; z = 0.0f; lo = 0.0f; hi = 0.0f; A = 0.0f; }
};

template <int NB, int P>
__device__ __forceinline__ void group_init(const SRow<P> &row, float eps, float smax, SGroup &gs) {
    constexpr float kQmax = (float)((1 << NB) - 1);
    // min and max in fp16 pairs (exact).  A NaN propagates into lo and hi, which sends the
    // warp down the clamped path (fmaxf(NaN, 0) = 0): table addresses stay in range whatever
    // W holds
    __half2 mn2 = *reinterpret_cast<const __half2 *>(&row.h[0]), mx2 = mn2;
#pragma unroll
    for (int i = 1; i < P / 2; ++i) {
        const __half2 v = *reinterpret_cast<const __half2 *>(&row.h[i]);
        mn2 = __hmin2_nan(mn2, v);
        mx2 = __hmax2_nan(mx2, v);
    }
    const float mn = fminf(__low2float(mn2), __high2float(mn2));
    const float mx = fmaxf(__low2float(mx2), __high2float(mx2));
    // [HQQ 算法解读, "第一拍：min-max 给一个可用的初值"]
    const float d = __fsub_rn(mx, mn);
    float s = (d < eps) ? 1.0f : __fdiv_rn(kQmax, d);
    s = fminf(s, smax);
    gs.s = s;
    gs.y = __frcp_rn(s);
    gs.z = __fsub_rn(0.0f, __fmul_rn(mn, s));
    gs.lo = __fmul_rn(mn, s);
    gs.hi = __fmul_rn(mx, s);
    gs.A = fmaxf(fabsf(gs.lo), fabsf(gs.hi));
}

// the row of a group into registers, in the paired layout.  From the lane's shared-memory
// slot, where 16-byte chunk v sits at position v ^ sw (the swizzle spreads the lanes of a
// quarter warp over all banks), or (sw < 0) straight from global memory.
template <int P>
__device__ __forceinline__ void load_row(SRow<P> &row, const __half *src_row, int sw) {
    const uint4 *src = reinterpret_cast<const uint4 *>(src_row);
#pragma unroll
    for (int c = 0; c < P / 16; ++c) {
        const uint4 a = src[sw < 0 ? 2 * c : (2 * c) ^ sw];
        const uint4 b = src[sw < 0 ? 2 * c + 1 : (2 * c + 1) ^ sw];
        pair_block(&row.h[8 * c], a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w);
    }
}

// the row of group `grp` (2P bytes, 16-byte aligned) into the lane's slot, asynchronously
template <int P>
__device__ __forceinline__ void prefetch_row(__half *slot, const __half *W, int64_t grp, int sw) {
    const char *src = reinterpret_cast<const char *>(W + grp * P);
    const uint32_t dst = (uint32_t)__cvta_generic_to_shared(slot);
#pragma unroll
    for (int v = 0; v < P / 8; ++v)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * (v ^ sw)), "l"(src + 16 * v));
    asm volatile("cp.async.commit_group;" ::);
}

__device__ __forceinline__ void prefetch_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// the slot swizzle of a lane: the P/8 chunks of lanes l .. l+7 (one quarter warp of 16-byte
// accesses) must land in 8 different 16-byte bank groups
template <int P>
__device__ __forceinline__ int slot_swizzle(int lane) {
    constexpr int C = P / 8;  // chunks per slot: 2, 4, 8 or 16
    return C >= 8 ? (lane & 7) : C == 4 ? ((lane >> 1) & 3) : ((lane >> 2) & 1);
}

struct StreamSmem {
    static __host__ __device__ int bytes(int P, int nq, int K) {
        const int Kc = K > 0 ? K : 1;
        return kWarps * (nq * 32 * 4)                 // tables: [NQ][32] floats per warp
               + kWarps * 2 * Kc * 4 * 4              // per-warp round counters
               + kWarps * 32 * P * 2                  // prefetch slots: one row per lane
               + ((Kc * 4 + 15) / 16 * 16) + Kc * 8;  // thresholds and betas
    }
};

// claim one group per requesting lane from the global counter (one atomic per warp)
__device__ __forceinline__ int64_t claim(const QParams &Pm, bool want) {
    const unsigned lane = threadIdx.x & 31;
    const unsigned m = __ballot_sync(kFull, want);
    unsigned long long base = 0;
    if (lane == 0 && m) base = atomicAdd(&ctl_of(Pm)->work, (unsigned long long)__popc(m));
    base = __shfl_sync(kFull, base, 0);
    const int64_t id = (int64_t)base + __popc(m & ((1u << lane) - 1u));
    return (want && id < Pm.G) ? id : -1;
}

// position of the k-th (from 0) set bit of mask, or -1
__device__ __forceinline__ int nth_set_bit(unsigned mask, int k) {
    for (int i = 0; i < k; ++i) mask &= mask - 1u;
    return __ffs(mask) - 1;
}

// ------------------------------------------------------------------------------------------
// Tail of the streaming engine.  Once the global counter is exhausted, a warp whose lanes are
// mostly idle would spend full rounds on its last few groups, and these few long chains set
// the kernel's end.  The warp then re-splits its remaining groups over L lanes each (2 to
// 16): lane l of a segment holds elements [l E, (l+1) E) of the group (E = P/L, whole 32-bit
// words of codes), builds every L-th table entry, and the segment adds its partial sums with
// xor shuffles.  Each lane's chunks are summed by recursive halving and the shuffle levels
// continue the halving across lanes, so the group sums keep the oracle's order.  As groups
// finish, the warp splits again into wider segments.
// The split costs about twice the instructions per group-round, so it only pays once the
// warp is nearly empty: at most kTailLanes groups left (4096^2 4-bit g64: 103.7 -> 97.8 us
// with 4; a threshold of 16 was slower than no split at all).
// ------------------------------------------------------------------------------------------
constexpr int kTailLanes = 4;

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

// the widest split of a group: every lane keeps at least one 8-element chunk and whole
// 32-bit words of codes (1: no split)
template <int NB, int P>
struct TailMax {
    static constexpr int a = NB * P / 32, b = P / 8;
    static constexpr int value = (a < b ? a : b) > 16 ? 16 : (a < b ? a : b);
};

struct TailState {  // a segment's group, replicated in all of its lanes
    int64_t cur;
    SGroup gs;
    int it;
    bool act;
};

// One proximal round over a lane's E consecutive elements of its group (natural fp16 pairs),
// with e = 0: returns the lane's pairwise partial sums and its code words.
template <int NB, int E, bool CLIP>
__device__ __forceinline__ void tail_round(const uint32_t (&h)[E / 2], float s, float z,
                                           uint32_t tab_adj, float &esum, float &zsum,
                                           uint32_t (&cw)[E * NB / 32]) {
    constexpr int NCH = E / 8;
    constexpr int LOGN = NCH == 1 ? 0 : NCH == 2 ? 1 : NCH == 4 ? 2 : NCH == 8 ? 3 : 4;
    constexpr int CPW = 32 / NB;
    constexpr float kQmax = (float)((1 << NB) - 1);
    float sa[LOGN + 1], st[LOGN + 1];
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        float ar[8], tm[8];
#pragma unroll
        for (int m2 = 0; m2 < 8; m2 += 2) {
            const float2 wp = __half22float2(*reinterpret_cast<const __half2 *>(&h[(8 * ch + m2) / 2]));
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int m = m2 + hh, j = 8 * ch + m;
                const float w = hh ? wp.y : wp.x;
                const float ws = __fmul_rn(w, s);
                float t = __fadd_rn(ws, z);
                if (CLIP) t = fminf(fmaxf(t, 0.0f), kQmax);
                const float u = __fadd_rn(t, kMagic);
                const float qf = __fsub_rn(u, kMagic);
                const uint32_t bits = __float_as_uint(u);
                const float what = lds_f32(tab_adj + (bits << 7));
                uint32_t d;
                asm("bfi.b32 %0, %1, %2, %3, %4;" : "=r"(d)
                    : "r"(bits), "r"(j % CPW == 0 ? 0u : cw[j / CPW]), "r"(NB * (j % CPW)), "r"(NB));
                cw[j / CPW] = d;
                ar[m] = fabsf(__fsub_rn(w, what));
                tm[m] = __fsub_rn(qf, ws);  // q - (W - 0) s
            }
        }
        pw_push<LOGN>(sa, ch, tree8(ar));
        pw_push<LOGN>(st, ch, tree8(tm));
    }
    esum = sa[LOGN];
    zsum = st[LOGN];
}

// Runs the warp's groups in segments of L lanes until they are all done, or until few enough
// remain for a split into segments of 2L lanes (owners then marks the lanes holding them).
// owners on entry: the lanes whose ts holds a group; segment i takes the i-th of them.
template <int NB, int P, int L>
__device__ void tail_epoch(const QParams &Pm, TailState &ts, unsigned &owners, float *tabw,
                           unsigned *acc_w, const float *thr_s, const double *beta_s,
                           float thr_last) {
    constexpr int E = P / L, CW = E * NB / 32, NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    const int K = Pm.K;
    const int lane = threadIdx.x & 31, seg = lane / L, l = lane % L;
    const int n = __popc(owners);
    const int pos = seg < n ? nth_set_bit(owners, seg) : -1;
    const int src = pos >= 0 ? pos : lane;
    TailState me;
    me.cur = __shfl_sync(kFull, ts.cur, src);
    me.gs.s = __shfl_sync(kFull, ts.gs.s, src);
    me.gs.y = __shfl_sync(kFull, ts.gs.y, src);
    me.gs.z = __shfl_sync(kFull, ts.gs.z, src);
    me.gs.lo = __shfl_sync(kFull, ts.gs.lo, src);
    me.gs.hi = __shfl_sync(kFull, ts.gs.hi, src);
    me.gs.A = __shfl_sync(kFull, ts.gs.A, src);
    me.it = __shfl_sync(kFull, ts.it, src);
    me.act = pos >= 0;
    uint32_t h[E / 2];
    if (me.act) {  // this lane's slice of the row (in L2: the row was read a moment ago)
        const uint4 *src_row = reinterpret_cast<const uint4 *>(Pm.W + me.cur * P + l * E);
#pragma unroll
        for (int v = 0; v < E / 8; ++v) {
            const uint4 x = src_row[v];
            h[4 * v] = x.x; h[4 * v + 1] = x.y; h[4 * v + 2] = x.z; h[4 * v + 3] = x.w;
        }
    } else {  // a segment without a group: zero row, zero state (inside every range)
#pragma unroll
        for (int i = 0; i < E / 2; ++i) h[i] = 0;
        me.gs.idle();
        me.it = 0;
    }
    // every lane looks up in its own column; lane l of a segment computes entries k = l, l + L,
    // ... and writes each into all L columns of the segment (rotated, so the lanes of a
    // segment store to L different banks at a time)
    const uint32_t col = (uint32_t)__cvta_generic_to_shared(tabw + lane);
    const uint32_t col0 = col - 4u * l;
    const uint32_t tab_adj = col - (0x4B400000u << 7);
    uint32_t cw[CW];
#pragma unroll
    for (int i = 0; i < CW; ++i) cw[i] = 0;
    while (true) {
        const int ri = min(me.it, K - 1);
        __syncwarp();
#pragma unroll
        for (int kk = 0; kk < (NQ + L - 1) / L; ++kk) {
            const int k = l + kk * L;
            if (k < NQ) {
                const float v = table_entry((float)k, me.gs.s, me.gs.y, me.gs.z);
#pragma unroll
                for (int i = 0; i < L; ++i) sts_f32(col0 + 4u * ((l + i) & (L - 1)) + 128u * k, v);
            }
        }
        __syncwarp();
        const float lz = __fadd_rn(me.gs.lo, me.gs.z), hz = __fadd_rn(me.gs.hi, me.gs.z);
        const bool inside = lz >= -0.5f && hz < kQmax + 0.5f;
        float esum, zsum;
        if (__all_sync(kFull, inside))
            tail_round<NB, E, false>(h, me.gs.s, me.gs.z, tab_adj, esum, zsum, cw);
        else
            tail_round<NB, E, true>(h, me.gs.s, me.gs.z, tab_adj, esum, zsum, cw);
#pragma unroll
        for (int off = 1; off < L; off <<= 1) {
            esum = __fadd_rn(esum, __shfl_xor_sync(kFull, esum, off));
            zsum = __fadd_rn(zsum, __shfl_xor_sync(kFull, zsum, off));
        }
        const float B = resid_bound(lz, hz, me.gs.A, me.gs.z, me.gs.y, kQmax);
        const bool slow = me.act && B > thr_s[ri];
        if (slow) zsum = group_zsum_shrink<NB>(Pm.W + me.cur * P, P, P, me.gs.s, me.gs.z, tab_adj, beta_s[ri], Pm.p);
        const float znew = __fmul_rn(zsum, 1.0f / (float)P);
        if (me.act) {
            const bool done = (!slow && !(B > thr_last) && znew == me.gs.z) || me.it == K - 1;
            if (l == 0) {
                const u64 fx = err_fixed(esum);
                add_fixed(acc_w + 4 * me.it, fx);
                if (done && me.it + 1 < K) add_fixed(acc_w + 4 * (K + me.it + 1), fx);
            }
            if (done) {
                uint32_t *dst = reinterpret_cast<uint32_t *>(Pm.packed) + me.cur * (P * NB / 32) + l * CW;
#pragma unroll
                for (int i = 0; i < CW; ++i) dst[i] = cw[i];
                if (l == 0) stream_meta(Pm, me.cur, me.gs.s, me.gs.y, me.gs.z, me.it);
                me.act = false;  // keeps its consistent row and state
            } else {
                me.gs.z = znew;
                ++me.it;
            }
        }
        const unsigned lead = __ballot_sync(kFull, l == 0 && me.act);
        if (lead == 0 || (2 * L <= TailMax<NB, P>::value && __popc(lead) * 2 * L <= 32)) {
            owners = lead;
            ts = me;
            return;
        }
    }
}

// the rest of the warp's groups: owners marks the lanes whose (cur, gs, it) hold one
template <int NB, int P>
__device__ __noinline__ void tail_run(const QParams &Pm, unsigned owners, int64_t cur, const SGroup &gs,
                         int it, float *tabw, unsigned *acc_w, const float *thr_s,
                         const double *beta_s, float thr_last) {
    constexpr int LM = TailMax<NB, P>::value;
    static_assert(LM >= 2, "no tail split for this group shape");
    TailState ts;
    ts.cur = cur;
    ts.gs = gs;
    ts.it = it;
    ts.act = true;
    while (owners) {
        const int n = __popc(owners);
        int L = 32;
        while (L > 1 && n * L > 32) L >>= 1;
        if (L > LM) L = LM;
        if (L >= 16 && LM >= 16) tail_epoch<NB, P, (LM >= 16 ? 16 : 2)>(Pm, ts, owners, tabw, acc_w, thr_s, beta_s, thr_last);
        else if (L >= 8 && LM >= 8) tail_epoch<NB, P, (LM >= 8 ? 8 : 2)>(Pm, ts, owners, tabw, acc_w, thr_s, beta_s, thr_last);
        else if (L >= 4 && LM >= 4) tail_epoch<NB, P, (LM >= 4 ? 4 : 2)>(Pm, ts, owners, tabw, acc_w, thr_s, beta_s, thr_last);
        else tail_epoch<NB, P, 2>(Pm, ts, owners, tabw, acc_w, thr_s, beta_s, thr_last);
    }
}

template <int NB, int P>
__global__ void __launch_bounds__(kThreads, P <= 64 ? 2 : 1) hqq_stream_kernel(const __grid_constant__ QParams Pm) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K = Pm.K;
    const int Kc = K > 0 ? K : 1;
    float *tabw = reinterpret_cast<float *>(smem) + warp * NQ * 32;
    unsigned *acc = reinterpret_cast<unsigned *>(smem + kWarps * NQ * 32 * 4);
    unsigned *acc_w = acc + warp * 8 * Kc;
    __half *slot = reinterpret_cast<__half *>(smem + kWarps * NQ * 32 * 4 + kWarps * 8 * Kc * 4) +
                   (warp * 32 + lane) * P;
    float *thr_s = reinterpret_cast<float *>(smem + kWarps * NQ * 32 * 4 + kWarps * 8 * Kc * 4 +
                                             kWarps * 32 * P * 2);
    double *beta_s = reinterpret_cast<double *>(reinterpret_cast<unsigned char *>(thr_s) +
                                                (Kc * 4 + 15) / 16 * 16);
    __shared__ bool last;
    for (int i = threadIdx.x; i < kWarps * 8 * Kc; i += kThreads) acc[i] = 0;
    for (int i = threadIdx.x; i < K; i += kThreads) { thr_s[i] = Pm.thr[i]; beta_s[i] = Pm.beta[i]; }
    __syncthreads();
    const float thr_last = K > 0 ? thr_s[K - 1] : 0.0f;
    constexpr float kInvG = 1.0f / (float)P;  // g = P = 2^k: z = zsum * (1/g) exactly
    const uint32_t col = (uint32_t)__cvta_generic_to_shared(tabw + lane);
    const uint32_t tab_adj = col - (0x4B400000u << 7);
    const int sw = slot_swizzle<P>(lane);

    SRow<P> row;
#pragma unroll
    for (int i = 0; i < P / 2; ++i) row.h[i] = 0;
    SCodes<NB, P, true> codes;
#pragma unroll
    for (int i = 0; i < SCodes<NB, P, true>::kWords; ++i) codes.w[i] = 0;
    SGroup gs;
    gs.idle();
    int it = 0;
    int64_t cur = -1;
    // the round sums and the group counter were zeroed by the kernel launched before this one
    wait_prerequisite();
    // a small tensor is spread thin: only the first stream_warps warps of each CTA take groups,
    // so its few groups run on many SMs rather than crowding a few
    int64_t nxt = warp < Pm.stream_warps ? claim(Pm, true) : -1;
    if (nxt >= 0) prefetch_row<P>(slot, Pm.W, nxt, sw);
    while (true) {
        // ---- a lane without a group takes the prefetched one and prefetches another
        const bool need = cur < 0 && nxt >= 0;
        if (__any_sync(kFull, need)) {
            if (need) {
                prefetch_wait();
                cur = nxt;
                load_row<P>(row, slot, sw);
                group_init<NB, P>(row, Pm.eps_tiny, Pm.scale_max, gs);
                it = 0;
            }
            const int64_t n2 = claim(Pm, need);
            if (need) {
                nxt = n2;
                if (nxt >= 0) prefetch_row<P>(slot, Pm.W, nxt, sw);
            }
        }
        // Once nothing is left to claim (a lane whose claim failed holds no group), the k-th
        // idle lane takes the queued group of the k-th lane that holds one it has not started;
        // the row is already in that lane's slot.
        {
            const unsigned idle_m = __ballot_sync(kFull, cur < 0 && nxt < 0);
            const unsigned donor_m = __ballot_sync(kFull, cur >= 0 && nxt >= 0);
            if (idle_m != 0u && donor_m != 0u) {
                const bool is_donor = (donor_m >> lane) & 1u, is_idle = (idle_m >> lane) & 1u;
                if (is_donor) prefetch_wait();
                __syncwarp();
                const unsigned below = (1u << lane) - 1u;
                const int npair = min(__popc(idle_m), __popc(donor_m));
                const int ri = __popc(idle_m & below), rd = __popc(donor_m & below);
                const bool takes = is_idle && ri < npair;
                const int src = takes ? nth_set_bit(donor_m, ri) : lane;
                const int64_t dn = __shfl_sync(kFull, nxt, src);
                if (takes) {
                    cur = dn;
                    load_row<P>(row, slot + (src - lane) * P, slot_swizzle<P>(src));
                    group_init<NB, P>(row, Pm.eps_tiny, Pm.scale_max, gs);
                    it = 0;
                }
                if (is_donor && rd < npair) nxt = -1;
                __syncwarp();
            }
        }
        const bool active = cur >= 0;
        if (!__any_sync(kFull, active)) break;
        if constexpr (TailMax<NB, P>::value >= 2) {
            // nothing left to claim and at most kTailLanes groups left in the warp: split them
            if (K > 0 && __all_sync(kFull, nxt < 0)) {
                const unsigned owners = __ballot_sync(kFull, active);
                if (__popc(owners) <= kTailLanes) {
                    tail_run<NB, P>(Pm, owners, cur, gs, it, tabw, acc_w, thr_s, beta_s, thr_last);
                    break;
                }
            }
        }
        bool done = active && K == 0;
        if (__any_sync(kFull, active && K > 0)) {
            const int ri = min(it, max(K - 1, 0));
            build_table<NQ>(col, gs.s, gs.y, gs.z);
            // no clip is needed when [lo + z, hi + z] rounds inside [0, 2^b - 1]; a lane without
            // a group holds a zero row and zero state, or its last group's row and state
            const float lz = __fadd_rn(gs.lo, gs.z), hz = __fadd_rn(gs.hi, gs.z);
            const bool inside = lz >= -0.5f && hz < kQmax + 0.5f;
            float esum, zsum;
            if (__all_sync(kFull, inside))
                stream_round<NB, P, false, true>(row, gs.s, gs.z, tab_adj, esum, zsum, codes);
            else
                stream_round<NB, P, true, true>(row, gs.s, gs.z, tab_adj, esum, zsum, codes);
            // lp shrink: a residual that may exceed the round's safe threshold -> exact binary64
            const float B = resid_bound(lz, hz, gs.A, gs.z, gs.y, kQmax);
            const bool slow = active && B > thr_s[ri];
            if (slow) zsum = group_zsum_shrink<NB>(Pm.W + cur * P, P, P, gs.s, gs.z, tab_adj, beta_s[ri], Pm.p);
            const float znew = __fmul_rn(zsum, kInvG);
            if (active && K > 0) {
                done = (!slow && !(B > thr_last) && znew == gs.z) || it == K - 1;
                const u64 fx = err_fixed(esum);
                add_fixed(acc_w + 4 * it, fx);
                if (done && it + 1 < K) add_fixed(acc_w + 4 * (K + it + 1), fx);
                if (!done) {
                    gs.z = znew;
                    ++it;
                }
            }
        }
        if (done) {
            // the codes of a group's last round are its final codes (z is the kept zero);
            // with no round at all they are computed here
            if (K == 0) {
                group_store_codes<NB, P>(Pm, row, cur, gs.s, gs.z);
            } else {
                uint32_t *dst = reinterpret_cast<uint32_t *>(Pm.packed) + cur * (P * NB / 32);
#pragma unroll
                for (int i = 0; i < SCodes<NB, P, true>::kWords; ++i) dst[i] = codes.w[i];
            }
            stream_meta(Pm, cur, gs.s, gs.y, gs.z, it);
            // the lane keeps its finished group's row and state until it takes the next one:
            // the pair stays consistent, so its rounds stay inside the table
            cur = -1;
        }
    }
    allow_dependents();  // the fixup kernel may take the SMs this CTA leaves
    // this warp's per-round sums (16-bit chunks) -> 128-bit global sums
    __syncwarp();
    for (int i = lane; i < 2 * K; i += 32) {
        const unsigned *c = acc_w + 4 * i;
        const unsigned __int128 v = (unsigned __int128)c[0] + ((unsigned __int128)c[1] << 16) +
                                    ((unsigned __int128)c[2] << 32) + ((unsigned __int128)c[3] << 48);
        const u64 lo64 = (u64)v, hi64 = (u64)(v >> 64);
        if (lo64 | hi64) {
            const u64 old = atomicAdd(Pm.acc + 2 * i, lo64);
            const u64 carry = (old + lo64 < old) ? 1ull : 0ull;
            if (hi64 + carry) atomicAdd(Pm.acc + 2 * i + 1, hi64 + carry);
        }
    }
    // the last CTA to finish applies the stop rule once for the whole tensor
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&ctl_of(Pm)->done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (last && threadIdx.x == 0) {
        __threadfence();
        stop_rule(Pm);
    }
}

// Groups whose own last round f lies past the kept round b make exactly min(b, f) zero
// updates again and rewrite their codes and metadata.  Nothing to do when b = iters - 1.
template <int NB, int P>
__global__ void __launch_bounds__(kThreads) hqq_stream_fixup_kernel(const __grid_constant__ QParams Pm) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int NQ = 1 << NB;
    constexpr float kQmax = (float)(NQ - 1);
    const int K = Pm.K;
    wait_prerequisite();  // the stream kernel has finished and applied the stop rule
    const int b = __ldcg(&ctl_of(Pm)->b);
    if (K == 0 || b >= K - 1) return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *tabw = reinterpret_cast<float *>(smem) + warp * NQ * 32;
    const uint32_t col = (uint32_t)__cvta_generic_to_shared(tabw + lane);
    const uint32_t tab_adj = col - (0x4B400000u << 7);
    // each lane scans 16 groups' last rounds with one 16-byte load (fk is 16-byte aligned: it
    // follows the 32-byte-multiple round sums in the workspace), then the warp replays the
    // stale ones, one per lane at a time
    const int64_t wstride = (int64_t)gridDim.x * kWarps * 512;
    for (int64_t wbase = ((int64_t)blockIdx.x * kWarps + warp) * 512; wbase < Pm.G; wbase += wstride) {
        const int64_t c0 = wbase + 16 * lane;
        uint32_t mask = 0;  // bit j: group c0 + j is stale
        if (c0 + 16 <= Pm.G) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(Pm.fk + c0));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if ((int)((w4[j >> 2] >> (8 * (j & 3))) & 0xffu) > b) mask |= 1u << j;
        } else {
            for (int j = 0; j < 16 && c0 + j < Pm.G; ++j)
                if ((int)__ldcg(Pm.fk + c0 + j) > b) mask |= 1u << j;
        }
        while (__any_sync(kFull, mask != 0u)) {
            const bool stale = mask != 0u;
            const int64_t grp = stale ? c0 + (__ffs(mask) - 1) : 0;
            mask &= mask - 1u;
            const int f = stale ? (int)__ldcg(Pm.fk + grp) : 0;
            SRow<P> row;
#pragma unroll
            for (int i = 0; i < P / 2; ++i) row.h[i] = 0;
            SGroup gs;
            gs.idle();
            if (stale) {
                load_row<P>(row, Pm.W + grp * P, -1);  // synchronous: the row is read once
                group_init<NB, P>(row, Pm.eps_tiny, Pm.scale_max, gs);
            }
            const int n = stale ? min(b, f) : 0;
            for (int r = 0; __any_sync(kFull, r < n); ++r) {
                build_table<NQ>(col, gs.s, gs.y, gs.z);
                float esum, zsum;
                SCodes<NB, P, false> nocodes;
                stream_round<NB, P, true, false>(row, gs.s, gs.z, tab_adj, esum, zsum, nocodes);
                const int rr = min(r, K - 1);
                const float B = resid_bound(__fadd_rn(gs.lo, gs.z), __fadd_rn(gs.hi, gs.z), gs.A, gs.z, gs.y, kQmax);
                const bool slow = r < n && B > Pm.thr[rr];
                if (slow) zsum = group_zsum_shrink<NB>(Pm.W + grp * P, P, P, gs.s, gs.z, tab_adj, Pm.beta[rr], Pm.p);
                const float znew = __fmul_rn(zsum, 1.0f / (float)P);
                if (r < n) gs.z = znew;
            }
            if (stale) {
                group_store_codes<NB, P>(Pm, row, grp, gs.s, gs.z);
                stream_meta(Pm, grp, gs.s, gs.y, gs.z, -1);
            }
        }
    }
}

// byte-per-code staging -> packed words (only for axis = 0 layouts that tiles cannot pack)
template <int NB>
__global__ void pack_codes_kernel(const uint8_t *codes, int64_t N, uint8_t *packed,
                                  int64_t packed_bytes) {
    constexpr int CPW = Pack<NB>::cpw;
    wait_prerequisite();  // the fixup kernel has rewritten its stale codes
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
    wait_prerequisite();  // the codes may come from the kernel launched just before
    allow_dependents();
    uint32_t wd[kDqU];
    // MODE 3 (axis 1, g >= codes per word): a word spans at most two groups; both metadata
    // pairs are loaded here, alongside the word, and codes c < cb belong to the first
    float z0[MODE == 3 ? kDqU : 1], d0[MODE == 3 ? kDqU : 1], z1[MODE == 3 ? kDqU : 1],
        d1[MODE == 3 ? kDqU : 1];
    int cb[MODE == 3 ? kDqU : 1];
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
            if constexpr (MODE == 3) {
                const int64_t n0 = wi * CPW;
                const int64_t k0 = wpg_shift >= 0 ? (n0 >> wpg_shift) : n0 / g;
                const int64_t k1 = k0 + 1 < G ? k0 + 1 : k0;
                cb[u] = (int)(g - (n0 - k0 * g));
                z0[u] = __half2float(__ldg(zero + k0));
                d0[u] = __half2float(__ldg(scale + k0));
                z1[u] = __half2float(__ldg(zero + k1));
                d1[u] = __half2float(__ldg(scale + k1));
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
        if constexpr (MODE == 3) {
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                const bool first = c < cb[u];
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (NB * c)) & MASK)), 8388608.0f);
                v[c] = __fmul_rn(__fsub_rn(qf, first ? z0[u] : z1[u]), first ? d0[u] : d1[u]);
            }
        } else if (MODE == 0) {
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

template <int NB>
cudaError_t launch_dequant(const uint8_t *pk, const __half *sc, const __half *ze, int64_t N, int g,
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
    // programmatic launch: overlaps the kernel before it, which the kernel waits for
    if (axis == 1 && g % CPW == 0)
        return launch_pdl(hqq_dequant_kernel<NB, 0>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, shift, false, out);
    if (axis == 1 && g >= CPW) {  // a word spans at most two groups
        int gs = -1;
        if ((g & (g - 1)) == 0) { gs = 0; while ((1 << gs) < g) ++gs; }
        return launch_pdl(hqq_dequant_kernel<NB, 3>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, gs, false, out);
    }
    if (axis == 1)
        return launch_pdl(hqq_dequant_kernel<NB, 1>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, -1, false, out);
    return launch_pdl(hqq_dequant_kernel<NB, 2>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, -1, vec_meta, out);
}


// ==========================================================================================
// The quantized layer's forward product for one input vector [HQQ 算法解读,
// "从压缩文件到一次前向"]: unpack -> (q - zero) * scale -> x @ W_hat.T, fused so that W_hat never
// reaches memory.  Each W_hat[r, c] is the exact fp16 value hqq_dequantize writes; the product
// with the fp16 x[c] is exact in binary32, and the row sum runs in binary32.
// ==========================================================================================

// Axis 1, 2- or 4-bit, cols and g multiples of the codes per word: one warp per output row.
// Lane l takes the row's words l, l + 32, ... (every warp load covers 128 contiguous bytes) and
// loads kGvU of them, with their metadata, before using any: a 4096-column 4-bit row is one
// batch, so a warp waits for memory once.  A word's codes are dequantized in pairs exactly as
// hqq_dequantize does (a code c becomes 2^23 + c by a byte permute against 0x4B000000, then
// (q - z) * Delta in binary32, rounded to fp16) and multiplied with x in packed binary32 FMAs.
constexpr int kGvU = 16;

template <int NB>
__device__ __forceinline__ float2 gemv_word(uint32_t w, float zf, float df, const __half *xw,
                                            float2 acc) {
    const float2 nm = make_float2(-8388608.0f, -8388608.0f), nz = make_float2(-zf, -zf);
    const float2 d2 = make_float2(df, df);
    constexpr int CPW = Pack<NB>::cpw;
    uint32_t xs[CPW / 2];
#pragma unroll
    for (int v = 0; v < CPW / 8; ++v) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(xw) + v);
        xs[4 * v] = xv.x; xs[4 * v + 1] = xv.y; xs[4 * v + 2] = xv.z; xs[4 * v + 3] = xv.w;
    }
    if constexpr (NB == 4) {
        const uint32_t ev = w & 0x0F0F0F0Fu, od = (w >> 4) & 0x0F0F0F0Fu;  // codes 2i, 2i+1 in byte i
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 q = make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u + i)),
                                         __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u + i)));
            const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
            const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xs[i]));
            acc = __ffma2_rn(__half22float2(__floats2half2_rn(v.x, v.y)), xf, acc);
        }
    } else {  // 2 bit: field s of byte b is code 4b + s
        uint32_t f[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) f[s] = (w >> (2 * s)) & 0x03030303u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // codes 2i, 2i+1: byte i/2, fields 2(i%2) and +1
            const int b = i >> 1, s = 2 * (i & 1);
            const float2 q = make_float2(__uint_as_float(__byte_perm(f[s], 0x4B000000u, 0x7540u + b)),
                                         __uint_as_float(__byte_perm(f[s + 1], 0x4B000000u, 0x7540u + b)));
            const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
            const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xs[i]));
            acc = __ffma2_rn(__half22float2(__floats2half2_rn(v.x, v.y)), xf, acc);
        }
    }
    return acc;
}

template <int NB>
__global__ void __launch_bounds__(256) hqq_gemv_kernel(const uint32_t *__restrict__ packed,
                                                       const __half *__restrict__ scale,
                                                       const __half *__restrict__ zero,
                                                       int64_t rows, int wpr, int gpr,
                                                       int wpg_shift, int wpg,
                                                       const __half *__restrict__ x,
                                                       float *__restrict__ y) {
    constexpr int CPW = Pack<NB>::cpw;
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    wait_prerequisite();  // codes and x may come from the kernel launched just before
    allow_dependents();
    if (row >= rows) return;  // whole warps
    const uint32_t *prow = packed + row * wpr;
    const int64_t k0 = row * gpr;
    float2 acc = make_float2(0.0f, 0.0f);
    for (int w0 = lane; w0 < wpr; w0 += 32 * kGvU) {
        uint32_t wd[kGvU];
        float zf[kGvU], df[kGvU];
#pragma unroll
        for (int u = 0; u < kGvU; ++u) {
            const int w = w0 + 32 * u;
            wd[u] = 0;
            zf[u] = 0.0f;
            df[u] = 0.0f;
            if (w < wpr) {
                const int64_t k = k0 + (wpg_shift >= 0 ? (w >> wpg_shift) : w / wpg);
                wd[u] = __ldcs(prow + w);
                zf[u] = __half2float(__ldg(zero + k));
                df[u] = __half2float(__ldg(scale + k));
            }
        }
#pragma unroll
        for (int u = 0; u < kGvU; ++u) {
            const int w = w0 + 32 * u;
            if (w < wpr) acc = gemv_word<NB>(wd[u], zf[u], df[u], x + (int64_t)w * CPW, acc);
        }
    }
    float s = __fadd_rn(acc.x, acc.y);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, off));
    if (lane == 0) y[row] = s;
}

// Any other layout: one warp per output row, each lane takes columns lane, lane + 32, ...
// and reads its codes one at a time (flat row-major code order, groups by axis).
template <int NB>
__global__ void __launch_bounds__(256) hqq_gemv_any_kernel(const uint8_t *__restrict__ packed,
                                                           const __half *__restrict__ scale,
                                                           const __half *__restrict__ zero,
                                                           int64_t rows, int64_t cols, int64_t g,
                                                           int64_t G, int axis,
                                                           const __half *__restrict__ x,
                                                           float *__restrict__ y) {
    constexpr uint32_t MASK = (1u << NB) - 1u;
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    wait_prerequisite();
    allow_dependents();
    if (row >= rows) return;
    float acc = 0.0f;
    for (int64_t c = lane; c < cols; c += 32) {
        const int64_t n = row * cols + c;
        uint32_t q;
        if (NB == 3) {
            const uint32_t wv = __ldg(reinterpret_cast<const uint32_t *>(packed) + n / 10);
            q = (wv >> (3 * (int)(n % 10))) & MASK;
        } else {
            const int per = 8 / NB;
            q = ((uint32_t)__ldg(packed + n / per) >> (NB * (int)(n % per))) & MASK;
        }
        const int64_t k = axis == 1 ? n / g : n % G;
        const float v = __fmul_rn(__fsub_rn((float)q, __half2float(__ldg(zero + k))), __half2float(__ldg(scale + k)));
        acc = __fmaf_rn(__half2float(__float2half_rn(v)), __half2float(__ldg(x + c)), acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, off));
    if (lane == 0) y[row] = acc;
}

template <int NB>
cudaError_t launch_gemv(const uint8_t *pk, const __half *sc, const __half *ze, int64_t rows,
                        int64_t cols, int64_t g, int64_t G, int axis, const __half *x, float *y,
                        cudaStream_t st) {
    constexpr int CPW = Pack<NB>::cpw;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    const int64_t wpr = cols / CPW;
    if (NB != 3 && axis == 1 && cols % CPW == 0 && g % CPW == 0 && ((uintptr_t)x & 15) == 0 &&
        wpr < ((int64_t)1 << 30)) {
        const int wpg = (int)(g / CPW);
        int shift = -1;
        if ((wpg & (wpg - 1)) == 0) { shift = 0; while ((1 << shift) < wpg) ++shift; }
        return launch_pdl(hqq_gemv_kernel<NB>, blocks, 256, 0, st, (const uint32_t *)pk, sc, ze,
                          rows, (int)wpr, (int)(cols / g), shift, wpg, x, y);
    }
    return launch_pdl(hqq_gemv_any_kernel<NB>, blocks, 256, 0, st, pk, sc, ze, rows, cols, g, G,
                      axis, x, y);
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
struct Plan {
    int64_t N, G;
    int g, P, L, stride, tile;  // stride: floats per tile row
    int64_t ntiles;
    bool aligned;  // packed words can be written per tile
    bool stream;   // axis 1 with groups up to 128 and a whole number of packed words
    size_t ws_acc, ws_fk, ws_tile, ws_stale, ws_codes, ws_total;
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
    pl->stride = P + (P >= 64 ? 8 : 0);  // halves per tile row (the padding staggers banks)
    const int target = 40960;            // halves of W per tile
    const int cap = std::max(1, target / pl->stride);
    const int unit = axis == 1 ? (int)(320 / gcd64(pl->g, 320))  // tiles of 320k elements: word
                               : 80;                             // (8, 16, 10 codes) and 16-byte
    pl->tile = unit * std::max(1, cap / unit);                   // aligned; 80 = lcm(8, 16, 10)
    // two CTAs per SM: keep the whole shared-memory layout within 110 KB
    while (pl->tile > unit &&
           smem_layout(pl->tile, pl->stride, 1 << nbits, pl->L, iters).total > 110 * 1024)
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
    // the streaming engine: axis 1, 2- and 4-bit codes, groups of 16 .. 128 that are whole
    // 32-bit words of the output (its codes are stored straight from registers)
    pl->stream = axis == 1 && nbits != 3 && P <= 128 && pl->g == P && (pl->g * nbits) % 32 == 0;
    const int K = iters > 0 ? iters : 1;
    pl->ws_acc = (size_t)4 * K * sizeof(u64) + 32;  // per-round sums + control words (zeroed)
    pl->ws_fk = (size_t)((pl->G + 15) / 16 * 16);
    pl->ws_tile = (size_t)((pl->ntiles + 15) / 16 * 16);
    pl->ws_stale = (size_t)(4 * pl->ntiles + 15) / 16 * 16;
    pl->ws_codes = pl->aligned ? 0 : (size_t)((N + 15) / 16 * 16);
    pl->ws_total = pl->ws_acc + pl->ws_fk + pl->ws_tile + pl->ws_stale + pl->ws_codes;
    return HQQ_OK;
}

bool aligned_to(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }


template <int NB, int L, bool FULL, bool DIRECT>
cudaError_t launch_quant(const QParams &P, int64_t ntiles, cudaStream_t st) {
    const SmemLayout lay = smem_layout(P.tile, P.stride, 1 << NB, L, P.K);
    cudaError_t e = cudaFuncSetAttribute(hqq_search_kernel<NB, L, FULL, DIRECT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(hqq_fixup_kernel<NB, L, FULL, DIRECT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    // zero kernel -> search -> fixup (-> pack), the later ones with programmatic launches
    hqq_zero_kernel<<<1, 256, 0, st>>>(P.acc, (int)P.acc_words);
    e = launch_pdl(hqq_search_kernel<NB, L, FULL, DIRECT>, (unsigned)ntiles, kThreads, lay.total, st, P);
    if (e != cudaSuccess) return e;
    const unsigned fix_blocks = (unsigned)std::min<int64_t>(ntiles, 148 * 2);  // one wave
    e = launch_pdl(hqq_fixup_kernel<NB, L, FULL, DIRECT>, fix_blocks, kThreads, lay.total, st, P);
    if (e != cudaSuccess) return e;
    if (P.codes_u8) {
        const int64_t nw = (P.N + Pack<NB>::cpw - 1) / Pack<NB>::cpw;
        const unsigned blocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 16);
        e = launch_pdl(pack_codes_kernel<NB>, blocks, 256, 0, st, (const uint8_t *)P.codes_u8, P.N,
                       P.packed, P.packed_bytes);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <int NB, bool FULL, bool DIRECT>
cudaError_t launch_quant_l(const QParams &P, int L, int64_t ntiles, cudaStream_t st) {
    switch (L) {
    case 1: return launch_quant<NB, 1, FULL, DIRECT>(P, ntiles, st);
    case 2: return launch_quant<NB, 2, FULL, DIRECT>(P, ntiles, st);
    case 4: return launch_quant<NB, 4, FULL, DIRECT>(P, ntiles, st);
    case 8: return launch_quant<NB, 8, FULL, DIRECT>(P, ntiles, st);
    default: return launch_quant<NB, 16, FULL, DIRECT>(P, ntiles, st);
    }
}

template <int NB, int P>
cudaError_t launch_stream(const QParams &Pm, cudaStream_t st) {
    const int smem = StreamSmem::bytes(P, 1 << NB, Pm.K);
    auto k1 = hqq_stream_kernel<NB, P>;
    auto k2 = hqq_stream_fixup_kernel<NB, P>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k1, kThreads, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    // warps that take groups in each CTA: all of them once the tensor fills the resident grid,
    // fewer (down to one) for a small tensor, so that its groups land on as many SMs as possible
    const int64_t slots = (int64_t)sms * per_sm;
    const int64_t warps_needed = (Pm.G + 31) / 32;
    QParams Q = Pm;
    Q.stream_warps = (int)std::min<int64_t>(kWarps, std::max<int64_t>(1, (warps_needed + slots - 1) / slots));
    const unsigned blocks = (unsigned)std::max<int64_t>(
        1, std::min<int64_t>(slots, (warps_needed + Q.stream_warps - 1) / Q.stream_warps));
    // zero kernel -> stream kernel -> fixup kernel, each later one launched with programmatic
    // stream serialization so that its launch overlaps the kernel before it
    hqq_zero_kernel<<<1, 256, 0, st>>>(Pm.acc, (int)Pm.acc_words);
    e = launch_pdl(k1, blocks, kThreads, smem, st, Q);
    if (e != cudaSuccess) return e;
    const unsigned fix_blocks = (unsigned)std::min<int64_t>(slots, (Pm.G + kWarps * 512 - 1) / (kWarps * 512));
    e = launch_pdl(k2, std::max(1u, fix_blocks), kThreads, smem, st, Q);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int NB>
cudaError_t launch_stream_nb(const QParams &Pm, int P, cudaStream_t st) {
    switch (P) {
    case 16: return launch_stream<NB, 16>(Pm, st);
    case 32: return launch_stream<NB, 32>(Pm, st);
    case 64: return launch_stream<NB, 64>(Pm, st);
    default: return launch_stream<NB, 128>(Pm, st);
    }
}

// full: group size a power of two >= 16 (every slot of a lane holds an element); direct:
// axis 1 with 2- or 4-bit codes and group size a multiple of 16 (a lane's 16 codes are whole
// bytes of the output)
template <int NB>
cudaError_t launch_quant_nb(const QParams &P, int L, bool full, bool direct, int64_t ntiles,
                            cudaStream_t st) {
    if (NB != 3 && direct && L == 16)
        return full ? launch_quant<NB, 16, true, NB != 3>(P, ntiles, st)
                    : launch_quant<NB, 16, false, NB != 3>(P, ntiles, st);
    return full ? launch_quant_l<NB, true, false>(P, L, ntiles, st)
                : launch_quant_l<NB, false, false>(P, L, ntiles, st);
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
    uint8_t *wsp = (uint8_t *)workspace;
    P.fk = wsp + pl.ws_acc;
    P.tile_maxf = wsp + pl.ws_acc + pl.ws_fk;
    P.stale = (int *)(wsp + pl.ws_acc + pl.ws_fk + pl.ws_tile);
    P.codes_u8 = pl.aligned ? nullptr : wsp + pl.ws_acc + pl.ws_fk + pl.ws_tile + pl.ws_stale;
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
    if (pl.stream) {  // one lane per group (each launcher zeroes the round sums itself)
        e = nbits == 4 ? launch_stream_nb<4>(P, pl.P, st) : launch_stream_nb<2>(P, pl.P, st);
    } else {
        const bool direct = axis == 1 && pl.g % 16 == 0;
        switch (nbits) {
        case 4: e = launch_quant_nb<4>(P, pl.L, pl.g == pl.P, direct, pl.ntiles, st); break;
        case 3: e = launch_quant_nb<3>(P, pl.L, pl.g == pl.P, false, pl.ntiles, st); break;
        default: e = launch_quant_nb<2>(P, pl.L, pl.g == pl.P, direct, pl.ntiles, st); break;
        }
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
    cudaError_t e;
    switch (nbits) {
    case 4: e = launch_dequant<4>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
    case 3: e = launch_dequant<3>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
    default: e = launch_dequant<2>(pk, sc, ze, pl.N, pl.g, pl.G, axis, pb, out, st); break;
    }
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
    cudaError_t e;
    switch (nbits) {
    case 4: e = launch_gemv<4>(pk, sc, ze, rows, cols, pl.g, pl.G, axis, xh, y, st); break;
    case 3: e = launch_gemv<3>(pk, sc, ze, rows, cols, pl.g, pl.G, axis, xh, y, st); break;
    default: e = launch_gemv<2>(pk, sc, ze, rows, cols, pl.g, pl.G, axis, xh, y, st); break;
    }
    return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HQQ_OK : HQQ_ERR_CUDA;
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
