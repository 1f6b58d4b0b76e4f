// hqq_stream.cu -- the stream engine of the B200 HQQ quantizer: axis 1, 2- or 4-bit codes,
// power-of-two groups of 16 .. 128 elements that fill whole 32-bit words of the output.
//
// A persistent kernel with one group per lane [HQQ 算法解读, "第二拍：half-quadratic 迭代修正零点"]:
// the lane keeps the group's fp16 row in registers for all its rounds, its table of the 2^b
// reconstructions in its own shared-memory column, and the next group's row in a swizzled
// shared-memory slot (cp.async, one group ahead).  Groups come from a global counter; once it
// is empty, idle lanes take the queued groups of busy ones, and a warp's last few groups are
// split over segments of lanes.  A group runs round after round until its zero stops moving
// (every later round would repeat it exactly) or `iters` rounds are done; its error goes to
// exact per-round counters, its last round's codes are its final codes, the last CTA applies
// the stop rule, and a fixup kernel replays the groups whose own last round lies past the kept
// one.
#include <algorithm>

#include "hqq_common.cuh"

namespace {

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

template <int NB, int P, bool DIRECT>
struct SCodes {  // a lane's codes of the current round, in the output's packed format
    static constexpr int kWords = DIRECT ? P * NB / 32 : 1;
    uint32_t w[kWords];
    // code j from the rounded value's bits 0x4B400000 + q: the word accumulates bits << (NB k)
    // (one shift-add per code, the word's first code slot first), and finish() takes the
    // constant part 0x4B400000 << (NB k) of every slot off (all arithmetic mod 2^32)
    __device__ __forceinline__ void put(int j, uint32_t bits) {
        constexpr int CPW = 32 / NB;
        const int k = j % CPW;
        w[j / CPW] = k == 0 ? bits : w[j / CPW] + (bits << (NB * k));
    }
    __device__ __forceinline__ void finish() {
        constexpr uint32_t bias = code_bias();
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] -= bias;
    }
    static __host__ __device__ constexpr uint32_t code_bias() {
        uint32_t c = 0;
        for (int k = 0; k < 32 / NB; ++k) c += 0x4B400000u << (NB * k);
        return c;
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
    if (DIRECT) codes.finish();
    esum = sa[LOGN];
    zsum = st[LOGN];
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
        if (__any_sync(kFull, slow)) {
            // the exact binary64 shrink, each lane over its own slice; the segment's shuffle
            // levels then continue the halving, the order of the whole-group evaluation
            float zs = slow ? group_zsum_shrink<NB>(Pm.W + me.cur * P + l * E, E, E, me.gs.s, me.gs.z, tab_adj,
                                                    beta_s[ri], Pm.p)
                            : 0.0f;
#pragma unroll
            for (int off = 1; off < L; off <<= 1) zs = __fadd_rn(zs, __shfl_xor_sync(kFull, zs, off));
            if (slow) zsum = zs;
        }
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
                if (l == 0 && Pm.zring) Pm.zring[me.cur * K + me.it] = znew;
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
    // so its few groups run on many SMs rather than crowding a few; a very small one also takes
    // only stream_lanes groups per warp, so that the lane split below starts at once
    int64_t nxt = warp < Pm.stream_warps ? claim(Pm, lane < Pm.stream_lanes) : -1;
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
                    if (Pm.zring) Pm.zring[cur * K + it] = znew;
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
                if constexpr ((P * NB / 32) % 4 == 0) {  // whole 16-byte pieces, 16-byte aligned
#pragma unroll
                    for (int i = 0; i < P * NB / 128; ++i)
                        reinterpret_cast<uint4 *>(dst)[i] = make_uint4(codes.w[4 * i], codes.w[4 * i + 1],
                                                                       codes.w[4 * i + 2], codes.w[4 * i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < SCodes<NB, P, true>::kWords; ++i) dst[i] = codes.w[i];
                }
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
            // with the zeros kept per update, the n-th one is read instead of replayed
            if (Pm.zring && stale && n > 0) gs.z = __ldcg(Pm.zring + grp * K + (n - 1));
            for (int r = 0; !Pm.zring && __any_sync(kFull, r < n); ++r) {
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
    QParams Q = Pm;
    // A tensor whose groups fit the resident grid at kTailLanes per warp runs split from the
    // start: every group on up to 8 lanes, so that its rounds, which run one after another,
    // take less time each (256x512 4-bit g64: 2048 groups on 512 warps).
    Q.stream_lanes = 32;
    if (TailMax<NB, P>::value >= 2 && Pm.K > 0 && Pm.G <= slots * kWarps * kTailLanes) Q.stream_lanes = kTailLanes;
    const int64_t warps_needed = (Pm.G + Q.stream_lanes - 1) / Q.stream_lanes;
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

}  // namespace

namespace hqq_impl {

cudaError_t launch_stream_engine(const QParams &P, int nbits, int group_size, cudaStream_t st) {
    return nbits == 4 ? launch_stream_nb<4>(P, group_size, st) : launch_stream_nb<2>(P, group_size, st);
}

}  // namespace hqq_impl
