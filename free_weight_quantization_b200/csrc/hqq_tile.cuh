// hqq_tile.cuh -- the tile engine of the B200 HQQ quantizer: axis 0 (groups strided along the
// output dimension), 3-bit codes, and group sizes that are not whole power-of-two rows.
//
// One CTA of 256 threads per tile of groups staged in shared memory [HQQ 算法解读, "`axis` 不是
// 一个无关紧要的开关"]; a segment of L = P/16 lanes holds one group (16 elements per lane) and runs
// round after round until its zero stops moving or `iters` rounds are done; exact per-round
// error counters, the stop rule in the last CTA to finish, and a fixup kernel that replays the
// groups whose own last round lies past the kept one.
#pragma once

#include <algorithm>

#include "hqq_common.cuh"

namespace {

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
__device__ __forceinline__ void round_elems(const float (&w)[kE], const float (&ws)[kE], float s, float z,
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
        if constexpr (TileTab<NB>::on)
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(what) : "r"(tab_adj + (bits << kShift)));
        else
            what = __fdiv_rn(__fsub_rn(qf, z), s);  // (q - z)/s, the IEEE division itself
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
            if constexpr (TileTab<NB>::on) {
                __syncwarp();
#pragma unroll
                for (int kk = 0; kk < (NQ + L - 1) / L; ++kk) {
                    const int k = l + kk * L;
                    if (k < NQ) tab[k * NSEG + sg] = __fdiv_rn(__fsub_rn(lf + (float)(kk * L), z), s);
                }
                __syncwarp();
            }
            float absr[kE], term[kE];
            if (noclip) round_elems<NB, NSEG, false, FULL, DIRECT>(w, ws, s, z, tab_adj, nvalid, absr, term, codes);
            else round_elems<NB, NSEG, true, FULL, DIRECT>(w, ws, s, z, tab_adj, nvalid, absr, term, codes);
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
                    const float what = TileTab<NB>::on ? tab[(__float_as_int(u) & (NQ - 1)) * NSEG + sg]
                                                       : __fdiv_rn(__fsub_rn(qf, z), s);
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
                    word |= (uint32_t)cb[grp * rowb + j] << (Pack<NB>::slot * k);
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
                if (col < tg) word |= (uint32_t)cb[col * rowb + j] << (Pack<NB>::slot * k);
            }
            store_word((j * P.G + t0) / CPW + wr, word);
        }
    }
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
        const SmemLayout lay = smem_layout(P.tile, P.stride, TileTab<NB>::nq, L, P.K);
        wh = reinterpret_cast<__half *>(base + lay.wh);
        s_t = reinterpret_cast<float *>(base + lay.s_t);
        z_t = reinterpret_cast<float *>(base + lay.z_t);
        lo_t = reinterpret_cast<float *>(base + lay.lo_t);
        hi_t = reinterpret_cast<float *>(base + lay.hi_t);
        f_t = base + lay.f_t;
        tab = reinterpret_cast<float *>(base + lay.tab) + (threadIdx.x >> 5) * TileTab<NB>::nq * (32 / L);
        acc = reinterpret_cast<unsigned *>(base + lay.acc);
        acc_w = acc + (threadIdx.x >> 5) * 8 * (P.K > 0 ? P.K : 1);
        thr = reinterpret_cast<float *>(base + lay.thr);
        beta = reinterpret_cast<double *>(base + lay.beta);
    }
};

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
            if (n < N) word |= (uint32_t)codes[n] << (Pack<NB>::slot * c);
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

// ---- host side
template <int NB, int L, bool FULL, bool DIRECT>
cudaError_t launch_quant(const QParams &P, int64_t ntiles, cudaStream_t st) {
    const SmemLayout lay = smem_layout(P.tile, P.stride, TileTab<NB>::nq, L, P.K);
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

// full: group size a power of two >= 16 (every slot of a lane holds an element); direct:
// axis 1 with 2- or 4-bit codes and group size a multiple of 16 (a lane's 16 codes are whole
// bytes of the output)
template <int NB>
cudaError_t launch_quant_nb(const QParams &P, int L, bool full, bool direct, int64_t ntiles,
                            cudaStream_t st) {
    constexpr bool kDirect = NB == 2 || NB == 4;
    if (kDirect && direct && L == 16)
        return full ? launch_quant<NB, 16, true, kDirect>(P, ntiles, st)
                    : launch_quant<NB, 16, false, kDirect>(P, ntiles, st);
    return full ? launch_quant_l<NB, true, false>(P, L, ntiles, st)
                : launch_quant_l<NB, false, false>(P, L, ntiles, st);
}


}  // namespace

namespace hqq_impl {

template <int NB>
cudaError_t launch_tile_nb(const QParams &P, int L, bool full, bool direct, int64_t ntiles,
                           cudaStream_t st) {
    return launch_quant_nb<NB>(P, L, full, direct, ntiles, st);
}

}  // namespace hqq_impl
