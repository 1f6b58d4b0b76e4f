// hqq_dequant.cu -- unpack + dequantize and the fused forward product of the B200 HQQ library
// [HQQ 算法解读, "量化公式" and "从压缩文件到一次前向"].
#include "hqq_common.cuh"

namespace {

// ------------------------------------------------------------------------------------------
// dequantize [HQQ 算法解读, "量化公式" and "从压缩文件到一次前向"]: W = (q - z) * Delta
// One packed 32-bit word (8, 16 or 10 codes) per lane and step, so that a warp's loads cover
// 128 contiguous bytes and its stores 512 contiguous bytes (4 bit).  A thread handles kDqU
// words spaced a block apart, all loaded before any is expanded.
//   MODE 0: axis 1, group_size a multiple of the codes per word: one group per word
//   MODE 1: axis 1, any group size
//   MODE 2: axis 0 (element n belongs to group n % G)
//   MODE 3: axis 1, group_size at least the codes per word: a word spans two groups at most
// Two more kernels below take layouts these serve less well: 3-bit codes four words per thread
// (16-byte stores), and axis-0 4-bit codes with each word's metadata loaded once per column.
// The forward products follow them.
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
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (Pack<NB>::slot * c)) & MASK)), 8388608.0f);
                v[c] = __fmul_rn(__fsub_rn(qf, first ? z0[u] : z1[u]), first ? d0[u] : d1[u]);
            }
        } else if (MODE == 0) {
            const int64_t k = wpg_shift >= 0 ? (wi >> wpg_shift) : (n0 / g);
            const float zf = __half2float(zero[k]), df = __half2float(scale[k]);
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (Pack<NB>::slot * c)) & MASK)), 8388608.0f);
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
                    const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (Pack<NB>::slot * (c8 + c))) & MASK)), 8388608.0f);
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
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (Pack<NB>::slot * c)) & MASK)), 8388608.0f);
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

// 3-bit codes, axis 1, group size >= 40: four packed words (40 codes) per thread and step, so
// that each thread reads 16 bytes and writes its 80 output bytes with five 16-byte stores
// (a 10-code word alone is 20 bytes of output, which only 4-byte stores can write).  40
// consecutive codes touch at most two groups; both metadata pairs are loaded with the words.
constexpr int kDq3U = 2;

__global__ void __launch_bounds__(kDqThreads) hqq_dequant3_kernel(
    const uint32_t *__restrict__ packed, const __half *__restrict__ scale,
    const __half *__restrict__ zero, int64_t N, int g, int64_t G, int gshift,
    __half *__restrict__ out) {
    const int64_t nwords = (N + 9) / 10, nunits = (N + 39) / 40;
    const int64_t ubase = (int64_t)blockIdx.x * (kDqThreads * kDq3U) + threadIdx.x;
    wait_prerequisite();  // the codes may come from the kernel launched just before
    allow_dependents();
    uint32_t wd[kDq3U][4];
    float z0[kDq3U], d0[kDq3U], z1[kDq3U], d1[kDq3U];
    int cb[kDq3U];
#pragma unroll
    for (int u = 0; u < kDq3U; ++u) {
        const int64_t t = ubase + u * kDqThreads;
#pragma unroll
        for (int i = 0; i < 4; ++i) wd[u][i] = 0u;
        z0[u] = d0[u] = z1[u] = d1[u] = 0.0f;
        cb[u] = 40;
        if (t < nunits) {
            if (4 * t + 4 <= nwords) {
                const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(packed) + t);
                wd[u][0] = v.x; wd[u][1] = v.y; wd[u][2] = v.z; wd[u][3] = v.w;
            } else {  // the last unit may hold fewer than four words
                for (int i = 0; i < 4 && 4 * t + i < nwords; ++i) wd[u][i] = __ldcs(packed + 4 * t + i);
            }
            const int64_t n0 = 40 * t;
            const int64_t k0 = gshift >= 0 ? (n0 >> gshift) : n0 / g;
            const int64_t k1 = k0 + 1 < G ? k0 + 1 : k0;
            cb[u] = (int)(g - (n0 - k0 * g));  // codes c < cb belong to group k0
            z0[u] = __half2float(__ldg(zero + k0));
            d0[u] = __half2float(__ldg(scale + k0));
            z1[u] = __half2float(__ldg(zero + k1));
            d1[u] = __half2float(__ldg(scale + k1));
        }
    }
#pragma unroll
    for (int u = 0; u < kDq3U; ++u) {
        const int64_t t = ubase + u * kDqThreads;
        if (t >= nunits) break;
        const int64_t n0 = 40 * t;
        uint32_t res[20];
#pragma unroll
        for (int c = 0; c < 40; c += 2) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int cc = c + e;
                const bool first = cc < cb[u];
                const uint32_t q = (wd[u][cc / 10] >> (3 * (cc % 10))) & 7u;
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)q), 8388608.0f);
                v[e] = __fmul_rn(__fsub_rn(qf, first ? z0[u] : z1[u]), first ? d0[u] : d1[u]);
            }
            const __half2 h2 = __floats2half2_rn(v[0], v[1]);
            memcpy(&res[c / 2], &h2, 4);
        }
        if (n0 + 40 <= N) {  // 80 bytes at a multiple of 80: 16-byte aligned
            uint4 *dst = reinterpret_cast<uint4 *>(out + n0);
#pragma unroll
            for (int i = 0; i < 5; ++i)
                __stcs(dst + i, make_uint4(res[4 * i], res[4 * i + 1], res[4 * i + 2], res[4 * i + 3]));
        } else {
            unsigned short *o16 = reinterpret_cast<unsigned short *>(out + n0);
#pragma unroll
            for (int c = 0; c < 40; ++c)
                if (n0 + c < N) o16[c] = (unsigned short)(res[c / 2] >> (16 * (c % 2)));
        }
    }
}

// Axis 0 with g dividing rows (and CPW = 8: 4-bit codes): element n is in group n mod G and G is
// a whole number of rows, so the metadata of a word's 8 groups repeats every G elements.  A
// thread owns one such word position j (elements 8 j .. 8 j + 7 of each G-element stripe),
// loads its 8 scale/zero pairs once (two 16-byte loads) and dequantizes kDqA0M of the g words
// at j, j + G/8, ...; consecutive threads take consecutive words, so loads and 16-byte stores
// stay coalesced.  (The general axis-0 path reloads the metadata for every word: four bytes of
// metadata per weight from L2, twice the output's bytes.)
constexpr int kDqA0M = 16;

__global__ void __launch_bounds__(kDqThreads) hqq_dequant_a0_kernel(
    const uint32_t *__restrict__ packed, const __half *__restrict__ scale,
    const __half *__restrict__ zero, int64_t G, int g, __half *__restrict__ out) {
    const int64_t wpg = G / 8;  // words per stripe
    const int64_t t = (int64_t)blockIdx.x * kDqThreads + threadIdx.x;
    const int64_t j = t % wpg, m0 = (t / wpg) * kDqA0M;
    wait_prerequisite();  // the codes may come from the kernel launched just before
    allow_dependents();
    if (m0 >= g) return;
    const uint4 zv = __ldg(reinterpret_cast<const uint4 *>(zero + 8 * j));
    const uint4 dv = __ldg(reinterpret_cast<const uint4 *>(scale + 8 * j));
    const __half *zh = reinterpret_cast<const __half *>(&zv), *dh = reinterpret_cast<const __half *>(&dv);
    float zf[8], df[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        zf[c] = __half2float(zh[c]);
        df[c] = __half2float(dh[c]);
    }
    const int mend = m0 + kDqA0M < g ? (int)m0 + kDqA0M : g;
    uint32_t wd[kDqA0M];
#pragma unroll
    for (int i = 0; i < kDqA0M; ++i) wd[i] = (int)m0 + i < mend ? __ldcs(packed + (m0 + i) * wpg + j) : 0u;
#pragma unroll
    for (int i = 0; i < kDqA0M; ++i) {
        if ((int)m0 + i >= mend) break;
        uint32_t res[4];
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[i] >> (4 * (c + e))) & 15u)), 8388608.0f);
                v[e] = __fmul_rn(__fsub_rn(qf, zf[c + e]), df[c + e]);
            }
            const __half2 h2 = __floats2half2_rn(v[0], v[1]);
            memcpy(&res[c / 2], &h2, 4);
        }
        __stcs(reinterpret_cast<uint4 *>(out) + (m0 + i) * wpg + j, make_uint4(res[0], res[1], res[2], res[3]));
    }
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
    if (NB == 3 && axis == 1 && g >= 40 && ((uintptr_t)pk & 15) == 0 && ((uintptr_t)out & 15) == 0) {
        int gs = -1;
        if ((g & (g - 1)) == 0) { gs = 0; while ((1 << gs) < g) ++gs; }
        const int64_t nunits = (N + 39) / 40;
        const unsigned b3 = (unsigned)((nunits + kDqThreads * kDq3U - 1) / (kDqThreads * kDq3U));
        return launch_pdl(hqq_dequant3_kernel, b3, kDqThreads, 0, st, pw, sc, ze, N, g, G, gs, out);
    }
    if (axis == 1 && g >= CPW) {  // a word spans at most two groups
        int gs = -1;
        if ((g & (g - 1)) == 0) { gs = 0; while ((1 << gs) < g) ++gs; }
        return launch_pdl(hqq_dequant_kernel<NB, 3>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, gs, false, out);
    }
    if (axis == 1)
        return launch_pdl(hqq_dequant_kernel<NB, 1>, blocks, kDqThreads, 0, st, pw, sc, ze, N, g, G, pb, -1, false, out);
    // axis 0, 4-bit, whole 8-group words in every stripe (G % 8 == 0 and N = g G), aligned
    if (NB == 4 && G % 8 == 0 && N == (int64_t)g * G && vec_meta && ((uintptr_t)pk & 15) == 0 &&
        ((uintptr_t)out & 15) == 0) {
        const int64_t threads = (G / 8) * ((g + kDqA0M - 1) / kDqA0M);
        return launch_pdl(hqq_dequant_a0_kernel, (unsigned)((threads + kDqThreads - 1) / kDqThreads), kDqThreads, 0, st,
                          pw, sc, ze, G, g, out);
    }
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

// Axis 1, 2- or 4-bit, group size a multiple of 32 dividing cols: the same product, laid out so
// that the ALU work, not memory latency, sets the pace.  A piece is 32 consecutive codes of a
// row (16 bytes of 4-bit codes, 8 of 2-bit), inside one group.  Each warp takes kGv2Rows rows;
// lane l takes pieces l, l + 32, .. (one warp load covers 512 or 256 contiguous bytes), and
// loads kGv2U pieces of each row with their scale and zero point before using any, then reads
// the piece's 32 values of x once for all the warp's rows.  One row per warp at 63 registers
// lets four CTAs of eight warps share an SM, which hides the loads best (4096^2 4-bit, back to
// back: two rows per warp at two CTAs per SM 9.4 us, two rows at three 11.0 us, one row at
// four 8.3 us).
constexpr int kGv2Rows = 1;
constexpr int kGv2U = 4;

// dot product of one piece (NB words of codes, one group) with its 32 values of x (xs: 16 fp16
// pairs), each W_hat value exactly hqq_dequantize's, accumulated in binary32 pairs
template <int NB>
__device__ __forceinline__ float2 gemv_piece(const uint32_t *cw, float zf, float df, const uint32_t *xs,
                                             float2 acc) {
    const float2 nm = make_float2(-8388608.0f, -8388608.0f), nz = make_float2(-zf, -zf);
    const float2 d2 = make_float2(df, df);
#pragma unroll
    for (int wi = 0; wi < NB; ++wi) {
        const uint32_t w = cw[wi];
        if constexpr (NB == 4) {  // word wi: codes 8 wi .. 8 wi + 7, codes 2i, 2i+1 in byte i
            const uint32_t ev = w & 0x0F0F0F0Fu, od = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 q = make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u + i)),
                                             __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u + i)));
                const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
                const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xs[4 * wi + i]));
                acc = __ffma2_rn(__half22float2(__floats2half2_rn(v.x, v.y)), xf, acc);
            }
        } else {  // word wi: codes 16 wi .. 16 wi + 15; field s of byte b is code 4b + s
            uint32_t f[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) f[s] = (w >> (2 * s)) & 0x03030303u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int b = i >> 1, s = 2 * (i & 1);
                const float2 q = make_float2(__uint_as_float(__byte_perm(f[s], 0x4B000000u, 0x7540u + b)),
                                             __uint_as_float(__byte_perm(f[s + 1], 0x4B000000u, 0x7540u + b)));
                const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
                const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xs[8 * wi + i]));
                acc = __ffma2_rn(__half22float2(__floats2half2_rn(v.x, v.y)), xf, acc);
            }
        }
    }
    return acc;
}

// gshift >= 0: pieces per group 2^gshift; else gpp pieces per group
template <int NB>
__global__ void __launch_bounds__(256, 4) hqq_gemv2_kernel(const uint8_t *__restrict__ packed,
                                                           const __half *__restrict__ scale,
                                                           const __half *__restrict__ zero,
                                                           int64_t rows, int ppr, int gshift, int gpp,
                                                           const __half *__restrict__ x,
                                                           float *__restrict__ y) {
    constexpr int PB = 4 * NB;  // bytes per piece
    const int lane = threadIdx.x & 31;
    const int64_t r0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kGv2Rows;
    wait_prerequisite();  // codes and x may come from the kernel launched just before
    allow_dependents();
    if (r0 >= rows) return;  // whole warps
    const int64_t gpr = gshift >= 0 ? (int64_t)(ppr >> gshift) : (int64_t)(ppr / gpp);  // groups per row
    float2 acc[kGv2Rows];
#pragma unroll
    for (int r = 0; r < kGv2Rows; ++r) acc[r] = make_float2(0.0f, 0.0f);
    for (int p0 = lane; p0 < ppr; p0 += 32 * kGv2U) {
        uint32_t cw[kGv2Rows][kGv2U][NB];
        float zf[kGv2Rows][kGv2U], df[kGv2Rows][kGv2U];
#pragma unroll
        for (int r = 0; r < kGv2Rows; ++r) {
#pragma unroll
            for (int i = 0; i < kGv2U; ++i) {
                const int p = p0 + 32 * i;
#pragma unroll
                for (int wi = 0; wi < NB; ++wi) cw[r][i][wi] = 0u;
                zf[r][i] = 0.0f;
                df[r][i] = 0.0f;
                if (p < ppr && r0 + r < rows) {  // absent pieces: codes 0, z = Delta = 0: zero terms
                    const uint8_t *src = packed + ((r0 + r) * ppr + p) * PB;
                    if constexpr (NB == 4) {
                        const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(src));
                        cw[r][i][0] = v.x; cw[r][i][1] = v.y; cw[r][i][2] = v.z; cw[r][i][3] = v.w;
                    } else {
                        const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(src));
                        cw[r][i][0] = v.x; cw[r][i][1] = v.y;
                    }
                    const int64_t k = (r0 + r) * gpr + (gshift >= 0 ? (p >> gshift) : p / gpp);
                    zf[r][i] = __half2float(__ldg(zero + k));
                    df[r][i] = __half2float(__ldg(scale + k));
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kGv2U; ++i) {
            const int p = p0 + 32 * i;
            if (p < ppr) {
                uint32_t xs[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)p * 32) + v);
                    xs[4 * v] = xv.x; xs[4 * v + 1] = xv.y; xs[4 * v + 2] = xv.z; xs[4 * v + 3] = xv.w;
                }
#pragma unroll
                for (int r = 0; r < kGv2Rows; ++r) acc[r] = gemv_piece<NB>(cw[r][i], zf[r][i], df[r][i], xs, acc[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kGv2Rows; ++r) {
        float s = __fadd_rn(acc[r].x, acc[r].y);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, off));
        if (lane == 0 && r0 + r < rows) y[r0 + r] = s;
    }
}

// The same product with the memory side moved to the bulk-copy engine: a CTA owns 16 rows in
// two stages of 8 (warp w: rows w and w + 8).  One thread issues, per stage, a bulk copy
// (cp.async.bulk, completing on an mbarrier) of the stage's packed rows and of their scale and
// zero rows into shared memory, so that all of a wave's bytes are requested at once without
// holding one register per byte in flight.  The second stage's copy lands while the first is
// computed.  Codes and metadata are then read from shared memory; x (the same for every row)
// through L1.  Waits are bounded: a stage that never lands writes NaN into its outputs.
constexpr int kGv3Rows = 16;  // rows per CTA: two stages of eight
constexpr uint32_t kGv3WaitLimit = 1u << 20;

__device__ __forceinline__ bool gv3_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < kGv3WaitLimit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred P1;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, P1;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (i >= 4) __nanosleep(64);
    }
    return false;
}

__device__ __forceinline__ void gv3_bulk(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// shared memory: codes [16][row_bytes] | scale [16][gpr] | zero [16][gpr] (fp16) | 2 mbarriers
struct Gv3Layout {
    int64_t codes, meta, bars, total;
    __host__ __device__ Gv3Layout(int64_t row_bytes, int64_t gpr) {
        codes = 0;
        meta = kGv3Rows * row_bytes;                                    // a multiple of 16
        bars = (meta + 2 * kGv3Rows * gpr * 2 + 15) / 16 * 16;
        total = bars + 16;
    }
};

template <int NB>
__global__ void __launch_bounds__(256, 2) hqq_gemv3_kernel(const uint8_t *__restrict__ packed,
                                                           const __half *__restrict__ scale,
                                                           const __half *__restrict__ zero,
                                                           int64_t rows, int ppr, int gpr, int gshift,
                                                           int gpp, const __half *__restrict__ x,
                                                           float *__restrict__ y) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int PB = 4 * NB;  // bytes per piece
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row_bytes = (int64_t)ppr * PB;
    const Gv3Layout L(row_bytes, gpr);
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t bar0 = sbase + (uint32_t)L.bars;
    const __half *s_scale = reinterpret_cast<const __half *>(smem + L.meta);
    const __half *s_zero = s_scale + kGv3Rows * gpr;
    const int64_t r0 = (int64_t)blockIdx.x * kGv3Rows;
    wait_prerequisite();  // codes and x may come from the kernel launched just before
    allow_dependents();
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // metadata bytes past the last multiple of 16 of a stage go by plain loads
    for (int s = 0; s < 2; ++s) {
        const int64_t rs = r0 + 8 * s;
        const int nr = (int)(rs < rows ? (rows - rs < 8 ? rows - rs : 8) : 0);
        const int nh = nr * gpr, nbulk = nh / 8 * 8;  // halves; bulk part a multiple of 16 bytes
        for (int i = nbulk + tid; i < nh; i += 256) {
            const_cast<__half *>(s_scale)[8 * s * gpr + i] = scale[rs * gpr + i];
            const_cast<__half *>(s_zero)[8 * s * gpr + i] = zero[rs * gpr + i];
        }
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            const int64_t rs = r0 + 8 * s;
            const int nr = (int)(rs < rows ? (rows - rs < 8 ? rows - rs : 8) : 0);
            const uint32_t cb = (uint32_t)(nr * row_bytes), mb = (uint32_t)(nr * gpr / 8 * 16);
            if (nr == 0) continue;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s), "r"(cb + 2 * mb) : "memory");
            gv3_bulk(sbase + (uint32_t)(8 * s * row_bytes), packed + rs * row_bytes, cb, bar0 + 8 * s);
            if (mb) {
                gv3_bulk(sbase + (uint32_t)(L.meta + 8 * s * gpr * 2), scale + rs * gpr, mb, bar0 + 8 * s);
                gv3_bulk(sbase + (uint32_t)(L.meta + (kGv3Rows + 8 * s) * gpr * 2), zero + rs * gpr, mb, bar0 + 8 * s);
            }
        }
    }
    for (int s = 0; s < 2; ++s) {
        const int lr = warp + 8 * s;  // row within the CTA
        const int64_t row = r0 + lr;
        if (r0 + 8 * s >= rows) break;  // the stage is empty (uniform over the CTA)
        const bool ok = gv3_wait(bar0 + 8 * s, 0u);
        if (row >= rows) continue;  // whole warps
        const unsigned char *crow = smem + lr * row_bytes;
        const __half *srow = s_scale + lr * gpr, *zrow = s_zero + lr * gpr;
        float2 acc = make_float2(0.0f, 0.0f);
        for (int p0 = lane; p0 < ppr; p0 += 32 * kGv2U) {
            uint32_t cw[kGv2U][NB];
            float zf[kGv2U], df[kGv2U];
#pragma unroll
            for (int i = 0; i < kGv2U; ++i) {
                const int p = p0 + 32 * i;
#pragma unroll
                for (int wi = 0; wi < NB; ++wi) cw[i][wi] = 0u;
                zf[i] = df[i] = 0.0f;
                if (p < ppr) {
                    if constexpr (NB == 4) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(crow + p * PB);
                        cw[i][0] = v.x; cw[i][1] = v.y; cw[i][2] = v.z; cw[i][3] = v.w;
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2 *>(crow + p * PB);
                        cw[i][0] = v.x; cw[i][1] = v.y;
                    }
                    const int k = gshift >= 0 ? (p >> gshift) : p / gpp;
                    zf[i] = __half2float(zrow[k]);
                    df[i] = __half2float(srow[k]);
                }
            }
#pragma unroll
            for (int i = 0; i < kGv2U; ++i) {
                const int p = p0 + 32 * i;
                if (p < ppr) {
                    uint32_t xs[16];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)p * 32) + v);
                        xs[4 * v] = xv.x; xs[4 * v + 1] = xv.y; xs[4 * v + 2] = xv.z; xs[4 * v + 3] = xv.w;
                    }
                    acc = gemv_piece<NB>(cw[i], zf[i], df[i], xs, acc);
                }
            }
        }
        float sum = __fadd_rn(acc.x, acc.y);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(kFull, sum, off));
        if (lane == 0) y[row] = ok ? sum : __int_as_float(0x7fc00000);
    }
}

// Axis 0, 4-bit, g dividing rows, cols a multiple of 32: element (r, c) is in group
// (r mod R) cols + c with R = rows / g, so a row's groups are cols consecutive ones and every
// code has its own scale and zero (read through L2: the R rows of metadata are shared by the g
// rows of each stripe).  One warp per row; lane l takes pieces of 32 codes l, l + 32, ..., with
// the piece's 32 zeros, scales and x values as 16-byte loads; pairs are dequantized in packed
// binary32 exactly as dequantize does and multiplied with x in packed FMAs.
template <int NB>
__global__ void __launch_bounds__(256, 3) hqq_gemv_a0_kernel(const uint8_t *__restrict__ packed,
                                                             const __half *__restrict__ scale,
                                                             const __half *__restrict__ zero,
                                                             int64_t rows, int ppr, int R,
                                                             const __half *__restrict__ x,
                                                             float *__restrict__ y) {
    static_assert(NB == 4, "4-bit codes");
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    wait_prerequisite();  // codes and x may come from the kernel launched just before
    allow_dependents();
    if (row >= rows) return;  // whole warps
    const int64_t cols = (int64_t)ppr * 32;
    const uint8_t *crow = packed + row * cols / 2;
    const __half *zrow = zero + (row % R) * cols, *srow = scale + (row % R) * cols;
    const float2 nm = make_float2(-8388608.0f, -8388608.0f);
    float2 acc = make_float2(0.0f, 0.0f);
    for (int p = lane; p < ppr; p += 32) {
        const uint4 cv = __ldcs(reinterpret_cast<const uint4 *>(crow + (int64_t)p * 16));
        const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {  // word wi: codes 8 wi .. 8 wi + 7 of the piece
            const uint4 zv = __ldg(reinterpret_cast<const uint4 *>(zrow + (int64_t)p * 32) + wi);
            const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(srow + (int64_t)p * 32) + wi);
            const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (int64_t)p * 32) + wi);
            const uint32_t zs[4] = {zv.x, zv.y, zv.z, zv.w}, ss[4] = {sv.x, sv.y, sv.z, sv.w};
            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
            const uint32_t ev = cw[wi] & 0x0F0F0F0Fu, od = (cw[wi] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // codes 2i, 2i + 1 of the word
                const float2 q = make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u + i)),
                                             __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u + i)));
                const float2 zf = __half22float2(*reinterpret_cast<const __half2 *>(&zs[i]));
                const float2 df = __half22float2(*reinterpret_cast<const __half2 *>(&ss[i]));
                const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), make_float2(-zf.x, -zf.y)), df);
                const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xs[i]));
                acc = __ffma2_rn(__half22float2(__floats2half2_rn(v.x, v.y)), xf, acc);
            }
        }
    }
    float s = __fadd_rn(acc.x, acc.y);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(kFull, s, off));
    if (lane == 0) y[row] = s;
}

// 3-bit codes, axis 1, g >= 10, cols even: words of 10 codes may straddle rows (cols need not be
// a multiple of 10).  One warp per row; the CTA first copies x into shared memory, so that the
// 10 x values of a word, at any offset, are five 4-byte shared loads (cols is even, so code
// pairs (2i, 2i + 1) of a word sit at even columns).  A word lies in at most two groups; codes
// outside the row contribute nothing.  Values as dequantize computes them, products and sums in
// binary32.
template <int NB>
__global__ void __launch_bounds__(256) hqq_gemv_b3_kernel(const uint32_t *__restrict__ packed,
                                                          const __half *__restrict__ scale,
                                                          const __half *__restrict__ zero,
                                                          int64_t rows, int64_t cols, int g, int64_t G,
                                                          const __half *__restrict__ x,
                                                          float *__restrict__ y) {
    static_assert(NB == 3, "3-bit codes");
    extern __shared__ __align__(16) unsigned char smem[];
    __half *xs = reinterpret_cast<__half *>(smem);
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    wait_prerequisite();  // codes and x may come from the kernel launched just before
    allow_dependents();
    for (int64_t i = threadIdx.x; i < cols / 2; i += blockDim.x)
        reinterpret_cast<uint32_t *>(xs)[i] = __ldg(reinterpret_cast<const uint32_t *>(x) + i);
    __syncthreads();
    if (row >= rows) return;  // whole warps
    const int64_t nb = row * cols, ne = nb + cols;  // the row's flat code range
    const int64_t w0 = nb / 10, w1 = (ne - 1) / 10;
    constexpr int U = 4;  // words per lane loaded before any is used
    float acc = 0.0f;
    for (int64_t wb = w0 + lane; wb <= w1; wb += 32 * U) {
        uint32_t wd[U];
        float za[U], da[U], zb[U], db[U];
        int cb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t w = wb + 32 * u;
            wd[u] = 0u;
            za[u] = da[u] = zb[u] = db[u] = 0.0f;
            cb[u] = 10;
            if (w <= w1) {
                wd[u] = __ldcs(packed + w);
                const int64_t n0 = 10 * w, k0 = n0 / g;
                cb[u] = (int)(g - (n0 - k0 * g));  // codes j < cb belong to group k0
                const int64_t k1 = cb[u] < 10 && k0 + 1 < G ? k0 + 1 : k0;  // past the last group: padding
                za[u] = __half2float(__ldg(zero + k0));
                da[u] = __half2float(__ldg(scale + k0));
                zb[u] = __half2float(__ldg(zero + k1));
                db[u] = __half2float(__ldg(scale + k1));
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t w = wb + 32 * u;
            if (w > w1) break;
            const int64_t n0 = 10 * w;
            const bool whole = n0 >= nb && n0 + 10 <= ne;
#pragma unroll
            for (int j = 0; j < 10; j += 2) {
                float v[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int jj = j + e;
                    const float qf = __fsub_rn(__int_as_float(0x4B000000 | (int)((wd[u] >> (3 * jj)) & 7u)), 8388608.0f);
                    const bool first = jj < cb[u];
                    v[e] = __fmul_rn(__fsub_rn(qf, first ? za[u] : zb[u]), first ? da[u] : db[u]);
                }
                const float2 wh = __half22float2(__floats2half2_rn(v[0], v[1]));
                const int64_t c = n0 + j - nb;  // column of code j (even)
                if (whole || (c >= 0 && c + 1 < cols)) {  // both codes in the row
                    const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(xs + c));
                    acc = __fmaf_rn(wh.x, xf.x, acc);
                    acc = __fmaf_rn(wh.y, xf.y, acc);
                }
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, off));
    if (lane == 0) y[row] = acc;
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
        } else {  // slots of 1, 2, 4 or 8 bits inside bytes
            constexpr int per = 8 / Pack<NB>::slot;
            q = ((uint32_t)__ldg(packed + n / per) >> (Pack<NB>::slot * (int)(n % per))) & MASK;
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
cudaError_t launch_gemv_nb(const uint8_t *pk, const __half *sc, const __half *ze, int64_t rows,
                        int64_t cols, int64_t g, int64_t G, int axis, const __half *x, float *y,
                        cudaStream_t st) {
    constexpr int CPW = Pack<NB>::cpw;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    const int64_t wpr = cols / CPW;
    if constexpr (NB == 2 || NB == 4) {  // the fast paths: 2- and 4-bit axis-1 layouts
        // groups must not cross rows (cols % g == 0): the kernels find a word's group by row
        if (axis == 1 && g % 32 == 0 && cols % g == 0 && ((uintptr_t)x & 15) == 0 && ((uintptr_t)pk & 15) == 0 &&
            cols / 32 < ((int64_t)1 << 30)) {
            const int gpp = (int)(g / 32);
            int shift = -1;
            if ((gpp & (gpp - 1)) == 0) { shift = 0; while ((1 << shift) < gpp) ++shift; }
            // Large matrices (16 MiB of codes and more): the bulk-copy kernel, whose requests
            // keep HBM busier (4096x11008 4-bit: 23.8 -> 21.4 us; 11008x4096: 23.1 -> 18.8 us).
            // Below that its 16-row CTAs are too few to hide the arithmetic (4096^2 4-bit:
            // 11.6 us against 9.3 us).  Bulk copies want 16-byte aligned sources and sizes:
            // rows of whole 16-byte units, aligned metadata; and the 16 rows must fit in shared
            // memory beside a second CTA.
            const int64_t row_bytes = cols * NB / 8, gpr = cols / g;
            const Gv3Layout L3(row_bytes, gpr);
            if (rows * row_bytes >= ((int64_t)16 << 20) && row_bytes % 16 == 0 && ((uintptr_t)sc & 15) == 0 &&
                ((uintptr_t)ze & 15) == 0 && L3.total <= 100 * 1024) {
                cudaError_t e = cudaFuncSetAttribute(hqq_gemv3_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)L3.total);
                if (e != cudaSuccess) return e;
                const unsigned b3 = (unsigned)((rows + kGv3Rows - 1) / kGv3Rows);
                return launch_pdl(hqq_gemv3_kernel<NB>, b3, 256, (size_t)L3.total, st, pk, sc, ze, rows,
                                  (int)(cols / 32), (int)gpr, shift, gpp, x, y);
            }
            const unsigned b2 = (unsigned)((rows + 8 * kGv2Rows - 1) / (8 * kGv2Rows));
            return launch_pdl(hqq_gemv2_kernel<NB>, b2, 256, 0, st, pk, sc, ze, rows, (int)(cols / 32), shift, gpp, x, y);
        }
        if (axis == 1 && cols % CPW == 0 && g % CPW == 0 && cols % g == 0 && ((uintptr_t)x & 15) == 0 &&
            wpr < ((int64_t)1 << 30)) {
            const int wpg = (int)(g / CPW);
            int shift = -1;
            if ((wpg & (wpg - 1)) == 0) { shift = 0; while ((1 << shift) < wpg) ++shift; }
            return launch_pdl(hqq_gemv_kernel<NB>, blocks, 256, 0, st, (const uint32_t *)pk, sc, ze,
                              rows, (int)wpr, (int)(cols / g), shift, wpg, x, y);
        }
    }
    if constexpr (NB == 3) {  // axis 1, x staged in shared memory (at most 48 KB of it)
        if (axis == 1 && g >= 10 && cols % 2 == 0 && cols * 2 <= 48 * 1024 && ((uintptr_t)x & 3) == 0)
            return launch_pdl(hqq_gemv_b3_kernel<NB>, blocks, 256, (int)(cols * 2), st,
                              reinterpret_cast<const uint32_t *>(pk), sc, ze, rows, cols, (int)g, G, x, y);
    }
    if constexpr (NB == 4) {  // axis 0 with whole stripes of rows: per-code metadata by row
        if (axis == 0 && rows % g == 0 && cols % 32 == 0 && cols / 32 < ((int64_t)1 << 30) &&
            rows / g < ((int64_t)1 << 30) &&
            ((((uintptr_t)x | (uintptr_t)pk | (uintptr_t)sc | (uintptr_t)ze) & 15) == 0))
            return launch_pdl(hqq_gemv_a0_kernel<NB>, blocks, 256, 0, st, pk, sc, ze, rows, (int)(cols / 32),
                              (int)(rows / g), x, y);
    }
    return launch_pdl(hqq_gemv_any_kernel<NB>, blocks, 256, 0, st, pk, sc, ze, rows, cols, g, G,
                      axis, x, y);
}

}  // namespace

namespace hqq_impl {

cudaError_t launch_dequantize(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                              int64_t N, int g, int64_t G, int axis, int64_t pb, __half *out,
                              cudaStream_t st) {
    switch (nbits) {
    case 1: return launch_dequant<1>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 2: return launch_dequant<2>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 3: return launch_dequant<3>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 4: return launch_dequant<4>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 5: return launch_dequant<5>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 6: return launch_dequant<6>(pk, sc, ze, N, g, G, axis, pb, out, st);
    case 7: return launch_dequant<7>(pk, sc, ze, N, g, G, axis, pb, out, st);
    default: return launch_dequant<8>(pk, sc, ze, N, g, G, axis, pb, out, st);
    }
}

cudaError_t launch_gemv(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                        int64_t rows, int64_t cols, int64_t g, int64_t G, int axis,
                        const __half *x, float *y, cudaStream_t st) {
    switch (nbits) {
    case 1: return launch_gemv_nb<1>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 2: return launch_gemv_nb<2>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 3: return launch_gemv_nb<3>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 4: return launch_gemv_nb<4>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 5: return launch_gemv_nb<5>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 6: return launch_gemv_nb<6>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    case 7: return launch_gemv_nb<7>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    default: return launch_gemv_nb<8>(pk, sc, ze, rows, cols, g, G, axis, x, y, st);
    }
}

}  // namespace hqq_impl
