// hqq_gemm.cu -- the quantized layer's forward product for a batch of input vectors on the B200
// tensor cores [HQQ 算法解读, "从压缩文件到一次前向", and its `axis` table row "追求低 batch 推理吞吐"]:
//     Y[b, r] = sum_c W_hat[r, c] * X[b, c]
// with W_hat[r, c] exactly the fp16 value hqq_dequantize writes (q - z) * Delta.
//
// Fast path (axis 1, 2- or 4-bit codes, group size a multiple of 8 dividing cols, cols a
// multiple of 64):
//   a CTA owns 128 rows of W (the M of one tcgen05.mma) and a range of 64-column tiles (the
//   columns are split over CTAs so that the grid fills the SMs, two CTAs per SM where shared
//   memory allows).  Its ten warps have fixed roles:
//   * a copy warp: one lane moves the packed codes with TMA in chunks of 128 rows x 128 bytes
//     (four tiles of 4-bit codes, eight of 2-bit; rows past the matrix read as zero) into two
//     chunk buffers, and each tile's 64 columns of X (rows past the batch read as zero) into a
//     ring of S slots, both with the 128-byte swizzle (the tensor cores read K-major B so);
//   * eight dequantization warps: thread (m, h) turns codes 32 h .. 32 h + 31 of tile row m into
//     fp16, with the scales and zero points that the CTA's rows and columns use (read once at
//     the start into shared memory as binary32 pairs, zero for rows past the matrix), and
//     stores them with tcgen05.st into one of four A buffers in tensor memory (lane m, 32
//     columns of fp16 pairs per tile), so that the A operand never crosses shared memory;
//   * an MMA warp: one lane issues four tcgen05.mma.cta_group::1.kind::f16 (K = 16 each, A from
//     tensor memory, B = X from shared memory) per tile that accumulate D = W_hat_tile X_tile^T
//     in binary32 in tensor memory (128 lanes = rows, one column per batch entry), and commits
//     them to the barriers that free the tile's X slot and A buffer.
//   The roles meet only at mbarriers, so copies, dequantization and the tensor cores overlap.
//   At the end the eight dequantization warps read the accumulator with tcgen05.ld (warp w:
//   lanes 32 (w mod 4) .., half the columns each) and add it into Y (atomically when the
//   columns are split over CTAs; Y is zeroed by a small kernel before).
// Every product of two fp16 values is exact in binary32, and the tensor cores accumulate them in
// binary32, so Y is within cols * 2^-23 * sum_c |W_hat X| of the exact sum whatever the order.
// Every other layout runs the generic forward product once per batch entry.
//
// Waits on mbarriers are bounded: a wait that runs out (it never should) makes the CTA write
// NaN into its outputs, so that a wrong result cannot pass silently; every later wait is bounded
// too, the copy warp waits (bounded) for its loads in flight, and the kernel frees its tensor
// memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "hqq_common.cuh"

namespace {

constexpr int kGmM = 128;          // rows of W per CTA: the M of one MMA
constexpr int kGmK = 64;           // columns per tile: four MMAs of K = 16
constexpr int kGmDeqThreads = 256; // the eight dequantization warps
constexpr int kGmCopyWarp = 8;
constexpr int kGmMmaWarp = 9;
constexpr int kGmThreads = 320;
constexpr int kGmMaxBatch = 256;   // the N of one MMA at most
constexpr int kGmMaxGroups = 16;   // groups of one row that a CTA's column range may touch
constexpr int kGmMaxStages = 10;
constexpr int kGmLag = 4;          // A buffers (tensor memory): tiles dequantized ahead of the MMAs
// packed codes move in chunks of 128 rows x 128 bytes (4 tiles of 4-bit codes, 8 of 2-bit): one
// TMA row request carries 128 bytes, and the 128-byte swizzle spreads a warp's reads over the banks
constexpr int kGmChunkRow = 128;
constexpr int kGmChunkBytes = kGmM * kGmChunkRow;
constexpr uint32_t kGmWaitLimit = 1u << 20;

// shared-memory layout of a CTA (offsets from a 1024-byte aligned base): two code-chunk buffers,
// S X slots, the scale/zero table, the mbarriers and the tensor-memory address
struct GemmLayout {
    int c_off, x_off, x_bytes, m_off, bar_off, total;
    __host__ __device__ GemmLayout(int np, int stages, int gpad) {
        c_off = 0;
        x_off = 2 * kGmChunkBytes;
        x_bytes = np * kGmK * 2;               // a multiple of 2048
        m_off = x_off + stages * x_bytes;
        bar_off = m_off + kGmM * gpad * 8;
        // cfull[2], cempty[2], xfull[S], xempty[S], afull[lag], aempty[lag], done, tensor-memory address
        total = bar_off + 8 * (4 + 2 * stages + 2 * kGmLag + 1) + 8 + 1024;  // + alignment slack
    }
};

// tcgen05 shared-memory matrix descriptor: start address, leading-dimension byte offset,
// stride byte offset, all in 16-byte units; descriptor version 1; layout type (0: no swizzle,
// 2: 128-byte swizzle)
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)layout << 61);
}

// instruction descriptor of kind::f16: D binary32, A and B fp16, both K-major, M = 128, N = np
__host__ __device__ constexpr uint32_t umma_idesc_f16(int np) {
    return (1u << 4) | ((uint32_t)(np >> 3) << 17) | ((uint32_t)(kGmM >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}

// one test of the phase with the given parity
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait for the phase with the given parity, out of line: the hot loops only pay for it
// when the first test fails; false if the phase did not complete in time
__device__ __noinline__ bool mbar_wait_slow(uint32_t addr, uint32_t parity) {
    for (uint32_t i = 0; i < kGmWaitLimit; ++i) {
        if (mbar_try(addr, parity)) return true;
        if (i >= 4) __nanosleep(64);  // a waiting warp leaves the issue slots to the working ones
    }
    return false;
}

__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
    return mbar_try(addr, parity) || mbar_wait_slow(addr, parity);
}

__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t addr, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}

// 2-D tiled TMA load of the box at (x, y) into shared memory, completing on mbar
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(mbar) : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

// The 8 codes of one 16-byte piece of a W_hat row (k8 chunk), dequantized exactly as
// hqq_dequantize does: q as binary32 2^23 + c by a byte permute, then (q - 2^23 - z) * Delta
// in binary32, rounded once to fp16.  pair i holds codes 2i and 2i + 1 of the chunk.
template <int NB>
__device__ __forceinline__ uint4 dequant_chunk(uint32_t bits, float zf, float df) {
    const float2 nm = make_float2(-8388608.0f, -8388608.0f), nz = make_float2(-zf, -zf);
    const float2 d2 = make_float2(df, df);
    uint32_t out[4];
    if constexpr (NB == 4) {  // bits: one 32-bit word, eight 4-bit codes
        const uint32_t ev = bits & 0x0F0F0F0Fu, od = (bits >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 q = make_float2(__uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u + i)),
                                         __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u + i)));
            const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
            const __half2 h = __floats2half2_rn(v.x, v.y);
            out[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
    } else {  // NB == 2; bits: 16 bits, eight 2-bit codes; field s of byte b is code 4b + s
        uint32_t f[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) f[s] = (bits >> (2 * s)) & 0x03030303u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int b = i >> 1, s = 2 * (i & 1);
            const float2 q = make_float2(__uint_as_float(__byte_perm(f[s], 0x4B000000u, 0x7540u + b)),
                                         __uint_as_float(__byte_perm(f[s + 1], 0x4B000000u, 0x7540u + b)));
            const float2 v = __fmul2_rn(__fadd2_rn(__fadd2_rn(q, nm), nz), d2);
            const __half2 h = __floats2half2_rn(v.x, v.y);
            out[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// grid (row blocks, split): CTA (x, y) takes rows 128 x .. and a range of the cols / 64 column
// tiles: tq + 1 tiles for y < tr, else tq, ranges in order of y (tq >= 1).  G32: the group size is
// a multiple of 32, so the 32 codes a thread dequantizes per tile share one group.
template <int NB, bool G32>
__global__ void __launch_bounds__(kGmThreads, 2)
hqq_gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                   const __half *__restrict__ scale, const __half *__restrict__ zero, int64_t rows,
                   int64_t cols, int g, int batch, int np, int stages, int gpad, int tq, int tr, int split,
                   float *__restrict__ Y) {
    extern __shared__ unsigned char smem_raw[];
    constexpr int kRowBytes = 8 * NB;                   // packed bytes of one tile row (64 codes)
    constexpr int kChunkTiles = kGmChunkRow / kRowBytes;  // tiles per code chunk: 4 or 8
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rbase = (int64_t)blockIdx.x * kGmM;
    const int y = (int)blockIdx.y;
    const int kt_beg = y * tq + min(y, tr);
    const int ntile = tq + (y < tr ? 1 : 0);
    const int nchunk = (ntile + kChunkTiles - 1) / kChunkTiles;
    const GemmLayout L(np, stages, gpad);
    const uint32_t s_base = ((uint32_t)__cvta_generic_to_shared(smem_raw) + 1023u) & ~1023u;
    const uint32_t c_base = s_base + L.c_off, x_base = s_base + L.x_off;
    const uint32_t m_base = s_base + L.m_off;
    const uint32_t cfull0 = s_base + L.bar_off, cempty0 = cfull0 + 16;
    const uint32_t xfull0 = cempty0 + 16, xempty0 = xfull0 + 8 * stages;
    const uint32_t afull0 = xempty0 + 8 * stages, aempty0 = afull0 + 8 * kGmLag;
    const uint32_t done = aempty0 + 8 * kGmLag, tslot = done + 8;
    // tensor memory: the accumulator in columns [0, np), then kGmLag A buffers of 32 columns (one
    // tile row of 64 fp16 values per lane)
    const uint32_t a_col = (uint32_t)(np + 31) / 32 * 32;
    const uint32_t need = a_col + 32 * kGmLag;
    const uint32_t ncols = need <= 32 ? 32u : need <= 64 ? 64u : need <= 128 ? 128u : need <= 256 ? 256u : 512u;

    if (tid == 0) {
        for (int c = 0; c < 2; ++c) {
            mbar_init(cfull0 + 8 * c, 1);               // the copy lane's arrival + the chunk's bytes
            mbar_init(cempty0 + 8 * c, kGmDeqThreads);  // every dequantization thread is done with it
        }
        for (int s = 0; s < stages; ++s) {
            mbar_init(xfull0 + 8 * s, 1);   // the copy lane's arrival + the X tile's bytes
            mbar_init(xempty0 + 8 * s, 1);  // the tile's MMAs have completed
        }
        for (int a = 0; a < kGmLag; ++a) {
            mbar_init(afull0 + 8 * a, kGmDeqThreads);  // every dequantization thread has stored
            mbar_init(aempty0 + 8 * a, 1);             // the MMAs reading the buffer have completed
        }
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kGmMmaWarp) {  // the whole warp allocates the accumulator's columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tslot), "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tslot));

    bool ok = true;
    if (warp == kGmCopyWarp) {
        // the scale and zero-point loads go out first: the first tile needs them as much as its codes
        asm volatile("bar.sync 2, %0;" ::"n"(kGmDeqThreads + 32) : "memory");
        if (lane == 0) {
            int s = 0, xr = 0;  // X slot of tile j, and j / S
            for (int j = 0; j < ntile; ++j) {
                if (j % kChunkTiles == 0) {  // the chunk of tiles j .. j + kChunkTiles - 1
                    const int c = j / kChunkTiles, b = c & 1;
                    // the buffer's previous chunk (c - 2) has been dequantized
                    if (c >= 2) ok &= mbar_wait(cempty0 + 8 * b, (uint32_t)((c >> 1) - 1) & 1u);
                    mbar_expect_tx(cfull0 + 8 * b, (uint32_t)kGmChunkBytes);
                    tma_load_2d(c_base + (uint32_t)(b * kGmChunkBytes), &tm_codes, (kt_beg + j) * kRowBytes, (int)rbase, cfull0 + 8 * b);
                }
                // the slot's previous X tile (j - S) has been read by its MMAs
                if (xr > 0) ok &= mbar_wait(xempty0 + 8 * s, (uint32_t)(xr - 1) & 1u);
                mbar_expect_tx(xfull0 + 8 * s, (uint32_t)L.x_bytes);
                tma_load_2d(x_base + (uint32_t)(s * L.x_bytes), &tm_x, (kt_beg + j) * kGmK, 0, xfull0 + 8 * s);
                if (++s == stages) { s = 0; ++xr; }
            }
            // the last loads in flight have landed (they have, unless a wait above ran out)
            for (int j = ntile > stages ? ntile - stages : 0; j < ntile; ++j)
                mbar_wait(xfull0 + 8 * (j % stages), (uint32_t)(j / stages) & 1u);
            for (int c = nchunk > 2 ? nchunk - 2 : 0; c < nchunk; ++c)
                mbar_wait(cfull0 + 8 * (c & 1), (uint32_t)(c >> 1) & 1u);
        }
        __syncwarp();
    } else if (warp == kGmMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_f16(np);
            int s = 0, ph = 0, a = 0, ua = 0;
            for (int u = 0; u < ntile; ++u) {
                ok &= mbar_wait(afull0 + 8 * a, (uint32_t)ua & 1u);  // A buffer a holds tile u
                ok &= mbar_wait(xfull0 + 8 * s, (uint32_t)ph);       // X tile u has landed
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                if (ok) {
                    const uint32_t ta = tmem + a_col + 32u * (uint32_t)a;
                    const uint32_t sb = x_base + (uint32_t)(s * L.x_bytes);
#pragma unroll
                    for (int j = 0; j < kGmK / 16; ++j) {
                        // A: K = 16 is 8 tensor-memory columns; B: 32 bytes along the swizzled row
                        const uint64_t db = umma_desc(sb + (uint32_t)j * 32u, 16, 1024, 2);
                        const uint32_t acc = (u > 0 || j > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                            ::"r"(tmem), "r"(ta + 8u * (uint32_t)j), "l"(db), "r"(idesc), "r"(acc)
                            : "memory");
                    }
                }
                umma_commit(xempty0 + 8 * s);  // frees the X slot once these MMAs complete
                umma_commit(aempty0 + 8 * a);  // and the A buffer
                if (++a == kGmLag) { a = 0; ++ua; }
                if (++s == stages) { s = 0; ph ^= 1; }
            }
            umma_commit(done);
        }
        __syncwarp();
    } else {
        // ---- dequantization warps.  The scales and zero points of the CTA's rows and groups, as
        // binary32 (z, Delta) pairs; (0, 0) for rows past the matrix, whose codes read as zero.
        // Thread (m, h) fetches row m's groups h, h + 2, .. (at most 16 groups per range).
        // column offsets are below 2^31: 32-bit arithmetic
        const int gbeg = kt_beg * kGmK / g;                            // first group of the range
        const int gcta = ((kt_beg + ntile) * kGmK - 1) / g - gbeg + 1;  // <= gpad
        const int64_t gpr = (int64_t)((int)cols / g);                   // groups per row
        const int m = tid & (kGmM - 1), half = tid >> 7;  // this thread's row and half of a tile
        {
            const bool live = rbase + m < rows;
            const __half *zr = zero + (rbase + m) * gpr + gbeg, *sr = scale + (rbase + m) * gpr + gbeg;
            __half zv[kGmMaxGroups / 2], sv[kGmMaxGroups / 2];
#pragma unroll
            for (int j = 0; j < kGmMaxGroups / 2; ++j) {
                const int gi = half + 2 * j;
                zv[j] = sv[j] = __float2half_rn(0.0f);
                if (live && gi < gcta) {
                    zv[j] = __ldg(zr + gi);
                    sv[j] = __ldg(sr + gi);
                }
            }
            asm volatile("bar.arrive 2, %0;" ::"n"(kGmDeqThreads + 32) : "memory");  // loads issued
#pragma unroll
            for (int j = 0; j < kGmMaxGroups / 2; ++j) {
                const int gi = half + 2 * j;
                if (gi < gcta)
                    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(m_base + (uint32_t)(m * gpad + gi) * 8u),
                                 "f"(__half2float(zv[j])), "f"(__half2float(sv[j])) : "memory");
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kGmDeqThreads) : "memory");  // the table is complete
        }
        // this thread's 16 columns of an A buffer: lane m (warp w reaches lanes 32 (w mod 4) ..)
        const uint32_t a_thr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + a_col + 16u * (uint32_t)half;
        const uint32_t m_row = m_base + (uint32_t)(m * gpad) * 8u;
        // row m of a chunk buffer: 8 pieces of 16 bytes, piece p stored at (p ^ (m mod 8)) * 16
        const uint32_t c_row = c_base + (uint32_t)m * kGmChunkRow;
        // the group of this thread's next chunk: column col (relative to the range), local group
        // gi, first column of the next group bound (a range spans 16 groups of <= 256 columns)
        int col = 32 * half;
        int gi = (kt_beg * kGmK + col) / g - gbeg;
        int bound = (gbeg + gi + 1) * g - kt_beg * kGmK;
        int a = 0, ua = 0, t_in = 0, cb = 0, cr = 0;  // A buffer, u / lag, tile within chunk, chunk buffer, chunk / 2
        for (int u = 0; u < ntile; ++u) {
            if (t_in == 0) ok &= mbar_wait(cfull0 + 8 * cb, (uint32_t)cr & 1u);          // chunk landed
            if (u >= kGmLag) ok &= mbar_wait(aempty0 + 8 * a, (uint32_t)(ua - 1) & 1u);  // A free
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            uint32_t words[NB == 4 ? 4 : 2];
            if constexpr (NB == 4) {  // 32 bytes: piece 2 t_in + half
                const uint32_t cs = c_row + (uint32_t)cb * kGmChunkBytes + (uint32_t)(((2 * t_in + half) ^ (m & 7)) * 16);
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(words[0]), "=r"(words[1]), "=r"(words[2]), "=r"(words[3]) : "r"(cs) : "memory");
            } else {  // 16 bytes: half of piece t_in
                const uint32_t cs = c_row + (uint32_t)cb * kGmChunkBytes + (uint32_t)((t_in ^ (m & 7)) * 16 + half * 8);
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(words[0]), "=r"(words[1]) : "r"(cs) : "memory");
            }
            uint32_t av[16];  // fp16 pairs: codes 32 half + 2 i, + 2 i + 1 in word i
            float zf = 0.0f, df = 0.0f;
            if constexpr (G32) {
                while (col >= bound) {  // warp-uniform: every lane of a warp has the same half
                    ++gi;
                    bound += g;
                }
                asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(zf), "=f"(df) : "r"(m_row + (uint32_t)gi * 8u) : "memory");
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if constexpr (!G32) {
                    while (col + 8 * c >= bound) {
                        ++gi;
                        bound += g;
                    }
                    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(zf), "=f"(df) : "r"(m_row + (uint32_t)gi * 8u) : "memory");
                }
                const uint32_t bits = NB == 4 ? words[c] : (words[c >> 1] >> (16 * (c & 1))) & 0xFFFFu;
                const uint4 v = dequant_chunk<NB>(bits, zf, df);
                av[4 * c] = v.x;
                av[4 * c + 1] = v.y;
                av[4 * c + 2] = v.z;
                av[4 * c + 3] = v.w;
            }
            col += kGmK;
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
                ::"r"(a_thr + 32u * (uint32_t)a), "r"(av[0]), "r"(av[1]), "r"(av[2]), "r"(av[3]), "r"(av[4]), "r"(av[5]),
                  "r"(av[6]), "r"(av[7]), "r"(av[8]), "r"(av[9]), "r"(av[10]), "r"(av[11]), "r"(av[12]), "r"(av[13]),
                  "r"(av[14]), "r"(av[15]) : "memory");
            // the stores have completed and are ordered before the MMAs; then this thread's part is ready
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(afull0 + 8 * a);
            if (++a == kGmLag) { a = 0; ++ua; }
            if (++t_in == kChunkTiles || u == ntile - 1) {  // done with this chunk's codes
                mbar_arrive(cempty0 + 8 * cb);
                t_in = 0;
                if (++cb == 2) { cb = 0; ++cr; }
            }
        }
    }
    // a wait that ran out anywhere poisons the CTA's outputs
    ok = __syncthreads_and(ok) != 0;
    if (warp < kGmDeqThreads / 32) {
        if (ok) ok = mbar_wait(done, 0u);  // every MMA of this CTA has completed
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // Y may still be being zeroed by the kernel launched before this one
        wait_prerequisite();
        const int wq = warp & 3, cw = np / 2;  // lanes 32 wq ..: rows of W; half the columns each
        const int64_t row = rbase + 32 * wq + lane;
        for (int c0 = (warp >> 2) * cw; c0 < (warp >> 2) * cw + cw; c0 += 8) {
            uint32_t v[8];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                         : "r"(tmem + ((uint32_t)(32 * wq) << 16) + (uint32_t)c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            if (row < rows) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int n = c0 + i;
                    if (n < batch) {
                        const float y = ok ? __uint_as_float(v[i]) : __int_as_float(0x7fc00000);
                        if (split > 1) atomicAdd(Y + (int64_t)n * rows + row, y);
                        else Y[(int64_t)n * rows + row] = y;
                    }
                }
            }
        }
    }
    allow_dependents();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == kGmMmaWarp) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

__global__ void __launch_bounds__(256) hqq_zero_f32_kernel(float *__restrict__ y, int64_t n) {
    allow_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = 0.0f;
}

// most groups of one row that a CTA's column range touches, over the split's ranges
int64_t max_groups(int64_t tiles, int64_t split, int64_t g) {
    int64_t worst = 0;
    const int64_t lo = tiles / split, hi = (tiles + split - 1) / split;
    // a range of n tiles starting at column c touches (c + 64 n - 1) / g - c / g + 1 groups; a
    // range's start is a multiple of 64, and the count repeats with period lcm(64, g) <= 64 g
    for (int64_t n = lo; n <= hi; ++n)
        for (int64_t c = 0; c < g * kGmK && c < tiles * kGmK; c += kGmK)
            worst = std::max(worst, (c + kGmK * n - 1) / g - c / g + 1);
    return worst;
}

struct GemmConfig {
    int split, stages, gpad, smem;
};

// split and ring depth for one launch: enough CTAs to fill the SMs in one wave (two per SM where
// a ring of four X slots fits beside the rest), each CTA's groups within the table, as many X
// slots as fit
template <int NB>
GemmConfig gemm_config(int64_t rows, int64_t cols, int g, int np, int sms, int smem_sm, int smem_cta) {
    const int64_t row_blocks = (rows + kGmM - 1) / kGmM, tiles = cols / kGmK;
    GemmConfig c{};
    for (int per_sm = 2; per_sm >= 1; --per_sm) {
        const int budget = per_sm == 2 ? smem_sm / 2 - 1024 : smem_cta;
        const int64_t want = (int64_t)sms * per_sm / row_blocks;  // one wave at most
        int64_t split = std::min<int64_t>(std::max<int64_t>(want, 1), tiles);
        while (split < tiles && max_groups(tiles, split, g) > kGmMaxGroups) ++split;
        c.split = (int)split;
        c.gpad = (int)(max_groups(tiles, split, g) | 1);
        int stages = kGmMaxStages;
        while (stages > 2 && GemmLayout(np, stages, c.gpad).total > budget) --stages;
        c.stages = stages;
        c.smem = GemmLayout(np, stages, c.gpad).total;
        if (per_sm == 2 && stages >= 4 && c.smem <= budget) {
            // no third CTA on an SM: two take the tensor memory
            c.smem = std::max(c.smem, smem_sm / 3 + 1024);
            break;
        }
    }
    return c;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// tensor maps of the packed codes (bytes, rows x cols NB / 8; box 128 rows x 128 bytes, past the
// matrix read as 0) and of one launch's X (fp16, nb x cols; box np x 64; rows past nb read 0),
// both with the 128-byte swizzle
template <int NB>
cudaError_t gemm_maps(const uint8_t *pk, int64_t rows, int64_t cols, const __half *X, int nb, int np,
                      CUtensorMap *mc, CUtensorMap *mx) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t cdim[2] = {(cuuint64_t)(cols * NB / 8), (cuuint64_t)rows};
    const cuuint64_t cstride[1] = {(cuuint64_t)(cols * NB / 8)};
    const cuuint32_t cbox[2] = {(cuuint32_t)kGmChunkRow, (cuuint32_t)kGmM};
    const cuuint32_t unit[2] = {1, 1};
    if (enc(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(pk), cdim, cstride, cbox, unit,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const cuuint64_t xdim[2] = {(cuuint64_t)cols, (cuuint64_t)nb};
    const cuuint64_t xstride[1] = {(cuuint64_t)(cols * 2)};
    const cuuint32_t xbox[2] = {(cuuint32_t)kGmK, (cuuint32_t)np};
    if (enc(mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half *>(X), xdim, xstride, xbox, unit,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

template <int NB>
cudaError_t launch_gemm_tc_cfg(const uint8_t *pk, const __half *sc, const __half *ze, int64_t rows,
                               int64_t cols, int g, const __half *X, int nb, float *Y,
                               const GemmConfig &c, int sms, cudaStream_t st) {
    const int np = (nb + 15) / 16 * 16;
    const int64_t row_blocks = (rows + kGmM - 1) / kGmM;
    CUtensorMap mc, mx;
    cudaError_t e = gemm_maps<NB>(pk, rows, cols, X, nb, np, &mc, &mx);
    if (e != cudaSuccess) return e;
    auto k = g % 32 == 0 ? hqq_gemm_tc_kernel<NB, true> : hqq_gemm_tc_kernel<NB, false>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, c.smem);
    if (e != cudaSuccess) return e;
    if (c.split > 1) {
        const int64_t n = (int64_t)nb * rows;
        hqq_zero_f32_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4 * sms), 256, 0, st>>>(Y, n);
    }
    // the launch overlaps the zeroing kernel only; without a split it waits for the stream
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)row_blocks, (unsigned)c.split);
    cfg.blockDim = dim3(kGmThreads);
    cfg.dynamicSmemBytes = (size_t)c.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = c.split > 1 ? 1 : 0;
    const int tiles = (int)(cols / kGmK);
    return cudaLaunchKernelEx(&cfg, k, mc, mx, sc, ze, rows, cols, g, nb, np, c.stages, c.gpad,
                              tiles / c.split, tiles % c.split, c.split, Y);
}

template <int NB>
cudaError_t launch_gemm_tc_nb(const uint8_t *pk, const __half *sc, const __half *ze, int64_t rows,
                              int64_t cols, int g, const __half *X, int64_t batch, float *Y,
                              cudaStream_t st) {
    int dev = 0, sms = 148, smem_sm = 233472, smem_cta = 232448;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&smem_cta, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    }
    for (int64_t b0 = 0; b0 < batch; b0 += kGmMaxBatch) {
        const int nb = (int)std::min<int64_t>(kGmMaxBatch, batch - b0);
        const GemmConfig c = gemm_config<NB>(rows, cols, g, (nb + 15) / 16 * 16, sms, smem_sm, smem_cta);
        cudaError_t e = launch_gemm_tc_cfg<NB>(pk, sc, ze, rows, cols, g, X + b0 * cols, nb, Y + b0 * rows, c, sms, st);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace

namespace hqq_impl {

bool gemm_tc_layout(int nbits, int64_t rows, int64_t cols, int64_t g, int axis, const void *X) {
    // groups must not cross rows (cols % g == 0): the kernel finds a chunk's group by row; the
    // tensor maps take 32-bit coordinates
    return axis == 1 && (nbits == 2 || nbits == 4) && g % 8 == 0 && cols % kGmK == 0 && cols % g == 0 &&
           rows > 0 && rows < (int64_t(1) << 31) && cols < (int64_t(1) << 31) && ((uintptr_t)X & 15) == 0;
}

cudaError_t launch_gemm_tc(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                           int64_t rows, int64_t cols, int64_t g, const __half *X, int64_t batch,
                           float *Y, cudaStream_t st) {
    return nbits == 4 ? launch_gemm_tc_nb<4>(pk, sc, ze, rows, cols, (int)g, X, batch, Y, st)
                      : launch_gemm_tc_nb<2>(pk, sc, ze, rows, cols, (int)g, X, batch, Y, st);
}

}  // namespace hqq_impl
