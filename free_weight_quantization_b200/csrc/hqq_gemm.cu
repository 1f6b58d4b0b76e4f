// hqq_gemm.cu -- the quantized layer's forward product for a batch of input vectors on the B200
// tensor cores [HQQ 算法解读, "从压缩文件到一次前向", and its `axis` table row "追求低 batch 推理吞吐"]:
//     Y[b, r] = sum_c W_hat[r, c] * X[b, c]
// with W_hat[r, c] exactly the fp16 value hqq_dequantize writes (q - z) * Delta.
//
// Fast path (axis 1, 2- or 4-bit codes, group size a multiple of 8 dividing cols, cols a
// multiple of 64):
//   a CTA owns 128 rows of W (the M of one tcgen05.mma) and a range of columns (split-K, so
//   that the grid covers the SMs).  Its 256 threads dequantize the codes of a 128 x 64 tile
//   into fp16 in shared memory, in the canonical K-major layout without swizzle (8-row x 16-byte
//   core matrices: core (k8, m8) at byte (k8 * M/8 + m8) * 128), and copy the batch's 64
//   columns of X beside it in the same layout.  One elected thread then issues four
//   tcgen05.mma.cta_group::1.kind::f16 (K = 16 each) that accumulate D = W_hat_tile X_tile^T in
//   binary32 in tensor memory (128 lanes = rows, one column per batch entry), and commits them
//   to the stage's mbarrier.  Two stages alternate, so one tile is dequantized while the tensor
//   cores work on the other.  At the end each warp of the first four reads its 32 lanes with
//   tcgen05.ld and adds them into Y (atomically when the columns are split over CTAs; Y is
//   zeroed by a small kernel launched before).
// Every product of two fp16 values is exact in binary32, and the tensor cores accumulate them in
// binary32, so Y is within cols * 2^-23 * sum_c |W_hat X| of the exact sum whatever the order.
// Every other layout runs the generic forward product once per batch entry.
//
// Waits on mbarriers are bounded: a wait that runs out (it never should) writes NaN into the
// CTA's outputs, so that a wrong result cannot pass silently, and the kernel still frees its
// tensor memory and returns.
#include <algorithm>

#include "hqq_common.cuh"

namespace {

constexpr int kGmM = 128;         // rows of W per CTA: the M of one MMA
constexpr int kGmK = 64;          // columns per stage: four MMAs of K = 16
constexpr int kGmThreads = 256;
constexpr int kGmStages = 2;
constexpr int kGmMaxBatch = 256;  // the N of one MMA at most
constexpr uint32_t kGmWaitLimit = 1u << 22;

// shared-memory layout of a CTA: [stage][A tile | B tile], then two mbarriers and the
// tensor-memory address
struct GemmSmem {
    static __host__ __device__ int a_bytes() { return kGmM * kGmK * 2; }
    static __host__ __device__ int b_bytes(int np) { return np * kGmK * 2; }
    static __host__ __device__ int stage_bytes(int np) { return a_bytes() + b_bytes(np); }
    static __host__ __device__ int bytes(int np) { return kGmStages * stage_bytes(np) + 64; }
};

// tcgen05 shared-memory matrix descriptor: start address, leading-dimension byte offset (between
// the two core matrices along K), stride byte offset (between 8-row groups), all in 16-byte
// units; descriptor version 1; no swizzle
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// instruction descriptor of kind::f16: D binary32, A and B fp16, both K-major, M = 128, N = np
__host__ __device__ constexpr uint32_t umma_idesc_f16(int np) {
    return (1u << 4) | ((uint32_t)(np >> 3) << 17) | ((uint32_t)(kGmM >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}

// bounded wait for the phase with the given parity; false if it did not complete in time
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
    for (uint32_t i = 0; i < kGmWaitLimit; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred P1;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, P1;\n\t}"
            : "=r"(ok)
            : "r"(addr), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
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

template <int NB>
__global__ void __launch_bounds__(kGmThreads, 1)
hqq_gemm_tc_kernel(const uint8_t *__restrict__ packed, const __half *__restrict__ scale,
                   const __half *__restrict__ zero, int64_t rows, int64_t cols, int g,
                   const __half *__restrict__ X, int batch, int np, int tiles_per_cta,
                   float *__restrict__ Y, int split) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rbase = (int64_t)blockIdx.x * kGmM;
    const int64_t kt0 = (int64_t)blockIdx.y * tiles_per_cta;
    const int stage_bytes = GemmSmem::stage_bytes(np);
    const uint32_t s_base = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t bar0 = s_base + kGmStages * stage_bytes;          // two 8-byte mbarriers
    const uint32_t tslot = bar0 + 16;                                  // tensor-memory address
    const uint32_t ncols = np <= 32 ? 32u : np <= 64 ? 64u : np <= 128 ? 128u : 256u;
    const uint32_t idesc = umma_idesc_f16(np);
    const uint32_t lbo_a = (kGmM / 8) * 128, lbo_b = (uint32_t)(np / 8) * 128, sbo = 128;

    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {  // the whole warp allocates the accumulator's columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tslot), "r"(ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t tmem;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(tmem) : "r"(tslot));

    const int m = tid & (kGmM - 1), half = tid >> 7;  // this thread's row and half of the tile
    const int64_t r = rbase + m;
    const int64_t gpr = cols / g;                      // groups per row
    bool ok = true;
    for (int t = 0; t < tiles_per_cta; ++t) {
        const int st = t & 1;
        const uint32_t sa = s_base + st * stage_bytes, sb = sa + GemmSmem::a_bytes();
        // the stage's previous MMAs (tile t - 2) have read its buffers
        if (t >= 2) ok = ok && mbar_wait(bar0 + 8 * st, (uint32_t)((t - 2) >> 1) & 1u);
        const int64_t k0 = (kt0 + t) * kGmK;
        // ---- W_hat tile: this thread's row, chunks k8 = 4 half .. 4 half + 3 (32 codes)
        {
            uint32_t words[NB == 4 ? 4 : 2];
            if (r < rows) {
                const uint8_t *src = packed + (r * cols + k0 + 32 * half) * NB / 8;
                if constexpr (NB == 4) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src));
                    words[0] = v.x; words[1] = v.y; words[2] = v.z; words[3] = v.w;
                } else {
                    const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
                    words[0] = v.x; words[1] = v.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < (NB == 4 ? 4 : 2); ++i) words[i] = 0u;
            }
            int64_t gk = -1;
            float zf = 0.0f, df = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int k8 = 4 * half + c;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (r < rows) {
                    const int64_t k = r * gpr + (k0 + 8 * k8) / g;  // the chunk's group
                    if (k != gk) {
                        gk = k;
                        zf = __half2float(__ldg(zero + k));
                        df = __half2float(__ldg(scale + k));
                    }
                    const uint32_t bits = NB == 4 ? words[c] : (words[c >> 1] >> (16 * (c & 1))) & 0xFFFFu;
                    v = dequant_chunk<NB>(bits, zf, df);
                }
                const uint32_t dst = sa + (uint32_t)(k8 * (kGmM / 8) + (m >> 3)) * 128u + (uint32_t)(m & 7) * 16u;
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
            }
        }
        // ---- X tile: np rows (batch entries, zero past the batch) x 64 columns
        for (int c = tid; c < np * 8; c += kGmThreads) {
            const int n = c >> 3, k8 = c & 7;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (n < batch) v = __ldg(reinterpret_cast<const uint4 *>(X + (int64_t)n * cols + k0 + 8 * k8));
            const uint32_t dst = sb + (uint32_t)(k8 * (np / 8) + (n >> 3)) * 128u + (uint32_t)(n & 7) * 16u;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
        }
        // the generic-proxy stores become visible to the tensor cores' (async proxy) reads
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0 && ok) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int j = 0; j < kGmK / 16; ++j) {
                const uint64_t da = umma_desc(sa + (uint32_t)j * 2u * lbo_a, lbo_a, sbo);
                const uint64_t db = umma_desc(sb + (uint32_t)j * 2u * lbo_b, lbo_b, sbo);
                const uint32_t acc = (t > 0 || j > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                    ::"r"(tmem), "l"(da), "l"(db), "r"(idesc), "r"(acc)
                    : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(bar0 + 8 * st) : "memory");
        }
    }
    // every MMA of this CTA has completed once the last stage's commit has
    const int tl = tiles_per_cta - 1;
    ok = ok && mbar_wait(bar0 + 8 * (tl & 1), (uint32_t)(tl >> 1) & 1u);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // Y may still be being zeroed by the kernel launched before this one
    wait_prerequisite();
    if (warp < 4) {  // warp w reads tensor-memory lanes 32 w .. 32 w + 31: rows of W
        const int64_t row = rbase + 32 * warp + lane;
        for (int c0 = 0; c0 < np; c0 += 8) {
            uint32_t v[8];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                         : "r"(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0));
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
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols));
    }
}

__global__ void __launch_bounds__(256) hqq_zero_f32_kernel(float *__restrict__ y, int64_t n) {
    allow_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = 0.0f;
}

template <int NB>
cudaError_t launch_gemm_tc_nb(const uint8_t *pk, const __half *sc, const __half *ze, int64_t rows,
                           int64_t cols, int g, const __half *X, int64_t batch, float *Y,
                           cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t row_blocks = (rows + kGmM - 1) / kGmM;
    const int64_t tiles = cols / kGmK;
    for (int64_t b0 = 0; b0 < batch; b0 += kGmMaxBatch) {
        const int nb = (int)std::min<int64_t>(kGmMaxBatch, batch - b0);
        const int np = (nb + 15) / 16 * 16;
        const int smem = GemmSmem::bytes(np);
        auto k = hqq_gemm_tc_kernel<NB>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        // split the columns so that the grid covers the SMs; the split must divide the tiles
        int64_t split = 1;
        while (row_blocks * split * 2 <= sms && tiles % (split * 2) == 0 && tiles / (split * 2) >= 2) split *= 2;
        float *Yb = Y + b0 * rows;
        if (split > 1) {
            const int64_t n = (int64_t)nb * rows;
            hqq_zero_f32_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4 * sms), 256, 0, st>>>(Yb, n);
        }
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)row_blocks, (unsigned)split);
        cfg.blockDim = dim3(kGmThreads);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k, pk, sc, ze, rows, cols, g, X + b0 * cols, nb, np,
                               (int)(tiles / split), Yb, (int)split);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace

namespace hqq_impl {

bool gemm_tc_layout(int nbits, int64_t rows, int64_t cols, int64_t g, int axis, const void *X) {
    // groups must not cross rows (cols % g == 0): the kernel finds a chunk's group by row
    return axis == 1 && (nbits == 2 || nbits == 4) && g % 8 == 0 && cols % kGmK == 0 && cols % g == 0 &&
           rows > 0 && ((uintptr_t)X & 15) == 0;
}

cudaError_t launch_gemm_tc(int nbits, const uint8_t *pk, const __half *sc, const __half *ze,
                           int64_t rows, int64_t cols, int64_t g, const __half *X, int64_t batch,
                           float *Y, cudaStream_t st) {
    return nbits == 4 ? launch_gemm_tc_nb<4>(pk, sc, ze, rows, cols, (int)g, X, batch, Y, st)
                      : launch_gemm_tc_nb<2>(pk, sc, ze, rows, cols, (int)g, X, batch, Y, st);
}

}  // namespace hqq_impl
