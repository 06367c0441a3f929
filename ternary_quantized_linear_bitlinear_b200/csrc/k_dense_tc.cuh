// Backward of the quantization-aware BitLinear, weight gradient, with the
// straight-through estimator and the hard or soft STE scale ("Distillix"
// README, 1. BitNet b1.58 Core: STE; "bitone" README, Soft-STE notes):
//
//   dW[n, k] = (sum_m dY[m, n] * x_q[m, k] / s[m]) * scale(W[n, k] / gamma)
//   scale(r) = |r| <= 1 ? 1 : 0                (hard, beta <= 0)
//            = 1 - tanh(beta * r)^2            (soft)
//
// with r = float(W / gamma), the forward's division.  The sum runs over the
// tokens m, which are the rows of both dY [M, N] and x_q [M, K], so two
// preparation kernels first lay both operands out with m contiguous (the
// K-major form the tensor cores read): dYt [N, Mp] = dY^T in bf16 and
// xst [K, Mp] = bf16(x_q / s)^T, zero for m >= M.  Then a dense
// tcgen05.mma.cta_group::1.kind::f16 GEMM (128 x 256 output tile per CTA,
// TMA operands in 128-byte-swizzled stages, f32 accumulators in TMEM)
// multiplies them, and its epilogue applies the scale and writes dW.
//
// Roles: warp 0 TMA producer (one thread), warp 1 TMEM allocator + MMA
// issuer (one thread), warps 2..5 epilogue (TMEM lane = row n).  Every
// mbarrier wait is bounded (globaltimer); a wait that gives up raises the
// device error word and the CTA's abort flag, the producer waits for its
// in-flight copies and the MMA thread for its last commit (both bounded)
// before TMEM is freed.
#pragma once

#include <cuda.h>

#include "bl_common.cuh"

namespace bl {

constexpr int DT_BM = 128;                   // output rows n per CTA (TMEM lanes)
constexpr int DT_BN = 256;                   // output columns k per CTA (TMEM columns)
constexpr int DT_BK = 64;                    // tokens m per stage (bf16: 128-byte rows)
constexpr int DT_STAGES = 4;
constexpr int DT_A_BYTES = DT_BM * DT_BK * 2;  // 16 KiB
constexpr int DT_B_BYTES = DT_BN * DT_BK * 2;  // 32 KiB
constexpr int DT_THREADS = 192;
constexpr int DT_OFF_B = DT_STAGES * DT_A_BYTES;
constexpr int DT_OFF_BAR = DT_OFF_B + DT_STAGES * DT_B_BYTES;
constexpr int DT_SMEM_BYTES = DT_OFF_BAR + 2 * DT_STAGES * 8 + 8 + 16 + 1024;
static_assert(DT_SMEM_BYTES <= 227 * 1024, "dense GEMM shared memory");

struct DenseParams {
    const void *W;       // latent weights [N, K] (f32 or bf16)
    int w_bf16;
    const float *gamma;
    float beta;          // <= 0: hard scale
    float *dW;           // [N, K] f32 out
    int N, K, Mp;        // Mp: padded token count (multiple of 64)
    int k_stages;
    unsigned long long timeout_ns;
};

struct DenseMaps {
    CUtensorMap a;  // dYt [N, Mp] bf16, box 64 x 128
    CUtensorMap b;  // xst [K, Mp] bf16, box 64 x 256
};

// dYt[n, m] = dY[m, n] (bf16 copy), zero for M <= m < Mp.  32 x 32 tiles.
__global__ void __launch_bounds__(256) k_dw_prep_dy(const uint16_t *__restrict__ dY, int M, int N, int Mp,
                                                     uint16_t *__restrict__ dYt) {
    __shared__ uint16_t t[32][33];
    const int m0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows per pass
    for (int r = ty; r < 32; r += 8) {
        const int m = m0 + r, n = n0 + tx;
        t[r][tx] = (m < M && n < N) ? dY[(size_t)m * N + n] : (uint16_t)0;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int n = n0 + r, m = m0 + tx;
        if (n < N && m < Mp) dYt[(size_t)n * Mp + m] = t[tx][r];
    }
}

// xst[k, m] = bf16(float(x_q[m, k]) / s[m]) (round to nearest even), zero
// for M <= m < Mp.  32 x 32 tiles.
__global__ void __launch_bounds__(256) k_dw_prep_x(const int8_t *__restrict__ x_q, const float *__restrict__ s,
                                                    int M, int K, int Mp, uint16_t *__restrict__ xst) {
    __shared__ uint16_t t[32][33];
    const int m0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) {
        const int m = m0 + r, k = k0 + tx;
        uint16_t v = 0;
        if (m < M && k < K) {
            const float q = __fdiv_rn((float)x_q[(size_t)m * K + k], s[m]);
            v = __bfloat16_as_ushort(__float2bfloat16_rn(q));
        }
        t[r][tx] = v;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int k = k0 + r, m = m0 + tx;
        if (k < K && m < Mp) xst[(size_t)k * Mp + m] = t[tx][r];
    }
}

__device__ __forceinline__ void dt_mma_f16(u32 d_tmem, unsigned long long a_desc, unsigned long long b_desc, u32 idesc,
                                           u32 accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void dt_commit(u32 bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// D f32, A bf16, B bf16, both K-major, N = DT_BN, M = DT_BM
__host__ __device__ constexpr u32 dt_idesc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((u32)(DT_BN >> 3) << 17) | ((u32)(DT_BM >> 4) << 24);
}

__device__ __forceinline__ unsigned long long dt_desc_sw128(u32 saddr) {
    unsigned long long d = 0;
    d |= (unsigned long long)((saddr >> 4) & 0x3FFFu);
    d |= (unsigned long long)1u << 16;            // leading byte offset (unused for swizzled K-major)
    d |= (unsigned long long)(1024u >> 4) << 32;  // stride byte offset: 8-row groups 1024 bytes apart
    d |= (unsigned long long)1u << 46;            // descriptor version
    d |= (unsigned long long)2u << 61;            // SWIZZLE_128B
    return d;
}

__global__ void __launch_bounds__(DT_THREADS, 1)
    k_dw_gemm(const __grid_constant__ DenseMaps maps, const __grid_constant__ DenseParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const u32 sbase = smem_u32(sm);
    const u32 bar0 = sbase + DT_OFF_BAR;
    auto BAR_FULL = [&](int s) { return bar0 + 8u * s; };
    auto BAR_EMPTY = [&](int s) { return bar0 + 8u * (DT_STAGES + s); };
    const u32 BAR_ACC = bar0 + 8u * (2 * DT_STAGES);
    u32 *s_tmem = reinterpret_cast<u32 *>(sm + DT_OFF_BAR + 2 * DT_STAGES * 8 + 8);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + DT_OFF_BAR + 2 * DT_STAGES * 8 + 12);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * DT_BM, k0 = blockIdx.y * DT_BN;
    const unsigned long long TO = p.timeout_ns;
    if (threadIdx.x == 0) {
        for (int s = 0; s < DT_STAGES; ++s) {
            mbar_init(BAR_FULL(s), 1);
            mbar_init(BAR_EMPTY(s), 1);
        }
        mbar_init(BAR_ACC, 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.a) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.b) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(DT_BN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const u32 tmem = *s_tmem;
    const int KS = p.k_stages;

    if (warp == 0) {
        if (lane == 0) {
            bool failed = false;
            int ks = 0;
            for (; ks < KS; ++ks) {
                const int s = ks % DT_STAGES;
                if (ks >= DT_STAGES &&
                    !mbar_wait(BAR_EMPTY(s), (u32)(((ks / DT_STAGES) & 1) ^ 1), TO, s_abort)) {
                    failed = true;
                    break;
                }
                mbar_arrive_expect_tx(BAR_FULL(s), DT_A_BYTES + DT_B_BYTES);
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                    ::"r"(sbase + s * DT_A_BYTES), "l"(&maps.a), "r"(ks * DT_BK), "r"(n0), "r"(BAR_FULL(s))
                    : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                    ::"r"(sbase + DT_OFF_B + s * DT_B_BYTES), "l"(&maps.b), "r"(ks * DT_BK), "r"(k0), "r"(BAR_FULL(s))
                    : "memory");
            }
            if (failed) {
                raise_device_error(DEVERR_TIMEOUT_PRODUCER);
                *s_abort = 1;
            }
            // the last copies issued land before the CTA exits
            for (int j = ks - DT_STAGES; j < ks; ++j)
                if (j >= 0) mbar_wait(BAR_FULL(j % DT_STAGES), (u32)((j / DT_STAGES) & 1), TO, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const u32 idesc = dt_idesc();
            bool failed = false, issued = false;
            for (int ks = 0; ks < KS; ++ks) {
                const int s = ks % DT_STAGES;
                if (!mbar_wait(BAR_FULL(s), (u32)((ks / DT_STAGES) & 1), TO, s_abort)) {
                    failed = true;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const u32 as = sbase + s * DT_A_BYTES, bs = sbase + DT_OFF_B + s * DT_B_BYTES;
#pragma unroll
                for (int kk = 0; kk < DT_BK / 16; ++kk)
                    dt_mma_f16(tmem, dt_desc_sw128(as + kk * 32), dt_desc_sw128(bs + kk * 32), idesc,
                               (ks | kk) != 0 ? 1u : 0u);
                dt_commit(BAR_EMPTY(s));
                issued = true;
            }
            dt_commit(BAR_ACC);  // completes once every MMA issued so far has completed
            if (failed) {
                raise_device_error(DEVERR_TIMEOUT_MMA);
                *s_abort = 1;
                // drain: the MMAs already issued complete before TMEM is freed
                if (issued) mbar_wait(BAR_ACC, 0, TO, nullptr);
            }
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int q = warp & 3;                  // TMEM lane quarter
        const int n = n0 + q * 32 + lane;        // this thread's output row
        const float gamma = *p.gamma;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(BAR_ACC, 0, TO, s_abort));
        if (!ok) {
            if (lane == 0) {
                raise_device_error(DEVERR_TIMEOUT_EPILOGUE);
                *s_abort = 1;
            }
        } else {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
            for (int c0 = 0; c0 < DT_BN; c0 += 32) {
                u32 r[32];
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                    "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                    "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                    : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                      "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                      "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                    : "r"(tmem + ((u32)(q * 32) << 16) + (u32)c0)
                    : "memory");
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int k = k0 + c0 + j;
                        if (k >= p.K) break;
                        const size_t idx = (size_t)n * p.K + k;
                        const float w = p.w_bf16 ? __uint_as_float((u32)reinterpret_cast<const uint16_t *>(p.W)[idx] << 16)
                                                 : reinterpret_cast<const float *>(p.W)[idx];
                        const float rr = __fdiv_rn(w, gamma);
                        float sc;
                        if (p.beta <= 0.f) {
                            sc = fabsf(rr) <= 1.f ? 1.f : 0.f;
                        } else {
                            const float th = tanhf(__fmul_rn(p.beta, rr));
                            sc = __fsub_rn(1.f, __fmul_rn(th, th));
                        }
                        p.dW[idx] = __fmul_rn(__uint_as_float(r[j]), sc);
                    }
                }
                __syncwarp();
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(DT_BN) : "memory");
    }
}

}  // namespace bl

// ===========================================================================
// Host side

namespace bl {

inline size_t dw_mp(int64_t M) { return (size_t)((M + 63) / 64 * 64); }

inline size_t dw_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    const size_t mp = dw_mp(M);
    return ((size_t)N * mp * 2 + 255) / 256 * 256 + ((size_t)K * mp * 2 + 255) / 256 * 256;
}

inline cudaError_t dense_setup() {
    return cudaFuncSetAttribute(k_dw_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, DT_SMEM_BYTES);
}

template <typename EncFn>
inline bl_status dw_launch(EncFn enc, const void *dY, const int8_t *x_q, const float *s, const void *W, bool w_bf16,
                           const float *gamma, float beta, int64_t M, int64_t N, int64_t K, void *ws, float *dW,
                           cudaStream_t st) {
    const int64_t Mp = (int64_t)dw_mp(M);
    uint16_t *dYt = reinterpret_cast<uint16_t *>(ws);
    uint16_t *xst = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(ws) +
                                                 ((size_t)N * Mp * 2 + 255) / 256 * 256);
    const dim3 g1((unsigned)((Mp + 31) / 32), (unsigned)((N + 31) / 32));
    k_dw_prep_dy<<<g1, 256, 0, st>>>(reinterpret_cast<const uint16_t *>(dY), (int)M, (int)N, (int)Mp, dYt);
    const dim3 g2((unsigned)((Mp + 31) / 32), (unsigned)((K + 31) / 32));
    k_dw_prep_x<<<g2, 256, 0, st>>>(x_q, s, (int)M, (int)K, (int)Mp, xst);
    if (cudaGetLastError() != cudaSuccess) return BL_ERR_CUDA;
    DenseMaps maps;
    memset(&maps, 0, sizeof(maps));
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)Mp, (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)Mp * 2};
        const cuuint32_t box[2] = {(cuuint32_t)DT_BK, (cuuint32_t)DT_BM};
        if (enc(&maps.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dYt, gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)Mp, (cuuint64_t)K};
        const cuuint64_t gstride[1] = {(cuuint64_t)Mp * 2};
        const cuuint32_t box[2] = {(cuuint32_t)DT_BK, (cuuint32_t)DT_BN};
        if (enc(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xst, gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    DenseParams p;
    p.W = W;
    p.w_bf16 = w_bf16 ? 1 : 0;
    p.gamma = gamma;
    p.beta = beta;
    p.dW = dW;
    p.N = (int)N;
    p.K = (int)K;
    p.Mp = (int)Mp;
    p.k_stages = (int)(Mp / DT_BK);
    p.timeout_ns = 2000000000ull;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + DT_BM - 1) / DT_BM), (unsigned)((K + DT_BN - 1) / DT_BN));
    cfg.blockDim = dim3(DT_THREADS);
    cfg.dynamicSmemBytes = DT_SMEM_BYTES;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, k_dw_gemm, maps, p) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

}  // namespace bl
