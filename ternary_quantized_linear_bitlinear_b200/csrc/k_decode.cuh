// Steps 3 + 4 for decode-sized M (<= 16): the ternary x INT8 GEMV engine.
//
// What it computes ("bitone" README, How 1.58-bit Works and Forward pass):
//   acc[m, n] = sum_k x_q[m, k] * W_q[n, k];  Y[m, n] = acc * (gamma / s[m])
//
// The work is bound by streaming the packed weights from HBM (2 bits per
// weight).  Design:
//   - A CTA (8 warps) owns 8/G consecutive 32-row groups of one problem;
//     their packed rows are one contiguous byte range, which one thread
//     requests with cp.async.bulk copies into shared memory (one mbarrier per
//     tile, bounded waits), so the memory system sees a few large requests
//     per CTA and the warps issue no global loads for weights.
//   - A warp owns 32 rows (two 16-row MMA tiles that share every x_q
//     fragment); G warps split their K range (G picked per problem from K so
//     that each warp has at most 4 steps of 256 k and a CTA at most 48 KiB
//     of weights; the host raises G for launches too small to fill the GPU).
//   - Unpacking costs 1-2 ALU ops per 4 weights: with the packed layout, word
//     (w << (6 - 2j)) & 0xC0C0C0C0 puts the codes of k = 16w' + 4j .. 4j+3 in
//     the top two bits of four bytes, i.e. the int8 values 64 * W_q.
//   - The MACs run on the tensor cores (mma.sync m16n8k32 s8): W tile as A
//     (16 rows), tokens as B (8 columns, zero for m >= M).  Because the
//     int32 sum is exact, the k order inside a step may be permuted as long
//     as A and B use the same permutation: thread t's A fragment for step
//     pair c holds k = 64t + 16c + (0..15), and its B fragment reads exactly
//     those x_q bytes.
//   - x_q is staged once per CTA in shared memory (rows of round_up(K, 256)
//     bytes, 16-byte chunks XOR-swizzled so that the B loads are free of
//     bank conflicts).
//   - acc = (sum of 64 * W_q * x_q) >> 6 exactly; the split-K partials meet
//     in shared memory; the epilogue rescales and stores Y (and acc).
//   - Fused variant (SRC = bf16 or f32 activations): step 2 runs inside the
//     CTA instead of a separate launch.  One warp per token row (for one or
//     two tokens without SubLN: the whole CTA) computes s = 127 / max|y|
//     (y = x, or the SubLN RMSNorm of x) and writes x_q straight into the
//     swizzled staging rows, with the same arithmetic as the stand-alone
//     activation quantizer, while the weights stream in.
//     Every CTA of a problem quantizes the (L2-resident) rows itself; the
//     problem's first CTA also writes x_q and s to global memory on request.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_SMEM_LIMIT = 200 * 1024;  // weight tiles + staged x_q, per CTA
constexpr int DEC_PF = 4;                   // target 256-k steps per warp (G is chosen from it)
constexpr int DEC_W_CAP = 48 * 1024;        // weight bytes per CTA above which G grows (3 CTAs per SM)
constexpr unsigned long long DEC_TIMEOUT_NS = 2000000000ull;

// Activation source of a launch: pre-quantized x_q, or X to quantize in-kernel.
enum : int { DEC_SRC_XQ = 0, DEC_SRC_BF16 = 1, DEC_SRC_F32 = 2 };

struct DecodeProblem {
    const uint8_t *packed;
    const float *gamma;
    const void *x;         // DEC_SRC_XQ: x_q [M, K] int8; else X [M, K] bf16 / f32
    float *s;              // DEC_SRC_XQ: s [M] in; else s [M] out or null
    float *Y;
    int32_t *acc;
    const float *gain;     // fused: SubLN gain [K] or null
    int8_t *xq_out;        // fused: x_q [M, K] out or null
    int N;
    int K;
    int g_log2;     // log2(G): warps per row tile
    int cta_begin;  // first CTA of this problem in the grouped grid
};

constexpr int DEC_CTA_TABLE = 2048;  // grids up to this size look their problem up in a table

struct DecodeParams {
    DecodeProblem p[BL_MAX_GROUP];
    int count;
    int M;
    int xq_off;  // shared-memory offset of the staged x_q (after the weight tiles)
    int use_table;
    float eps;   // fused: SubLN epsilon
    unsigned char cta_problem[DEC_CTA_TABLE];
};

__host__ __device__ inline int dec_row_stride(int K) { return (K + 255) & ~255; }

__host__ __device__ inline int dec_glog(int K) {
    // smallest G = 2^glog <= 8 with ceil(steps / G) <= DEC_PF and at most
    // DEC_W_CAP bytes of weights per CTA (8 / G groups of 32 rows), so that
    // three CTAs fit on an SM and a grouped launch stays one wave
    int steps = (K + 255) >> 8, g = 0;
    while (g < 3 && ((steps + (1 << g) - 1) >> g) > DEC_PF) ++g;
    while (g < 3 && (DEC_WARPS >> g) * 32 * (K >> 2) > DEC_W_CAP) ++g;
    return g;
}

constexpr int DEC_ROWS = 32;  // weight rows per warp

// bytes of packed weights one CTA stages
__host__ __device__ inline int dec_w_bytes(int K) { return (DEC_WARPS >> dec_glog(K)) * DEC_ROWS * (K >> 2); }

__device__ __forceinline__ u32 dec_unpack(u32 w, int j) {
    // codes of k = 4j .. 4j+3 of this 16-weight word -> int8 lanes holding 64 * W_q
    return (w << (6 - 2 * j)) & 0xC0C0C0C0u;
}

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], u32 a0, u32 a1, u32 a2, u32 a3, u32 b0, u32 b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Float bits of element j of a 16-byte activation vector.
template <bool BF16>
__device__ __forceinline__ u32 dec_x_bits(const uint4 &v, int j) {
    const u32 w = j < (BF16 ? 2 : 1) ? v.x : j < (BF16 ? 4 : 2) ? v.y : j < (BF16 ? 6 : 3) ? v.z : v.w;
    return BF16 ? ((j & 1) ? (w & 0xffff0000u) : (w << 16)) : w;
}

// A row of X is processed in blocks of 128 16-byte vectors, 4 per lane
// (vector blk * 128 + 32 i + lane in register i, zero past the row end); a
// row of at most one block is loaded once and every pass works on registers.
// (Four, not eight: the fused kernel runs once per CTA and its code is cold
// in the instruction cache, so a shorter unrolled body is faster.)
constexpr int DEC_QV = 4;
constexpr int DEC_QB = 8;  // block-cooperative quantization: X vectors per thread (M * K / 8 <= 2048 for bf16)

__device__ __forceinline__ void dec_load_block(uint4 (&c)[DEC_QV], const uint4 *xr, int nvec, int blk, int lane) {
#pragma unroll
    for (int i = 0; i < DEC_QV; ++i) {
        const int v = blk * (32 * DEC_QV) + 32 * i + lane;
        c[i] = v < nvec ? ldg_nc_v4(xr + v) : make_uint4(0, 0, 0, 0);
    }
}

// Exact sum of squares of one row, rounded once to double (valid on lane 0).
// x^2 = mant^2 * 2^(2e - 300) with e >= 1 (subnormals: e = 1, no hidden
// bit).  Each pass adds the values with e in [elo, ehi] (31 binades) as
// mant^2 << 2(e - elo) into a 128-bit lane accumulator (< 2^108 per term,
// at most 1024 terms per lane, a warp sum < 2^123), and lane 0 adds the warp
// sum into 576-bit limbs in units of 2^-298; a pass repeats one window lower
// only while some lane saw a smaller nonzero value (at most 9 passes).
template <bool BF16>
__device__ double dec_row_sumsq(uint4 (&c)[DEC_QV], const uint4 *xr, int nvec, int lane, u32 amax_bits) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int nblk = (nvec + 32 * DEC_QV - 1) / (32 * DEC_QV);
    u64 L[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
    int ehi = (int)(amax_bits >> 23);
    if (ehi < 1) ehi = 1;
    for (int pass = 0; pass < 10; ++pass) {
        const int elo = ehi - 30 < 1 ? 1 : ehi - 30;
        u64 lo = 0ull, hi = 0ull;
        bool below = false;
        for (int blk = 0; blk < nblk; ++blk) {
            if (nblk > 1) dec_load_block(c, xr, nvec, blk, lane);
#pragma unroll
            for (int i = 0; i < DEC_QV; ++i) {
#pragma unroll
                for (int j = 0; j < EPV; ++j) {
                    const u32 u = dec_x_bits<BF16>(c[i], j) & 0x7fffffffu;
                    const int e = (int)(u >> 23);
                    const int ee = e ? e : 1;
                    if (ee <= ehi && ee >= elo && u != 0u) {
                        u64 mm = (u64)(e ? ((u & 0x7fffffu) | 0x800000u) : u);
                        mm *= mm;
                        const int sh = 2 * (ee - elo);  // <= 60
                        const u64 plo = mm << sh;
                        const u64 phi = sh ? (mm >> (64 - sh)) : 0ull;
                        const u64 t = lo + plo;
                        hi += phi + (t < lo ? 1ull : 0ull);
                        lo = t;
                    } else if (ee < elo && u != 0u) {
                        below = true;
                    }
                }
            }
        }
        warp_sum_u128(lo, hi);
        if (lane == 0) limbs_add_u128_shl(L, lo, hi, 2 * (elo - 1));
        if (!__any_sync(0xffffffffu, below) || elo == 1) break;
        ehi = elo - 1;
    }
    return lane == 0 ? limbs_to_double_rn(L, -298) : 0.0;
}

// y of element j of vector v: x, or float(float(x / r) * g)
template <bool BF16>
__device__ __forceinline__ void dec_y4(const uint4 &raw, int q, const float4 *g4, int v, float r, float (&y)[4]) {
    constexpr int EPV = BF16 ? 8 : 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = __uint_as_float(dec_x_bits<BF16>(raw, 4 * q + j));
    if (g4 != nullptr) {
        const float4 g = __ldg(g4 + v * (EPV / 4) + q);
        y[0] = __fmul_rn(__fdiv_rn(y[0], r), g.x);
        y[1] = __fmul_rn(__fdiv_rn(y[1], r), g.y);
        y[2] = __fmul_rn(__fdiv_rn(y[2], r), g.z);
        y[3] = __fmul_rn(__fdiv_rn(y[3], r), g.w);
    }
}

// Step 2 for token row m by one warp, into the swizzled staging row (and,
// when out is set, x_q / s in global memory).  Arithmetic identical to the
// stand-alone quantizer:
//   y = x, or y = float(float(x / r) * g), r = sqrtf(float(double(sum x^2) / K) + eps)
//   s = float(127 / max(max|y|, 1e-5f)),  x_q = clamp(rne(float(y * s)), -128, 127)
// Returns s (on every lane).
template <bool BF16>
__device__ float dec_quant_row(const DecodeProblem &pr, int m, int K, int RS, uint8_t *s_xq, float eps, bool out,
                               int lane) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int nvec = K / EPV;
    const int nblk = (nvec + 32 * DEC_QV - 1) / (32 * DEC_QV);
    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.x) + (size_t)m * nvec;
    const float4 *g4 = reinterpret_cast<const float4 *>(pr.gain);
    uint4 c[DEC_QV];
    dec_load_block(c, xr, nvec, 0, lane);
    u32 amax = 0;
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk > 0) dec_load_block(c, xr, nvec, blk, lane);
#pragma unroll
        for (int i = 0; i < DEC_QV; ++i)
#pragma unroll
            for (int j = 0; j < EPV; ++j) amax = max(amax, dec_x_bits<BF16>(c[i], j) & 0x7fffffffu);
    }
    amax = warp_max_u32(amax);
    float r = 1.f;
    if (g4 != nullptr) {
        if (nblk > 1) dec_load_block(c, xr, nvec, 0, lane);
        const double S2 = dec_row_sumsq<BF16>(c, xr, nvec, lane, amax);
        if (lane == 0) r = __fsqrt_rn(__fadd_rn(__double2float_rn(__ddiv_rn(S2, (double)K)), eps));
        r = __shfl_sync(0xffffffffu, r, 0);
        amax = 0;
        for (int blk = 0; blk < nblk; ++blk) {
            if (nblk > 1) dec_load_block(c, xr, nvec, blk, lane);
#pragma unroll
            for (int i = 0; i < DEC_QV; ++i) {
                const int v = blk * (32 * DEC_QV) + 32 * i + lane;
                if (v >= nvec) continue;
#pragma unroll
                for (int q = 0; q < EPV / 4; ++q) {
                    float y[4];
                    dec_y4<BF16>(c[i], q, g4, v, r, y);
#pragma unroll
                    for (int j = 0; j < 4; ++j) amax = max(amax, __float_as_uint(y[j]) & 0x7fffffffu);
                }
            }
        }
        amax = warp_max_u32(amax);
    }
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(amax), 1e-5f));
    uint8_t *dst = s_xq + m * RS;
    int8_t *gq = out && pr.xq_out != nullptr ? pr.xq_out + (size_t)m * K : nullptr;
    for (int blk = 0; blk < nblk; ++blk) {
        if (nblk > 1) dec_load_block(c, xr, nvec, blk, lane);
#pragma unroll
        for (int i = 0; i < DEC_QV; ++i) {
            const int v = blk * (32 * DEC_QV) + 32 * i + lane;
            if (v >= nvec) continue;
            u32 word[EPV / 4];
#pragma unroll
            for (int q = 0; q < EPV / 4; ++q) {
                float y[4];
                dec_y4<BF16>(c[i], q, g4, v, r, y);
                u32 w = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int qi = __float2int_rn(__fmul_rn(y[j], s));
                    qi = max(-128, min(127, qi));
                    w |= ((u32)qi & 0xffu) << (8 * j);
                }
                word[q] = w;
            }
            // 16-byte chunk L of the row holds k = 16L .. 16L + 15
            const int L = BF16 ? (v >> 1) : (v >> 2);
            const int within = BF16 ? (v & 1) * 8 : (v & 3) * 4;
            const int x = (((L >> 3) & 1) << 1) | (m & 1);
            uint8_t *d = dst + ((((L & ~7) | ((L ^ x) & 7)) << 4) + within);
            if (BF16) {
                *reinterpret_cast<uint2 *>(d) = make_uint2(word[0], word[EPV / 4 - 1]);
                if (gq) *reinterpret_cast<uint2 *>(gq + (size_t)v * 8) = make_uint2(word[0], word[EPV / 4 - 1]);
            } else {
                *reinterpret_cast<u32 *>(d) = word[0];
                if (gq) *reinterpret_cast<u32 *>(gq + (size_t)v * 4) = word[0];
            }
        }
    }
    if (out && lane == 0 && pr.s != nullptr) pr.s[m] = s;
    return s;
}

// NT: 8-token column tiles (1: M <= 8, 2: M <= 16).  SRC: DEC_SRC_*.
template <int NT, int SRC>
__global__ void __launch_bounds__(DEC_THREADS, 3) k_decode(const __grid_constant__ DecodeParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_red[DEC_WARPS][2][NT][4][32];
    __shared__ __align__(8) u64 s_bar[DEC_WARPS];
    __shared__ float s_f[16];
    __shared__ u32 s_amax[16];
    __shared__ float s_sc[16];
    if (SRC != DEC_SRC_XQ && threadIdx.x < 16) s_amax[threadIdx.x] = 0u;

    // a programmatically dependent launch that follows may start its prologue
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int b = blockIdx.x;
    int pi;
    if (P.use_table) {
        pi = P.cta_problem[b];
    } else {  // binary search over the CTA prefix
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.p[mid].cta_begin <= b) lo = mid; else hi = mid - 1;
        }
        pi = lo;
    }
    const DecodeProblem &pr = P.p[pi];
    const int M = P.M, N = pr.N, K = pr.K;
    const int glog = pr.g_log2, G = 1 << glog;
    const int T = DEC_WARPS >> glog;  // 32-row groups per CTA
    const int Kw = K >> 2;            // packed bytes per row
    const int row_base = (b - pr.cta_begin) * T * DEC_ROWS;
    const int rows = min(T * DEC_ROWS, N - row_base);
    const int groups = (rows + DEC_ROWS - 1) / DEC_ROWS;

    // One thread requests the CTA's weight rows, one bulk copy (and one
    // mbarrier) per 32-row group, so each warp starts as soon as its rows land.
    // It is lane 0 of the last warp: the fused path quantizes token row m in
    // warp m, so for small M the first rows do not wait for the requests.
    if (threadIdx.x == DEC_THREADS - 32) {
        for (int i = 0; i < groups; ++i) mbar_init(smem_u32(&s_bar[i]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        const uint8_t *src = pr.packed + (size_t)row_base * Kw;
        const u32 dst = smem_u32(smem);
        const u64 policy = l2_policy_evict_first();  // weights are read once per launch
        for (int i = 0; i < groups; ++i) {
            const u32 nrows = (u32)min(DEC_ROWS, rows - DEC_ROWS * i);
            const u32 bytes = nrows * (u32)Kw;
            const u32 bar = smem_u32(&s_bar[i]);
            mbar_arrive_expect_tx(bar, bytes);
            const u32 off0 = (u32)(DEC_ROWS * i) * (u32)Kw;
            for (u32 off = 0; off < bytes; off += 32768u) {
                const u32 n = bytes - off < 32768u ? bytes - off : 32768u;
                bulk_g2s_hint(dst + off0 + off, src + off0 + off, n, bar, policy);
            }
        }
    }

    // x_q and s may be produced by the kernel launched just before this one.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // Stage x_q rows [0, M) into shared memory, swizzled, zero-padded to RS;
    // float(gamma / s[m]) once per token.
    const int RS = dec_row_stride(K);
    uint8_t *s_xq = smem + P.xq_off;
    if (SRC != DEC_SRC_XQ) {
        constexpr bool BF16 = SRC == DEC_SRC_BF16;
        constexpr int EPV = BF16 ? 8 : 4;
        const bool out = b == pr.cta_begin;
        const int nvec = K / EPV;
        const int tot = M * nvec;  // 16-byte vectors of X, rows contiguous
        if (pr.gain == nullptr && M <= 2 && tot <= DEC_QB * DEC_THREADS) {
            // fused step 2 for one or two tokens, no SubLN, all of X in
            // registers: thread t holds vectors t + 256 i; one load round
            // trip, per-row max by a warp reduction and a shared atomic (max
            // of the float bits of |x|).  (Measured: faster than a warp per
            // row for M <= 2, slower from M = 4 on.)
            const uint4 *xv = reinterpret_cast<const uint4 *>(pr.x);
            uint4 c[DEC_QB];
#pragma unroll
            for (int i = 0; i < DEC_QB; ++i) {
                const int idx = (int)threadIdx.x + DEC_THREADS * i;
                c[i] = idx < tot ? ldg_nc_v4(xv + idx) : make_uint4(0, 0, 0, 0);
            }
            __syncthreads();  // s_amax cleared
            const int lane = threadIdx.x & 31;
#pragma unroll
            for (int i = 0; i < DEC_QB; ++i) {
                const int idx = (int)threadIdx.x + DEC_THREADS * i;
                if (DEC_THREADS * i >= tot) break;  // uniform: no vector of this round is in range
                u32 a = 0;
                const int m = idx < tot ? idx / nvec : -1;
#pragma unroll
                for (int j = 0; j < EPV; ++j) a = max(a, dec_x_bits<BF16>(c[i], j) & 0x7fffffffu);
                // one shared atomic per warp when the warp's 32 vectors lie in one row
                const int m0 = __shfl_sync(0xffffffffu, m, 0);
                if (__all_sync(0xffffffffu, m == m0)) {
                    a = __reduce_max_sync(0xffffffffu, a);
                    if (lane == 0 && m0 >= 0) atomicMax(&s_amax[m0], a);
                } else if (m >= 0) {
                    atomicMax(&s_amax[m], a);
                }
            }
            __syncthreads();
            if (threadIdx.x < M) {
                const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(s_amax[threadIdx.x]), 1e-5f));
                s_sc[threadIdx.x] = s;
                s_f[threadIdx.x] = __fdiv_rn(*pr.gamma, s);
                if (out && pr.s != nullptr) pr.s[threadIdx.x] = s;
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < DEC_QB; ++i) {
                const int idx = (int)threadIdx.x + DEC_THREADS * i;
                if (idx >= tot) continue;
                const int m = idx / nvec, v = idx - m * nvec;
                const float s = s_sc[m];
                u32 word[EPV / 4];
#pragma unroll
                for (int q = 0; q < EPV / 4; ++q) {
                    u32 w = 0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        int qi = __float2int_rn(__fmul_rn(__uint_as_float(dec_x_bits<BF16>(c[i], 4 * q + j)), s));
                        qi = max(-128, min(127, qi));
                        w |= ((u32)qi & 0xffu) << (8 * j);
                    }
                    word[q] = w;
                }
                const int L = BF16 ? (v >> 1) : (v >> 2);
                const int within = BF16 ? (v & 1) * 8 : (v & 3) * 4;
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                uint8_t *d = s_xq + m * RS + ((((L & ~7) | ((L ^ x) & 7)) << 4) + within);
                int8_t *gq = out && pr.xq_out != nullptr ? pr.xq_out + (size_t)m * K : nullptr;
                if (BF16) {
                    *reinterpret_cast<uint2 *>(d) = make_uint2(word[0], word[EPV / 4 - 1]);
                    if (gq) *reinterpret_cast<uint2 *>(gq + (size_t)v * 8) = make_uint2(word[0], word[EPV / 4 - 1]);
                } else {
                    *reinterpret_cast<u32 *>(d) = word[0];
                    if (gq) *reinterpret_cast<u32 *>(gq + (size_t)v * 4) = word[0];
                }
            }
        } else {
            // fused step 2: warp w quantizes rows w, w + 8
            const int lane = threadIdx.x & 31;
            for (int m = threadIdx.x >> 5; m < M; m += DEC_WARPS) {
                const float s = dec_quant_row<BF16>(pr, m, K, RS, s_xq, P.eps, out, lane);
                if (lane == 0) s_f[m] = __fdiv_rn(*pr.gamma, s);
            }
        }
        const int chunks = RS >> 4, kchunks = K >> 4;
        for (int r = 0; r < M; ++r) {
            for (int L = kchunks + (int)threadIdx.x; L < chunks; L += DEC_THREADS) {
                const int x = (((L >> 3) & 1) << 1) | (r & 1);
                *reinterpret_cast<uint4 *>(s_xq + r * RS + (((L & ~7) | ((L ^ x) & 7)) << 4)) =
                    make_uint4(0, 0, 0, 0);
            }
        }
    } else {
        // every 16-byte chunk in flight at once (cp.async), one wait
        const int chunks = RS >> 4;
        const int kchunks = K >> 4;
        for (int r = 0; r < M; ++r) {
            const int8_t *src = static_cast<const int8_t *>(pr.x) + (size_t)r * K;
            uint8_t *dst = s_xq + r * RS;
            for (int L = threadIdx.x; L < chunks; L += DEC_THREADS) {
                const int x = (((L >> 3) & 1) << 1) | (r & 1);
                uint8_t *d = dst + (((L & ~7) | ((L ^ x) & 7)) << 4);
                if (L < kchunks) {
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(d)), "l"(src + L * 16)
                                 : "memory");
                } else {
                    *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (threadIdx.x < M) s_f[threadIdx.x] = __fdiv_rn(*pr.gamma, pr.s[threadIdx.x]);
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wg = warp >> glog, kslot = warp & (G - 1);
    const int row0 = wg * DEC_ROWS;  // within the CTA
    const int steps = (K + 255) >> 8;
    const int nchunk64 = K >> 6;

    // acc[tile][nt][4]: two 16-row tiles, each with two independent chains
    int acc[2][NT][4], acc2[2][NT][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[u][nt][i] = acc2[u][nt][i] = 0;

    bool ok = true;
    if (wg < groups) {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&s_bar[wg]), 0, DEC_TIMEOUT_NS, nullptr));
        if (!ok && lane == 0) raise_device_error(DEVERR_TIMEOUT_PRODUCER);
    }

    if (ok && wg < groups) {
        // rows g, g+8 (tile 0) and g+16, g+24 (tile 1)
        const uint8_t *w0 = smem + (row0 + g) * Kw + t * 16;
        const int Kw8 = 8 * Kw;
        // B fragments: token rows g (and g + 8); chunk c of a step sits at
        // 16 * (4t + (c ^ xb)) within the step's 256 bytes (the swizzle)
        const bool tv0 = g < M, tv1 = NT > 1 && g + 8 < M;
        const int xb0 = ((t >> 1) << 1) | (g & 1);
        const int xb1 = ((t >> 1) << 1) | ((g + 8) & 1);
        const uint8_t *xr0 = s_xq + g * RS + t * 64;
        const uint8_t *xr1 = s_xq + (g + 8) * RS + t * 64;
        int o0[4], o1[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            o0[c] = (c ^ xb0) << 4;
            o1[c] = (c ^ xb1) << 4;
        }
#pragma unroll 1
        for (int s2 = kslot; s2 < steps; s2 += G) {
            const bool kv = (s2 * 4 + t) < nchunk64;
            uint4 wv[4];
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4)
                wv[r4] = kv ? *reinterpret_cast<const uint4 *>(w0 + r4 * Kw8 + s2 * 64) : make_uint4(0, 0, 0, 0);
            const uint8_t *x0p = xr0 + s2 * 256;
            const uint8_t *x1p = xr1 + s2 * 256;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 x0 = tv0 ? *reinterpret_cast<const uint4 *>(x0p + o0[c]) : make_uint4(0, 0, 0, 0);
                uint4 x1 = make_uint4(0, 0, 0, 0);
                if (NT > 1 && tv1) x1 = *reinterpret_cast<const uint4 *>(x1p + o1[c]);
                const u32 xq0[4] = {x0.x, x0.y, x0.z, x0.w};
                const u32 xq1[4] = {x1.x, x1.y, x1.z, x1.w};
                const u32 wr[4] = {(&wv[0].x)[c], (&wv[1].x)[c], (&wv[2].x)[c], (&wv[3].x)[c]};
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    int(&A)[NT][4] = (c & 1) ? acc2[u] : acc[u];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const u32 a0 = dec_unpack(wr[2 * u], 2 * h), a2 = dec_unpack(wr[2 * u], 2 * h + 1);
                        const u32 a1 = dec_unpack(wr[2 * u + 1], 2 * h), a3 = dec_unpack(wr[2 * u + 1], 2 * h + 1);
                        mma_s8_16832(A[0], a0, a1, a2, a3, xq0[2 * h], xq0[2 * h + 1]);
                        if (NT > 1) mma_s8_16832(A[NT - 1], a0, a1, a2, a3, xq1[2 * h], xq1[2 * h + 1]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[u][nt][i] += acc2[u][nt][i];

    // split-K reduction through shared memory
    if (G > 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) s_red[warp][u][nt][i][lane] = acc[u][nt][i];
        __syncthreads();
        if (kslot == 0) {
            for (int q = 1; q < G; ++q)
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[u][nt][i] += s_red[warp + q][u][nt][i][lane];
        }
    }
    if (kslot != 0 || !ok || wg >= groups) return;

#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int m = nt * 8 + 2 * t + e;
            if (m >= M) continue;
            const float f = s_f[m];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int n = row_base + row0 + 16 * u + g + 8 * hh;
                    if (n < N) {
                        const int a_ = acc[u][nt][2 * hh + e] >> 6;  // exact: the sum is a multiple of 64
                        pr.Y[(size_t)m * N + n] = __fmul_rn(__int2float_rn(a_), f);
                        if (pr.acc) pr.acc[(size_t)m * N + n] = a_;
                    }
                }
            }
        }
    }
}

}  // namespace bl
