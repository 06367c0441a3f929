// Steps 3 + 4 for decode-sized M (<= 16): the ternary x INT8 GEMV engine.
//
// What it computes ("bitone" README, How 1.58-bit Works and Forward pass):
//   acc[m, n] = sum_k x_q[m, k] * W_q[n, k];  Y[m, n] = acc * (gamma / s[m])
//
// The work is bound by streaming the packed weights from HBM (2 bits per
// weight).  Design:
//   - A CTA owns a contiguous range of whole 32-row groups of one problem,
//     at most DEC_W_CAP packed bytes, so that three CTAs (of this launch or
//     of the next) share an SM.  Its rows are one contiguous byte range of
//     the packed matrix: lane 0 of the last warp requests them with one bulk
//     copy (cp.async.bulk, L2 evict-first) per group into shared memory, one
//     mbarrier per group, before waiting on the launch before this one: the
//     weights are static, so with BL_FWD_WEIGHTS_READY (a programmatic
//     dependent launch) a CTA that lands on an SM while that launch finishes
//     streams its weights at once.
//   - The CTA's 8 warps split its groups: G = 8 / T warps per group (T
//     groups per CTA) take every G-th 256-k step of it, G chosen per problem
//     from K so that a warp has a few steps.  Partial sums meet in shared
//     memory (int32, exact), and the CTA writes Y with a thread per (token,
//     row), 32 consecutive floats per warp and token.
//   - MACs on the tensor cores (mma.sync m16n8k32, u8 x s8): weight rows as
//     A (two 16-row tiles per group share every x_q fragment), tokens as B (8
//     columns per tile; the columns m >= M read token M - 1 and are never
//     stored).  The int32 sum is exact, so the k order inside a step may be
//     permuted as long as A and B use the same permutation: the lane with
//     k-slot t holds the packed bytes 16t .. 16t + 15 of the step (k = 64t ..
//     64t + 63), and its B fragment reads those x_q bytes.
//   - Unpacking: a packed word holds the codes c = 1 - W_q in {0, 1, 2};
//     (word << (6 - 2j)) & 0xC0C0C0C0 leaves the codes of k = 16w' + 4j ..
//     4j+3 in the top two bits of four bytes, the unsigned values 64 c, so
//     every plane shares one accumulator per tile:
//     sum_k W_q x = sum_k x - (sum_k 64 c x) / 64, exact (a multiple of 64),
//     with sum_k x the row sum of the staged x_q.
//   - x_q is staged once per CTA in shared memory (rows of round_up(K, 256)
//     bytes, 16-byte chunks XOR-swizzled so that the B loads are free of
//     bank conflicts).  Fused variant (SRC = bf16 or f32 activations): step
//     2 runs inside the CTA with the same arithmetic as the stand-alone
//     activation quantizer (a warp per row without SubLN, from registers
//     after one load, or the whole CTA in rounds for long rows; SubLN rows a
//     warp per row); the problem's first CTA also writes x_q and s on
//     request.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_ROWS = 32;                // weight rows per group (two MMA tiles)
constexpr int DEC_PF = 4;                   // target 256-k steps per warp (G is chosen from it)
constexpr int DEC_W_CAP = 56 * 1024;        // packed bytes per CTA above which G grows (three CTAs per SM)
constexpr int DEC_MAX_CTAS = 2048;          // CTAs per launch (larger calls are split into launches)
constexpr int DEC_X_MAX = 144 * 1024;       // staged activations per CTA
constexpr int DEC_MAX_PSLOTS = 1;           // problems per CTA (the staging helpers take a slot array)
constexpr unsigned long long DEC_TIMEOUT_NS = 2000000000ull;

// Activation source of a launch: pre-quantized x_q, or X to quantize in-kernel.
enum : int { DEC_SRC_XQ = 0, DEC_SRC_BF16 = 1, DEC_SRC_F32 = 2 };

struct DecodeProblem {
    const uint8_t *packed; // [N, K/4], 16-byte aligned
    const float *gamma;
    const void *x;         // DEC_SRC_XQ: x_q [M, K] int8; else X [M, K] bf16 / f32
    float *s;              // DEC_SRC_XQ: s [M] in; else s [M] out or null
    float *Y;              // [M, N]
    int32_t *acc;          // [M, N] or null
    const float *gain;     // fused: SubLN gain [K] or null
    int8_t *xq_out;        // fused: x_q [M, K] out or null
    int N, K;
    int row0;              // first row of this launch's part of the problem
    int rows;              // rows of that part
    int glog;              // log2(G): warps per group
    int cta_begin;         // first CTA of this problem in the launch
    int kch;               // K chunks: 1, or one group per CTA in chunks of DEC_KCH_B bytes a row
};

struct DecodeParams {
    DecodeProblem p[BL_MAX_GROUP];
    int count;
    int M;
    float eps;                                 // fused: SubLN epsilon
    int x_off;                                 // shared-memory offsets of the staged x_q and of the sums
    int acc_off;
    unsigned char cta_problem[DEC_MAX_CTAS];   // problem of each CTA
};

// A problem as one CTA sees it, in shared memory.
struct DecSlot {
    const void *x;
    float *s;
    const float *gain;
    int8_t *xq_out;
    int K;
    int first;  // this CTA holds the problem's first rows (writes x_q and s on request)
};

__host__ __device__ inline int dec_glog(int K) {
    // smallest G = 2^glog <= 8 with ceil(steps / G) <= DEC_PF and at most
    // DEC_W_CAP bytes of weights per CTA (8 / G groups of 32 rows)
    const int steps = (K + 255) >> 8;
    int g = 0;
    while (g < 3 && ((steps + (1 << g) - 1) >> g) > DEC_PF) ++g;
    while (g < 3 && (DEC_WARPS >> g) * DEC_ROWS * (K >> 2) > DEC_W_CAP) ++g;
    return g;
}

__host__ __device__ inline int dec_row_stride(int K) { return (K + 255) & ~255; }

// codes of k = 4j .. 4j+3 of this 16-weight word as u8 lanes 4^j * (1 - W_q)
__device__ __forceinline__ u32 dec_plane(u32 w, int j) { return w & (0x03030303u << (2 * j)); }

// the same codes moved to the top two bits: u8 lanes 64 * (1 - W_q)
__device__ __forceinline__ u32 dec_plane_top(u32 w, int j) { return (w << (6 - 2 * j)) & 0xC0C0C0C0u; }

// unsigned 8-bit A (the weight codes), signed 8-bit B (x_q)
__device__ __forceinline__ void mma_u8s8_16832(int (&c)[4], u32 a0, u32 a1, u32 a2, u32 a3, u32 b0, u32 b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
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
__device__ float dec_quant_row(const DecSlot &pr, int m, int K, int RS, uint8_t *s_xq, float eps, bool out,
                               int lane, int *rowsum) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int nvec = K / EPV;
    const int nblk = (nvec + 32 * DEC_QV - 1) / (32 * DEC_QV);
    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.x) + (size_t)m * nvec;
    const float4 *g4 = reinterpret_cast<const float4 *>(pr.gain);
    uint4 c[DEC_QV];
    dec_load_block(c, xr, nvec, 0, lane);
    u32 amax = 0;
    double dsq = 0.0;  // SubLN rows: the double estimate of sum x^2
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk > 0) dec_load_block(c, xr, nvec, blk, lane);
#pragma unroll
        for (int i = 0; i < DEC_QV; ++i)
#pragma unroll
            for (int j = 0; j < EPV; ++j) {
                const u32 b = dec_x_bits<BF16>(c[i], j);
                amax = max(amax, b & 0x7fffffffu);
                if (g4 != nullptr) {
                    const double xd = abs_as_double(b);
                    dsq = __fma_rn(xd, xd, dsq);
                }
            }
    }
    amax = warp_max_u32(amax);
    float r = 1.f;
    if (g4 != nullptr) {
        dsq = warp_sum_f64(dsq);
        float f;
        bool decided = subln_mean_sq_from_estimate(dsq, K, amax, &f);
        decided = __shfl_sync(0xffffffffu, decided, 0);  // lane 0's sum decides (lanes may round differently)
        f = __shfl_sync(0xffffffffu, f, 0);
        if (decided) {
            r = __fsqrt_rn(__fadd_rn(f, eps));
        } else {
            if (nblk > 1) dec_load_block(c, xr, nvec, 0, lane);
            const double S2 = dec_row_sumsq<BF16>(c, xr, nvec, lane, amax);
            if (lane == 0) r = __fsqrt_rn(__fadd_rn(__double2float_rn(__ddiv_rn(S2, (double)K)), eps));
            r = __shfl_sync(0xffffffffu, r, 0);
        }
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
    int rs = 0;
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
                    rs += qi;
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
    rs = __reduce_add_sync(0xffffffffu, rs);
    if (lane == 0) *rowsum = rs;
    return s;
}

// Step 2 for all (problem, token) rows of a CTA at once, rows without SubLN:
// the concatenated rows are taken in rounds of DEC_QBV * DEC_THREADS 16-byte
// vectors, every thread holding the vectors t, t + DEC_THREADS, ... of a
// round with all its loads in flight together (one memory round trip per
// round for the CTA, not one per row and warp).  Pass 1 meets the row maxima
// in shared memory (max of the float bits of |x|); pass 2 quantizes each
// vector into the staging rows, the rounds in reverse order so that the one
// still in registers is not loaded again.  Same arithmetic as dec_quant_row.
// vbase[ps] = first vector of problem slot ps (vbase[np] = the total);
// s_amax[np * M] and s_rs[np * M] zeroed before.
constexpr int DEC_QBV = 8;

template <bool BF16>
__device__ void dec_quant_block(const DecSlot *sl, int np, int M, const int *s_xoff, const int *vbase, uint8_t *s_x,
                                u32 *s_amax, float *s_sc, const float *s_gam, float (*s_f)[16], int *s_rs) {
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int RV = DEC_QBV * DEC_THREADS;  // vectors per round
    const int T = vbase[np];
    const int rounds = (T + RV - 1) / RV;
    const int lane = threadIdx.x & 31;
    uint4 c[DEC_QBV];
    int meta[DEC_QBV];  // (slot << 20) | (m << 16) | vector within the row; -1 past the end
    auto load_round = [&](int rd) {
#pragma unroll
        for (int i = 0; i < DEC_QBV; ++i) {
            const int idx = rd * RV + (int)threadIdx.x + DEC_THREADS * i;
            meta[i] = -1;
            c[i] = make_uint4(0, 0, 0, 0);
            if (idx < T) {
                int ps = 0;
                while (ps + 1 < np && idx >= vbase[ps + 1]) ++ps;
                const int nvec = sl[ps].K / EPV;
                const int local = idx - vbase[ps];
                const int m = local / nvec, v = local - m * nvec;
                meta[i] = (ps << 20) | (m << 16) | v;
                c[i] = ldg_nc_v4(reinterpret_cast<const uint4 *>(sl[ps].x) + (size_t)m * nvec + v);
            }
        }
    };
    for (int rd = 0; rd < rounds; ++rd) {
        load_round(rd);
#pragma unroll
        for (int i = 0; i < DEC_QBV; ++i) {
            if (rd * RV + DEC_THREADS * i >= T) break;  // uniform: no vector of this row of the round is in range
            u32 a = 0;
#pragma unroll
            for (int j = 0; j < EPV; ++j) a = max(a, dec_x_bits<BF16>(c[i], j) & 0x7fffffffu);
            const int row = meta[i] < 0 ? -1 : ((meta[i] >> 20) * M + ((meta[i] >> 16) & 15));
            const int row0 = __shfl_sync(0xffffffffu, row, 0);
            if (__all_sync(0xffffffffu, row == row0)) {
                a = __reduce_max_sync(0xffffffffu, a);
                if (lane == 0 && row0 >= 0) atomicMax(&s_amax[row0], a);
            } else if (row >= 0) {
                atomicMax(&s_amax[row], a);
            }
        }
    }
    __syncthreads();
    for (int r = threadIdx.x; r < np * M; r += DEC_THREADS) {
        const int ps = r / M, m = r - ps * M;
        const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(s_amax[r]), 1e-5f));
        s_sc[r] = s;
        s_f[ps][m] = __fdiv_rn(s_gam[ps], s);
        if (sl[ps].first && sl[ps].s != nullptr) sl[ps].s[m] = s;
    }
    __syncthreads();
    for (int rd = rounds - 1; rd >= 0; --rd) {
        if (rd != rounds - 1) load_round(rd);
#pragma unroll
        for (int i = 0; i < DEC_QBV; ++i) {
            if (rd * RV + DEC_THREADS * i >= T) break;  // uniform
            int rsum = 0;
            const int row = meta[i] < 0 ? -1 : ((meta[i] >> 20) * M + ((meta[i] >> 16) & 15));
            if (meta[i] >= 0) {
                const int ps = meta[i] >> 20, m = (meta[i] >> 16) & 15, v = meta[i] & 0xffff;
                const DecSlot &pr = sl[ps];
                const int K = pr.K, RS = dec_row_stride(K);
                const float s = s_sc[ps * M + m];
                u32 word[EPV / 4];
#pragma unroll
                for (int q = 0; q < EPV / 4; ++q) {
                    u32 w = 0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        int qi = __float2int_rn(__fmul_rn(__uint_as_float(dec_x_bits<BF16>(c[i], 4 * q + j)), s));
                        qi = max(-128, min(127, qi));
                        rsum += qi;
                        w |= ((u32)qi & 0xffu) << (8 * j);
                    }
                    word[q] = w;
                }
                const int L = BF16 ? (v >> 1) : (v >> 2);
                const int within = BF16 ? (v & 1) * 8 : (v & 3) * 4;
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                uint8_t *d = s_x + s_xoff[ps] + m * RS + ((((L & ~7) | ((L ^ x) & 7)) << 4) + within);
                int8_t *gq = (pr.first && pr.xq_out != nullptr) ? pr.xq_out + (size_t)m * K : nullptr;
                if (BF16) {
                    *reinterpret_cast<uint2 *>(d) = make_uint2(word[0], word[EPV / 4 - 1]);
                    if (gq) *reinterpret_cast<uint2 *>(gq + (size_t)v * 8) = make_uint2(word[0], word[EPV / 4 - 1]);
                } else {
                    *reinterpret_cast<u32 *>(d) = word[0];
                    if (gq) *reinterpret_cast<u32 *>(gq + (size_t)v * 4) = word[0];
                }
            }
            // the row sums of x_q, one shared atomic per warp when its vectors share a row
            const int row0 = __shfl_sync(0xffffffffu, row, 0);
            if (__all_sync(0xffffffffu, row == row0)) {
                rsum = __reduce_add_sync(0xffffffffu, rsum);
                if (lane == 0 && row0 >= 0) atomicAdd(&s_rs[row0], rsum);
            } else if (row >= 0) {
                atomicAdd(&s_rs[row], rsum);
            }
        }
    }
}

// Step 2 for rows without SubLN of at most DEC_RJ 16-byte vectors per lane
// (K <= 2048 for bf16, 1024 for f32): warp w quantizes the rows w, w +
// DEC_WARPS, ... (row = slot * M + token) from registers after one load
// each.
// Same arithmetic as dec_quant_row: s = float(127 / max(max|x|, 1e-5f)),
// x_q = clamp(rne(float(x * s)), -128, 127).
constexpr int DEC_RJ = 8;

template <bool BF16>
__device__ __forceinline__ void dec_row_load(uint4 (&c)[DEC_RJ], const DecSlot *sl, int M, int r, int lane) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int ps = r / M, m = r - ps * M;
    const int nvec = sl[ps].K / EPV;
    const uint4 *xr = reinterpret_cast<const uint4 *>(sl[ps].x) + (size_t)m * nvec;
#pragma unroll
    for (int j = 0; j < DEC_RJ; ++j) {
        const int v = lane + 32 * j;
        c[j] = v < nvec ? ldg_nc_v4(xr + v) : make_uint4(0, 0, 0, 0);
    }
}

// four products x * s rounded to the nearest even integer, saturated to
// int8 and packed, the first in the low byte
__device__ __forceinline__ u32 dec_q4(u32 a, u32 b, u32 c, u32 d, float s) {
    const int qa = __float2int_rn(__fmul_rn(__uint_as_float(a), s));
    const int qb = __float2int_rn(__fmul_rn(__uint_as_float(b), s));
    const int qc = __float2int_rn(__fmul_rn(__uint_as_float(c), s));
    const int qd = __float2int_rn(__fmul_rn(__uint_as_float(d), s));
    u32 hi, w;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(qd), "r"(qc));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(w) : "r"(qb), "r"(qa), "r"(hi));
    return w;
}

template <bool BF16>
__device__ __forceinline__ void dec_row_quant(const uint4 (&c)[DEC_RJ], const DecSlot *sl, int M, int r,
                                              uint8_t *s_x, const int *s_xoff, const float *s_gam, float (*s_f)[16],
                                              int *s_rs, int lane) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int ps = r / M, m = r - ps * M;
    const DecSlot &pr = sl[ps];
    const int K = pr.K, nvec = K / EPV, RS = dec_row_stride(K);
    // max |x| as float bits (bf16: 16-bit magnitudes, two per word)
    u32 am = 0;
#pragma unroll
    for (int j = 0; j < DEC_RJ; ++j) {
        if (BF16) {
            const u32 p = __vmaxu2(__vmaxu2(c[j].x & 0x7fff7fffu, c[j].y & 0x7fff7fffu),
                                   __vmaxu2(c[j].z & 0x7fff7fffu, c[j].w & 0x7fff7fffu));
            am = __vmaxu2(am, p);
        } else {
            am = max(am, max(max(c[j].x & 0x7fffffffu, c[j].y & 0x7fffffffu),
                             max(c[j].z & 0x7fffffffu, c[j].w & 0x7fffffffu)));
        }
    }
    if (BF16) am = max(am >> 16, am & 0xffffu) << 16;
    am = __reduce_max_sync(0xffffffffu, am);
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(am), 1e-5f));
    uint8_t *dst = s_x + s_xoff[ps] + m * RS;
    int8_t *gq = pr.first && pr.xq_out != nullptr ? pr.xq_out + (size_t)m * K : nullptr;
    int rs = 0;
#pragma unroll
    for (int j = 0; j < DEC_RJ; ++j) {
        const int v = lane + 32 * j;
        if (v < nvec) {
            // 16-byte chunk L of the row holds k = 16L .. 16L + 15
            const int L = BF16 ? (v >> 1) : (v >> 2);
            const int within = BF16 ? (v & 1) * 8 : (v & 3) * 4;
            const int x = (((L >> 3) & 1) << 1) | (m & 1);
            uint8_t *d = dst + ((((L & ~7) | ((L ^ x) & 7)) << 4) + within);
            if (BF16) {
                const u32 w0 = dec_q4(c[j].x << 16, c[j].x & 0xffff0000u, c[j].y << 16, c[j].y & 0xffff0000u, s);
                const u32 w1 = dec_q4(c[j].z << 16, c[j].z & 0xffff0000u, c[j].w << 16, c[j].w & 0xffff0000u, s);
                rs = __dp4a((int)w1, 0x01010101, __dp4a((int)w0, 0x01010101, rs));
                *reinterpret_cast<uint2 *>(d) = make_uint2(w0, w1);
                if (gq) *reinterpret_cast<uint2 *>(gq + (size_t)v * 8) = make_uint2(w0, w1);
            } else {
                const u32 w0 = dec_q4(c[j].x, c[j].y, c[j].z, c[j].w, s);
                rs = __dp4a((int)w0, 0x01010101, rs);
                *reinterpret_cast<u32 *>(d) = w0;
                if (gq) *reinterpret_cast<u32 *>(gq + (size_t)v * 4) = w0;
            }
        }
    }
    rs = __reduce_add_sync(0xffffffffu, rs);
    if (lane == 0) {
        s_rs[r] = rs;
        s_f[ps][m] = __fdiv_rn(s_gam[ps], s);
        if (pr.first && pr.s != nullptr) pr.s[m] = s;
    }
}

template <bool BF16>
__device__ void dec_quant_rows(const DecSlot *sl, int np, int M, uint8_t *s_x, const int *s_xoff, const float *s_gam,
                               float (*s_f)[16], int *s_rs, int warp, int lane) {
    uint4 c[DEC_RJ];
    for (int r = warp; r < np * M; r += DEC_WARPS) {
        dec_row_load<BF16>(c, sl, M, r, lane);
        dec_row_quant<BF16>(c, sl, M, r, s_x, s_xoff, s_gam, s_f, s_rs, lane);
    }
}

__device__ __forceinline__ int dec_nsteps(int K) { return (K + 255) >> 8; }

// Shared memory of a launch: the CTA's packed weights plus DEC_W_PAD, then
// at x_off the staged x_q (M rows of round_up(K, 256) bytes), then at
// acc_off the sums (T groups x 32 rows x M).  A group of whole rows is
// staged when it is at most DEC_W_WHOLE bytes and fits beside x_q in the
// budget; longer rows are staged in chunks of DEC_KCH_B bytes (one group per
// CTA; a bulk copy per row and chunk).
constexpr int DEC_W_PAD = 256;  // reads of a row's last step may run past the copied bytes
constexpr int DEC_W_WHOLE = 48 * 1024;
constexpr int DEC_KCH_B = 2048;
inline int dec_kch(int K, int M, size_t budget) {
    const size_t whole = (size_t)DEC_ROWS * (K >> 2);
    if (whole <= DEC_W_WHOLE && whole + DEC_W_PAD + (size_t)M * dec_row_stride(K) + DEC_ROWS * M * 4 + 256 <= budget)
        return 1;
    return ((K >> 2) + DEC_KCH_B - 1) / DEC_KCH_B;
}

// NT: 8-token column tiles (1: M <= 8, 2: M <= 16).  SRC: DEC_SRC_*.
template <int NT, int SRC>
__global__ void __launch_bounds__(DEC_THREADS, 3) k_decode(const __grid_constant__ DecodeParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) u64 s_bar[DEC_WARPS];
    __shared__ DecSlot s_sl[1];
    __shared__ float s_f[1][16];
    __shared__ float s_gam[1];
    __shared__ int s_xoff[2];
    __shared__ int s_vbase[2];
    __shared__ u32 s_amax[16];
    __shared__ float s_sc[16];
    __shared__ int s_rs[16];  // row sums of the staged x_q

    // a programmatically dependent launch that follows may start its prologue
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int b = blockIdx.x;
    const DecodeProblem &pr = P.p[P.cta_problem[b]];
    const int M = P.M, N = pr.N, K = pr.K;
    const int glog = pr.glog, G = 1 << glog;
    const int T = DEC_WARPS >> glog;  // 32-row groups per CTA
    const int RB = K >> 2;            // packed bytes per row
    const int rbase = pr.row0 + (b - pr.cta_begin) * T * DEC_ROWS;  // first row of this CTA
    const int rows = min(T * DEC_ROWS, pr.row0 + pr.rows - rbase);
    const int groups = (rows + DEC_ROWS - 1) / DEC_ROWS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *s_x = smem + P.x_off;
    int *s_acc = reinterpret_cast<int *>(smem + P.acc_off);

    // The weights are static: one thread requests the CTA's rows (one bulk
    // copy per group, each with its own mbarrier) before the wait below.  It
    // is lane 0 of the last warp, so that the first warps start staging the
    // activations at once.
    const int kch = pr.kch;
    const int WS = kch > 1 ? DEC_KCH_B : RB;  // shared-memory row stride of the weights
    const u64 policy = l2_policy_evict_first();  // read once per launch
    // chunk c of the single group (kch > 1): row r's bytes [c DEC_KCH_B, ...)
    // by lane r of the last warp, after lane 0 has set the expected bytes
    auto request_chunk = [&](int c) {
        const u32 cb = (u32)min(DEC_KCH_B, RB - c * DEC_KCH_B);
        const u32 bar = smem_u32(&s_bar[0]);
        if (lane == 0) mbar_arrive_expect_tx(bar, cb * (u32)rows);
        __syncwarp();
        if (lane < rows)
            bulk_g2s_hint(smem_u32(smem + lane * DEC_KCH_B), pr.packed + (size_t)(rbase + lane) * RB + (size_t)c * DEC_KCH_B,
                          cb, bar, policy);
    };
    if (warp == DEC_WARPS - 1) {
        if (lane == 0) {
            for (int i = 0; i < groups; ++i) mbar_init(smem_u32(&s_bar[i]), 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        if (kch > 1) {
            request_chunk(0);
        } else if (lane == 0) {
            const uint8_t *src = pr.packed + (size_t)rbase * RB;
            const u32 dst = smem_u32(smem);
            for (int i = 0; i < groups; ++i) {
                const u32 bytes = (u32)min(DEC_ROWS, rows - DEC_ROWS * i) * (u32)RB;
                const u32 bar = smem_u32(&s_bar[i]);
                mbar_arrive_expect_tx(bar, bytes);
                const u32 off0 = (u32)(DEC_ROWS * i) * (u32)RB;
                for (u32 off = 0; off < bytes; off += 32768u)
                    bulk_g2s_hint(dst + off0 + off, src + off0 + off, bytes - off < 32768u ? bytes - off : 32768u,
                                  bar, policy);
            }
        }
    }
    if (threadIdx.x == 0) {
        DecSlot &d = s_sl[0];
        d.x = pr.x;
        d.s = pr.s;
        d.gain = pr.gain;
        d.xq_out = pr.xq_out;
        d.K = K;
        d.first = rbase == 0;
        s_xoff[0] = 0;
        s_xoff[1] = M * dec_row_stride(K);
        s_vbase[0] = 0;
        s_vbase[1] = M * (K / (SRC == DEC_SRC_F32 ? 4 : 8));
    }
    if (threadIdx.x == 32) s_gam[0] = *pr.gamma;
    if (threadIdx.x < 16) {
        s_amax[threadIdx.x] = 0u;
        s_rs[threadIdx.x] = 0;
    }
    if (G > 1)
        for (int i = threadIdx.x; i < T * DEC_ROWS * M; i += DEC_THREADS) s_acc[i] = 0;
    __syncthreads();

    // x_q and s may be produced by the kernel launched just before this one.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- activations, staged (and quantized) -------------------------------
    const int RS = dec_row_stride(K);
    if (SRC != DEC_SRC_XQ) {
        constexpr bool BF16 = SRC == DEC_SRC_BF16;
        if (pr.gain == nullptr) {
            if (K <= DEC_RJ * 32 * (BF16 ? 8 : 4))
                dec_quant_rows<BF16>(s_sl, 1, M, s_x, s_xoff, s_gam, s_f, s_rs, warp, lane);
            else
                dec_quant_block<BF16>(s_sl, 1, M, s_xoff, s_vbase, s_x, s_amax, s_sc, s_gam, s_f, s_rs);
        } else {
            for (int m = warp; m < M; m += DEC_WARPS) {
                const float s = dec_quant_row<BF16>(s_sl[0], m, K, RS, s_x, P.eps, s_sl[0].first, lane, &s_rs[m]);
                if (lane == 0) s_f[0][m] = __fdiv_rn(s_gam[0], s);
            }
        }
        // zero the padding chunks K .. round_up(K, 256) of every row
        for (int m = warp; m < M; m += DEC_WARPS)
            for (int L = (K >> 4) + lane; L < (RS >> 4); L += 32) {
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                *reinterpret_cast<uint4 *>(s_x + m * RS + (((L & ~7) | ((L ^ x) & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            }
    } else {
        // plain loads, a warp per row
        for (int m = warp; m < M; m += DEC_WARPS) {
            const int8_t *src = static_cast<const int8_t *>(pr.x) + (size_t)m * K;
            int sum = 0;
            for (int L = lane; L < (RS >> 4); L += 32) {
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                const uint4 v = L < (K >> 4) ? ldg_nc_v4(src + L * 16) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(s_x + m * RS + (((L & ~7) | ((L ^ x) & 7)) << 4)) = v;
                sum = __dp4a((int)v.x, 0x01010101, sum);
                sum = __dp4a((int)v.y, 0x01010101, sum);
                sum = __dp4a((int)v.z, 0x01010101, sum);
                sum = __dp4a((int)v.w, 0x01010101, sum);
            }
            sum = __reduce_add_sync(0xffffffffu, sum);
            if (lane == 0) {
                s_rs[m] = sum;
                s_f[0][m] = __fdiv_rn(s_gam[0], pr.s[m]);
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------------------- the GEMV
    const int g8 = lane >> 2, t = lane & 3;
    const int xb = ((t >> 1) << 1) | (g8 & 1);  // x_q swizzle of this lane's token rows
    const int wg = warp >> glog, kslot = warp & (G - 1);
    bool ok = true;
    int acc[2][NT][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[u][nt][i] = 0;
    const int steps = dec_nsteps(K);
    const int SC = kch > 1 ? DEC_KCH_B / 64 : steps;  // steps per chunk
    // rows g8 + 8a of the group; a step's slice of a row past its end reads
    // the next row's bytes (or the padding): their k are past K, where x_q is
    // zero
    const uint8_t *w0 = smem + (wg * DEC_ROWS + g8) * WS + t * 16;
    const uint8_t *xr[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xr[nt] = s_x + min(g8 + 8 * nt, M - 1) * RS + t * 64;
    int last_c = 0;  // last chunk requested
    for (int c = 0; c < kch; ++c) {
        if (wg < groups) {
            ok = ok && __all_sync(0xffffffffu, mbar_wait(smem_u32(&s_bar[wg]), (u32)(c & 1), DEC_TIMEOUT_NS, nullptr));
            if (!ok && lane == 0) raise_device_error(DEVERR_TIMEOUT_PRODUCER);
        }
        if (ok && wg < groups) {
            const int st_end = min(steps, (c + 1) * SC);
#pragma unroll 1
            for (int st = c * SC + kslot; st < st_end; st += G) {
                const int so = (st - c * SC) * 64;
                uint4 wv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) wv[a] = *reinterpret_cast<const uint4 *>(w0 + a * 8 * WS + so);
                uint4 xv[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        xv[nt][q] = *reinterpret_cast<const uint4 *>(xr[nt] + st * 256 + ((q ^ xb) << 4));
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const u32 wa0 = (&wv[2 * u].x)[2 * hh], wa2 = (&wv[2 * u].x)[2 * hh + 1];
                        const u32 wa1 = (&wv[2 * u + 1].x)[2 * hh], wa3 = (&wv[2 * u + 1].x)[2 * hh + 1];
#pragma unroll
                        for (int jp = 0; jp < 4; ++jp) {
                            const u32 a0 = dec_plane_top(wa0, jp), a1 = dec_plane_top(wa1, jp);
                            const u32 a2 = dec_plane_top(wa2, jp), a3 = dec_plane_top(wa3, jp);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_u8s8_16832(acc[u][nt], a0, a1, a2, a3, (&xv[nt][2 * hh].x)[jp],
                                               (&xv[nt][2 * hh + 1].x)[jp]);
                        }
                    }
            }
        }
        if (c + 1 < kch) {
            // every warp is done with this chunk before the next one lands
            __syncthreads();
            if (warp == DEC_WARPS - 1 && ok) {
                request_chunk(c + 1);
                last_c = c + 1;
            }
        }
    }
    if (ok && wg < groups) {
        // this warp's sums of 64 c x into the CTA's [row][token] table (the
        // only writer when G == 1)
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = 8 * nt + 2 * t + (i & 1);
                    const int r = wg * DEC_ROWS + g8 + 16 * u + 8 * (i >> 1);
                    if (m < M) {
                        if (G == 1)
                            s_acc[r * M + m] = acc[u][nt][i];
                        else
                            atomicAdd(&s_acc[r * M + m], acc[u][nt][i]);
                    }
                }
    }
    __syncthreads();
    // Y[m, rbase + r] = (sum_k x - (sum_k 64 c x) / 64) * (gamma / s[m]); 32
    // consecutive rows per warp and token
    float *Y = pr.Y;
    int32_t *accp = pr.acc;
    const int TR = T * DEC_ROWS;
    for (int e = threadIdx.x; e < M * TR; e += DEC_THREADS) {
        const int m = e / TR, r = e - m * TR;
        if (r < rows) {
            const int a_ = s_rs[m] - (s_acc[r * M + m] >> 6);
            Y[(size_t)m * N + rbase + r] = __fmul_rn(__int2float_rn(a_), s_f[0][m]);
            if (accp) accp[(size_t)m * N + rbase + r] = a_;
        }
    }
    // a wait that gave up: the copies still in flight land (bounded) before
    // the CTA exits
    if (__syncthreads_or(!ok) && threadIdx.x == DEC_THREADS - 32) {
        if (kch > 1)
            mbar_wait(smem_u32(&s_bar[0]), (u32)(last_c & 1), DEC_TIMEOUT_NS, nullptr);
        else
            for (int i = 0; i < groups; ++i) mbar_wait(smem_u32(&s_bar[i]), 0, DEC_TIMEOUT_NS, nullptr);
    }
}

}  // namespace bl
