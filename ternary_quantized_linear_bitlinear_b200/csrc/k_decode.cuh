// Steps 3 + 4 for decode-sized M (<= 16): the ternary x INT8 GEMV engine.
//
// What it computes ("bitone" README, How 1.58-bit Works and Forward pass):
//   acc[m, n] = sum_k x_q[m, k] * W_q[n, k];  Y[m, n] = acc * (gamma / s[m])
//
// The work is bound by streaming the packed weights from HBM (2 bits per
// weight).  Design (one CTA per SM and launch, small enough that the CTA of
// the next launch fits beside it):
//   - Work unit: a group of 32 weight rows of one problem.  The host cuts the
//     flattened group list of all problems into one contiguous range per CTA
//     with about equal packed bytes.  Inside the CTA every warp takes whole
//     groups: its first one by its index, the next ones from a shared
//     counter as it needs them, so warps that meet short groups take more.
//   - Streaming: each warp owns a ring of DEC_WSTAGES shared-memory stages.
//     Its lane 0 cuts its groups into chunks of 32 rows x 128 bytes (512 k)
//     and requests each with a 2-D TMA tensor load (per-problem tensor map,
//     128-byte swizzle, L2 evict-first: each byte is read once) as soon as
//     the warp has consumed the stage, DEC_WSTAGES chunks ahead of its
//     compute; the first requests go out before griddepcontrol.wait, so a
//     programmatic dependent launch (BL_FWD_WEIGHTS_READY) streams its
//     weights while the launch before it finishes.  A warp consumes only its
//     own stages, in order: no cross-warp synchronization on the stream.
//   - MACs on the tensor cores (mma.sync m16n8k32 s8): weight rows as A (two
//     16-row tiles per chunk share every x_q fragment), tokens as B (8
//     columns per tile, zero for m >= M).  The int32 sum is exact, so the k
//     order inside a 256-k step may be permuted as long as A and B use the
//     same permutation: the lane with k-slot t holds the packed bytes
//     64t .. 64t + 15 of the step, and its B fragment reads those x_q bytes.
//     A group's accumulators stay in the warp's registers over its chunks;
//     the warp rescales them and writes Y when the group's last chunk is in.
//   - Unpacking costs one AND per 4 weights: a packed word holds the codes
//     c = 1 - W_q in {0, 1, 2}; word & (0x03030303 << 2j) leaves the codes of
//     k = 16w' + 4j .. 4j+3 in four bytes as the unsigned values 4^j c, which
//     the MMA takes as u8 (A) against the s8 activations (B), one accumulator
//     per plane j.  Then sum_k W_q x = sum_k x - sum_j D_j / 4^j (each D_j a
//     multiple of 4^j, so the shifts are exact), with sum_k x the row sum of
//     the staged x_q.  At M > 8 (two token tiles) the planes are moved to the
//     top two bits instead ((w << (6 - 2j)) & 0xC0C0C0C0, 64 c) and share one
//     accumulator per tile, to keep the registers of the second tile.
//   - Lane (g, t) of an MMA tile reads weight rows pi(g) and pi(g) + 8 with
//     pi(g) = (g >> 1) | ((g & 1) << 2): with the 128-byte swizzle, the eight
//     lanes of each quarter warp then hit eight different bank quads.
//   - x_q is staged once per CTA and problem in shared memory (rows of
//     round_up(K, 256) bytes, 16-byte chunks XOR-swizzled so that the B loads
//     are free of bank conflicts).  Fused variant (SRC = bf16 or f32
//     activations): step 2 runs inside the CTA with the same arithmetic as
//     the stand-alone activation quantizer (rows without SubLN by the whole
//     CTA at once, SubLN rows one warp per row); the CTA holding a problem's
//     first group also writes x_q and s on request.
//   - Every mbarrier wait is bounded (globaltimer); a wait that gives up
//     raises the device error word and the CTA's abort flag, and each warp
//     then waits (bounded) for its own copies in flight before it exits.
#pragma once

#include <cuda.h>

#include "bl_common.cuh"

namespace bl {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_ROWS = 32;                          // weight rows per group (two MMA tiles)
constexpr int DEC_CB = 128;                           // packed bytes per row per chunk (512 k)
constexpr int DEC_CHUNK = DEC_ROWS * DEC_CB;          // 4 KiB
constexpr int DEC_WSTAGES = 2;                        // ring stages per warp
constexpr int DEC_MAX_PSLOTS = 8;                     // problems per CTA
constexpr int DEC_MAX_CTAS = 320;
constexpr int DEC_X_MAX = 144 * 1024;                 // staged activations per CTA
constexpr int DEC_X_PAIR = 36 * 1024;                 // ... at most this keeps two CTAs per SM
constexpr unsigned long long DEC_TIMEOUT_NS = 2000000000ull;

__host__ __device__ constexpr int dec_fixed_smem(int) { return DEC_WARPS * DEC_WSTAGES * DEC_CHUNK; }

// Activation source of a launch: pre-quantized x_q, or X to quantize in-kernel.
enum : int { DEC_SRC_XQ = 0, DEC_SRC_BF16 = 1, DEC_SRC_F32 = 2 };

struct DecodeProblem {
    const float *gamma;
    const void *x;         // DEC_SRC_XQ: x_q [M, K] int8; else X [M, K] bf16 / f32
    float *s;              // DEC_SRC_XQ: s [M] in; else s [M] out or null
    float *Y;
    int32_t *acc;
    const float *gain;     // fused: SubLN gain [K] or null
    int8_t *xq_out;        // fused: x_q [M, K] out or null
    int N;
    int K;
    int gbase;             // first group of this problem in the flattened group list
};

struct DecodeParams {
    CUtensorMap wmap[BL_MAX_GROUP];  // packed weights per problem: {K/4 bytes, N rows}, box 128 x 32, 128B swizzle
    DecodeProblem p[BL_MAX_GROUP];
    int count;
    int M;
    int ngroups;
    int ncta;
    float eps;                        // fused: SubLN epsilon
    int cta_g[DEC_MAX_CTAS + 1];      // CTA c owns groups [cta_g[c], cta_g[c + 1])
};

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
__device__ float dec_quant_row(const DecodeProblem &pr, int m, int K, int RS, uint8_t *s_xq, float eps, bool out,
                               int lane, int *rowsum) {
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
// every thread takes the 16-byte vectors t, t + DEC_THREADS, ... of the
// concatenated rows with all its loads in flight together (one memory round
// trip for the CTA instead of one per row and warp), the row maxima meet in
// shared memory (max of the float bits of |x|), and each thread then
// quantizes its vectors into the staging rows.  Same arithmetic as
// dec_quant_row.  vbase[ps] = first vector of problem slot ps (vbase[np] =
// the total, at most DEC_QBV * DEC_THREADS); s_amax[np * M] zeroed before.
constexpr int DEC_QBV = 12;

template <bool BF16>
__device__ void dec_quant_block(const DecodeParams &P, int p_lo, int np, int g_begin, const int *s_xoff,
                                const int *vbase, uint8_t *s_x, u32 *s_amax, float *s_sc, float (*s_f)[16],
                                int *s_rs) {
    constexpr int EPV = BF16 ? 8 : 4;
    const int M = P.M, T = vbase[np];
    const int lane = threadIdx.x & 31;
    uint4 c[DEC_QBV];
    int meta[DEC_QBV];  // (slot << 20) | (m << 16) | vector within the row; -1 past the end
#pragma unroll
    for (int i = 0; i < DEC_QBV; ++i) {
        const int idx = (int)threadIdx.x + DEC_THREADS * i;
        meta[i] = -1;
        c[i] = make_uint4(0, 0, 0, 0);
        if (idx < T) {
            int ps = 0;
            while (ps + 1 < np && idx >= vbase[ps + 1]) ++ps;
            const int nvec = P.p[p_lo + ps].K / EPV;
            const int local = idx - vbase[ps];
            const int m = local / nvec, v = local - m * nvec;
            meta[i] = (ps << 20) | (m << 16) | v;
            c[i] = ldg_nc_v4(reinterpret_cast<const uint4 *>(P.p[p_lo + ps].x) + (size_t)m * nvec + v);
        }
    }
#pragma unroll
    for (int i = 0; i < DEC_QBV; ++i) {
        if (DEC_THREADS * i >= T) break;  // uniform: no vector of this round is in range
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
    __syncthreads();
    for (int r = threadIdx.x; r < np * M; r += DEC_THREADS) {
        const int ps = r / M, m = r - ps * M;
        const DecodeProblem &pr = P.p[p_lo + ps];
        const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(s_amax[r]), 1e-5f));
        s_sc[r] = s;
        s_f[ps][m] = __fdiv_rn(*pr.gamma, s);
        if (g_begin <= pr.gbase && pr.s != nullptr) pr.s[m] = s;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < DEC_QBV; ++i) {
        if (DEC_THREADS * i >= T) break;  // uniform: no vector of this round is in range
        int rsum = 0;
        const int row = meta[i] < 0 ? -1 : ((meta[i] >> 20) * M + ((meta[i] >> 16) & 15));
        if (meta[i] >= 0) {
        const int ps = meta[i] >> 20, m = (meta[i] >> 16) & 15, v = meta[i] & 0xffff;
        const DecodeProblem &pr = P.p[p_lo + ps];
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
        int8_t *gq = (g_begin <= pr.gbase && pr.xq_out != nullptr) ? pr.xq_out + (size_t)m * K : nullptr;
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
            if ((threadIdx.x & 31) == 0 && row0 >= 0) atomicAdd(&s_rs[row0], rsum);
        } else if (row >= 0) {
            atomicAdd(&s_rs[row], rsum);
        }
    }
}

// problem owning flattened group g (binary search over the group bases)
__device__ __forceinline__ int dec_problem_of(const DecodeParams &P, int g) {
    int lo = 0, hi = P.count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.p[mid].gbase <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int dec_nchunks(int K) { return (K + 4 * DEC_CB - 1) / (4 * DEC_CB); }

__device__ __forceinline__ void tma_load_2d_hint(u32 dst, const CUtensorMap *map, int x, int y, u32 bar, u64 pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}

// NT: 8-token column tiles (1: M <= 8, 2: M <= 16).  SRC: DEC_SRC_*.
template <int NT, int SRC>
__global__ void __launch_bounds__(DEC_THREADS, 2) k_decode(const __grid_constant__ DecodeParams P) {
    extern __shared__ uint8_t dsm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) u64 s_full[DEC_WARPS][DEC_WSTAGES];
    __shared__ int s_queue[DEC_WARPS][DEC_WSTAGES + 2];  // groups a warp has started requesting, in order
    __shared__ int s_next;                               // next group to hand out
    __shared__ float s_f[DEC_MAX_PSLOTS][16];
    __shared__ int s_xoff[DEC_MAX_PSLOTS + 1];
    __shared__ int s_vbase[DEC_MAX_PSLOTS + 1];
    __shared__ u32 s_amax[DEC_MAX_PSLOTS * 16];
    __shared__ float s_sc[DEC_MAX_PSLOTS * 16];
    __shared__ int s_rs[DEC_MAX_PSLOTS * 16];  // row sums of the staged x_q
    __shared__ volatile int s_abort;

    // a programmatically dependent launch that follows may start its prologue
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    constexpr int QN = DEC_WSTAGES + 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g_begin = P.cta_g[blockIdx.x], g_end = P.cta_g[blockIdx.x + 1];
    const int p_lo = dec_problem_of(P, g_begin), p_hi = dec_problem_of(P, g_end - 1);
    const int np = p_hi - p_lo + 1;
    const int M = P.M;
    uint8_t *s_x = sm + dec_fixed_smem(NT);

    if (threadIdx.x == 0) {
        for (int w = 0; w < DEC_WARPS; ++w)
            for (int s = 0; s < DEC_WSTAGES; ++s) mbar_init(smem_u32(&s_full[w][s]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
        s_next = g_begin + DEC_WARPS;
        int off = 0, vb = 0;
        for (int i = 0; i < np; ++i) {
            s_xoff[i] = off;
            s_vbase[i] = vb;
            off += M * dec_row_stride(P.p[p_lo + i].K);
            vb += M * (P.p[p_lo + i].K / (SRC == DEC_SRC_F32 ? 4 : 8));
        }
        s_xoff[np] = off;
        s_vbase[np] = vb;
    }
    if (threadIdx.x < DEC_MAX_PSLOTS * 16) {
        s_amax[threadIdx.x] = 0u;
        s_rs[threadIdx.x] = 0;
    }
    __syncthreads();

    // ---- this warp's request stream: its groups' chunks, in order ---------
    // (warp-uniform state; lane 0 issues the copies)
    uint8_t *ring = sm + warp * (DEC_WSTAGES * DEC_CHUNK);
    const u64 policy = l2_policy_evict_first();
    int i_g = -1, i_p = p_lo, i_k = 0, i_nch = 0;  // request cursor: group, problem, chunk, chunks of group
    int q_tail = 0;                                // groups queued for the consumer side
    long long issued = 0;
    auto next_group = [&]() -> int {
        int g;
        if (i_g < 0) {
            g = g_begin + warp;
        } else {
            g = 0;
            if (lane == 0) g = atomicAdd(&s_next, 1);
            g = __shfl_sync(0xffffffffu, g, 0);
        }
        return g < g_end ? g : -2;
    };
    auto issue_next = [&]() {
        if (i_g == -2) return;
        if (i_g < 0 || i_k == i_nch) {
            const int g = next_group();
            if (g < 0) {
                i_g = -2;
                return;
            }
            while (i_p + 1 < P.count && g >= P.p[i_p + 1].gbase) ++i_p;
            i_g = g;
            i_k = 0;
            i_nch = dec_nchunks(P.p[i_p].K);
            s_queue[warp][q_tail % QN] = g;  // every lane writes (and later reads) its own copy
            ++q_tail;
        }
        const int s = (int)(issued % DEC_WSTAGES);
        if (lane == 0) {
            const u32 bar = smem_u32(&s_full[warp][s]);
            mbar_arrive_expect_tx(bar, DEC_CHUNK);
            tma_load_2d_hint(smem_u32(ring + s * DEC_CHUNK), &P.wmap[i_p], i_k * DEC_CB,
                             (i_g - P.p[i_p].gbase) * DEC_ROWS, bar, policy);
        }
        ++i_k;
        ++issued;
    };
    if (lane == 0)
        for (int p = p_lo; p <= p_hi; ++p) asm volatile("prefetch.tensormap [%0];" ::"l"(&P.wmap[p]) : "memory");
    for (int i = 0; i < DEC_WSTAGES; ++i) issue_next();

    // x_q and s may be produced by the kernel launched just before this one.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- activations of this CTA's problems, staged (and quantized) --------
    bool block_quant = false;
    if (SRC != DEC_SRC_XQ) {
        bool gain = false;
        for (int i = 0; i < np; ++i) gain |= P.p[p_lo + i].gain != nullptr;
        block_quant = !gain && s_vbase[np] <= DEC_QBV * DEC_THREADS;
    }
    if (block_quant) {
        dec_quant_block<SRC == DEC_SRC_BF16>(P, p_lo, np, g_begin, s_xoff, s_vbase, s_x, s_amax, s_sc, s_f, s_rs);
        // zero the padding chunks K .. round_up(K, 256) of every row
        for (int r = warp; r < np * M; r += DEC_WARPS) {
            const int ps = r / M, m = r - ps * M;
            const int K = P.p[p_lo + ps].K, RS = dec_row_stride(K);
            uint8_t *xs = s_x + s_xoff[ps];
            for (int L = (K >> 4) + lane; L < (RS >> 4); L += 32) {
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                *reinterpret_cast<uint4 *>(xs + m * RS + (((L & ~7) | ((L ^ x) & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            }
        }
    }
    for (int r = warp; r < (block_quant ? 0 : np * M); r += DEC_WARPS) {
        const int ps = r / M, m = r - ps * M;
        const DecodeProblem &pr = P.p[p_lo + ps];
        const int K = pr.K, RS = dec_row_stride(K);
        uint8_t *xs = s_x + s_xoff[ps];
        if (SRC != DEC_SRC_XQ) {
            constexpr bool BF16 = SRC == DEC_SRC_BF16;
            const bool out = g_begin <= pr.gbase;  // this CTA holds the problem's first group
            const float s = dec_quant_row<BF16>(pr, m, K, RS, xs, P.eps, out, lane, &s_rs[ps * M + m]);
            if (lane == 0) s_f[ps][m] = __fdiv_rn(*pr.gamma, s);
            for (int L = (K >> 4) + lane; L < (RS >> 4); L += 32) {
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                *reinterpret_cast<uint4 *>(xs + m * RS + (((L & ~7) | ((L ^ x) & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            }
        } else {
            const int8_t *src = static_cast<const int8_t *>(pr.x) + (size_t)m * K;
            for (int L = lane; L < (RS >> 4); L += 32) {
                const int x = (((L >> 3) & 1) << 1) | (m & 1);
                uint8_t *d = xs + m * RS + (((L & ~7) | ((L ^ x) & 7)) << 4);
                if (L < (K >> 4))
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(d)), "l"(src + L * 16)
                                 : "memory");
                else
                    *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
            }
            if (lane == 0) s_f[ps][m] = __fdiv_rn(*pr.gamma, pr.s[m]);
        }
    }
    if (SRC == DEC_SRC_XQ) {
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        // row sums of the staged x_q (the padding is zero; the order of the
        // 16-byte chunks does not matter)
        for (int r = warp; r < np * M; r += DEC_WARPS) {
            const int ps = r / M, m = r - ps * M;
            const int RS = dec_row_stride(P.p[p_lo + ps].K);
            const uint4 *row = reinterpret_cast<const uint4 *>(s_x + s_xoff[ps] + m * RS);
            int sum = 0;
            for (int L = lane; L < (RS >> 4); L += 32) {
                const uint4 v = row[L];
                sum = __dp4a((int)v.x, 0x01010101, sum);
                sum = __dp4a((int)v.y, 0x01010101, sum);
                sum = __dp4a((int)v.z, 0x01010101, sum);
                sum = __dp4a((int)v.w, 0x01010101, sum);
            }
            sum = __reduce_add_sync(0xffffffffu, sum);
            if (lane == 0) s_rs[r] = sum;
        }
    }
    __syncthreads();

    // ------------------------------------------------------------- consumers
    const int g8 = lane >> 2, t = lane & 3;
    const int pg = (g8 >> 1) | ((g8 & 1) << 2);       // physical row phase of MMA row g8
    const int xb = ((t >> 1) << 1) | (g8 & 1);        // x_q swizzle of this lane's token rows
    // M <= 8: one accumulator per code plane and tile (plane j at scale 4^j);
    // M <= 16: the planes moved to scale 64, one accumulator per tile
    constexpr int PL = NT == 1 ? 4 : 1;
    long long consumed = 0;
    int q_head = 0, c_p = p_lo;
    bool ok = true;
    while (ok && q_head < q_tail) {
        const int g = s_queue[warp][q_head % QN];
        ++q_head;
        while (c_p + 1 < P.count && g >= P.p[c_p + 1].gbase) ++c_p;
        const DecodeProblem &pr = P.p[c_p];
        const int ps = c_p - p_lo;
        const int K = pr.K, RS = dec_row_stride(K);
        const uint8_t *xs = s_x + s_xoff[ps];
        const int nch = dec_nchunks(K);
        int acc[PL][2][NT][4];
#pragma unroll
        for (int c = 0; c < PL; ++c)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[c][u][nt][i] = 0;
        for (int kc = 0; kc < nch; ++kc, ++consumed) {
            const int s = (int)(consumed % DEC_WSTAGES);
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&s_full[warp][s]), (u32)((consumed / DEC_WSTAGES) & 1),
                                                  DEC_TIMEOUT_NS, &s_abort));
            if (!ok) {
                if (lane == 0) {
                    raise_device_error(DEVERR_TIMEOUT_MMA);
                    s_abort = 1;
                }
                break;
            }
            const int vb = min(DEC_CB, (K >> 2) - kc * DEC_CB);  // valid packed bytes per row (>= 16)
            const uint8_t *st = ring + s * DEC_CHUNK;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                if (64 * h2 >= vb) break;
                // weights: physical rows pg + 8a (a = 0..3), this lane's 16 bytes of the half
                uint4 wv[4];
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    wv[a] = *reinterpret_cast<const uint4 *>(st + (pg + 8 * a) * DEC_CB + (((4 * h2 + t) ^ pg) << 4));
                // x_q of tokens g8 (+ 8): the 64 bytes of k-slot t in 256-k step s2
                const int s2 = 2 * kc + h2;
                uint4 xv[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int m = g8 + 8 * nt;
                    const uint8_t *xr = xs + m * RS + s2 * 256 + t * 64;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        xv[nt][c] = m < M ? *reinterpret_cast<const uint4 *>(xr + ((c ^ xb) << 4))
                                          : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const u32 wa0 = (&wv[2 * u].x)[2 * hh], wa2 = (&wv[2 * u].x)[2 * hh + 1];
                        const u32 wa1 = (&wv[2 * u + 1].x)[2 * hh], wa3 = (&wv[2 * u + 1].x)[2 * hh + 1];
#pragma unroll
                        for (int jp = 0; jp < 4; ++jp) {
                            u32 a0, a1, a2, a3;
                            if (PL == 4) {
                                a0 = dec_plane(wa0, jp);
                                a1 = dec_plane(wa1, jp);
                                a2 = dec_plane(wa2, jp);
                                a3 = dec_plane(wa3, jp);
                            } else {
                                a0 = dec_plane_top(wa0, jp);
                                a1 = dec_plane_top(wa1, jp);
                                a2 = dec_plane_top(wa2, jp);
                                a3 = dec_plane_top(wa3, jp);
                            }
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_u8s8_16832(acc[jp % PL][u][nt], a0, a1, a2, a3, (&xv[nt][2 * hh].x)[jp],
                                               (&xv[nt][2 * hh + 1].x)[jp]);
                        }
                    }
                }
            }
            // the stage is free again: request this warp's next chunk into it
            __syncwarp();
            issue_next();
        }
        if (!ok) break;
        // epilogue: rows pg + 16u + 8(i >> 1), tokens 8nt + 2t + (i & 1)
        const int n_base = (g - pr.gbase) * DEC_ROWS + pg;
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = 8 * nt + 2 * t + (i & 1);
                    const int n = n_base + 16 * u + 8 * (i >> 1);
                    if (m < M && n < pr.N) {
                        // sum_k c x with c = 1 - W_q, each plane's sum a multiple of its scale
                        const int cx = PL == 4 ? acc[0][u][nt][i] + (acc[PL > 1 ? 1 : 0][u][nt][i] >> 2) +
                                                     (acc[PL > 2 ? 2 : 0][u][nt][i] >> 4) +
                                                     (acc[PL > 3 ? 3 : 0][u][nt][i] >> 6)
                                               : acc[0][u][nt][i] >> 6;
                        const int a_ = s_rs[ps * M + m] - cx;
                        pr.Y[(size_t)m * pr.N + n] = __fmul_rn(__int2float_rn(a_), s_f[ps][m]);
                        if (pr.acc) pr.acc[(size_t)m * pr.N + n] = a_;
                    }
                }
    }
    if (!ok) {
        // drain: this warp's copies in flight land before it exits
        for (long long j = consumed; j < issued; ++j)
            mbar_wait(smem_u32(&s_full[warp][(int)(j % DEC_WSTAGES)]), (u32)((j / DEC_WSTAGES) & 1), DEC_TIMEOUT_NS,
                      nullptr);
    }
}

}  // namespace bl
