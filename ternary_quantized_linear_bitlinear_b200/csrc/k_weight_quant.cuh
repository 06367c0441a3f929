// Step 1 of the BitLinear forward: absmean ternary weight quantization and
// 2-bit packing ("Distillix" README, 1. BitNet b1.58 Core; "bitone" README,
// Forward pass; "SLM750-Edge" section 3.1).
//
// Three launches on the caller's stream, each over one or several weight
// matrices (up to WQ_MAX_JOBS: e.g. the projections of a layer, so their
// reduction latency chains overlap), chained as programmatic dependents:
//   k_absmean_partial  one pass over W: each block's sum of |w| in double
//   k_absmean_final    one CTA per matrix: gamma = float(double(S) / n) +
//                      1e-5f for the exact S = sum |w| and the float
//                      threshold T with |w| >= T <=> float(|w|/gamma) > 0.5
//   k_ternary_pack     second pass over W (its first words requested before
//                      the wait for T): W_q = sign(w) * (|w| >= T), stored
//                      as the code 1 - W_q, four codes per byte in the
//                      packed word layout
// No CTA waits on another CTA of its own launch, and nothing in the
// workspace needs clearing: every word a launch reads there was written by
// the launch before it.
//
// gamma from a double estimate.  A float is exact in double, so the sum of
// |w| in double, S_hat, is within beta * S_hat of the sum of its terms when
// no term passes through more than D roundings on its way to the total
// (beta = 2 D 2^-53 for a non-negative sum; D is the longest chain of a
// thread plus the reduction tree, counted on the host).  The terms are the
// exact |w| except that zero and subnormal w enter as values below 2^-126
// (no per-element test), i.e. within A = n 2^-126 above S.  gamma is
// monotone in S, so when both ends of [S_hat (1 - beta) - A, S_hat (1 + beta)]
// give the same gamma that is gamma(S), bit for bit (tiny sums, e.g. an
// all-zero matrix, give 1e-5f at both ends).  Otherwise -- the mean within
// about 10^-14 of a float rounding boundary, or S_hat >= 2^127 (inf / NaN
// weights) -- the final CTA sums |w| exactly: every finite float is an
// integer multiple of 2^-149, so S is an integer in those units; each thread
// adds m << (e - base) for exponents in a 26-binade window chosen from a
// sample of the matrix into 128 bits, anything outside the window into exact
// shared-memory bins by exponent, and the block folds it all into 384-bit
// limbs, rounded once to double.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int WQ_THREADS = 512;
constexpr int WQ_PACK_THREADS = 256;
constexpr int WQ_WINDOW = 25;       // exact sum: base <= e <= base + 25
constexpr int WQ_PART_LIMBS = 6;    // workspace words per reduction block (one double used)
constexpr int WQ_MAX_BLOCKS = 1024; // over all matrices of a launch
constexpr int WQ_MAX_JOBS = 8;      // weight matrices per launch
constexpr size_t WQ_WS_PARTIALS = (size_t)WQ_MAX_BLOCKS * WQ_PART_LIMBS * 8;
constexpr size_t WQ_WS_BYTES = WQ_WS_PARTIALS + 256;  // + threshold words

// One weight matrix of a (grouped) quantization launch: blocks
// [blk0, blk0 + nblk) of the reduction grid sum it, block j of the final
// grid derives its gamma and T, blocks [pblk0, pblk0 + pnblk) of the pack
// grid pack it.  depth bounds the roundings any term of its double sum
// passes through.
struct WqJob {
    const uint4 *W;
    long long nvec;   // 16-byte vectors
    long long n;      // weights
    float *gamma;
    u32 *packed;
    long long nwords; // packed 32-bit words (16 weights each)
    int blk0;
    int nblk;
    int pblk0;
    int pnblk;
    int depth;
};

struct WqParams {
    WqJob j[WQ_MAX_JOBS];
    int count;
    u64 *partials;    // [WQ_MAX_BLOCKS][WQ_PART_LIMBS]: word 0 of a block holds its double sum
    u32 *thresh;      // [WQ_MAX_JOBS] float bits of T
};

// Float bits of the j-th element of a 16-byte vector.
template <bool BF16>
__device__ __forceinline__ u32 vec_elem_bits(const uint4 &v, int j) {
    const u32 w[4] = {v.x, v.y, v.z, v.w};
    if (BF16) {
        u32 word = w[j >> 1];
        return (j & 1) ? (word & 0xffff0000u) : (word << 16);
    } else {
        return w[j];
    }
}

// gamma = float(S / n) + 1e-5f (S already rounded to double) and the
// smallest float t with float(t / gamma) > 0.5.
__device__ __forceinline__ void wq_gamma_threshold_of(double S, long long n, float *g_out, u32 *t_out) {
    const float mean = __double2float_rn(__ddiv_rn(S, (double)n));
    const float g = __fadd_rn(mean, 1e-5f);
    // start at g/2 (exact, quotient 0.5)
    float t = __fmul_rn(0.5f, g);
    for (int it = 0; it < 64 && !(__fdiv_rn(t, g) > 0.5f); ++it) t = __uint_as_float(__float_as_uint(t) + 1u);
    *g_out = g;
    *t_out = __float_as_uint(t);
}

// Exact sum of |w| over vectors first, first + stride, ... < nvec by the
// whole block (NT threads), as 384-bit limbs in units of 2^-149 in thread 0.
template <bool BF16, int NT>
__device__ void wq_exact_block_sum(const uint4 *__restrict__ W, long long first, long long stride, long long nvec,
                                   u64 (&L)[WQ_PART_LIMBS]) {
    constexpr int EPV = BF16 ? 8 : 4;
    __shared__ u64 s_bins[256];
    __shared__ u32 s_emax;
    __shared__ u64 s_wlo[NT / 32], s_whi[NT / 32];
    const int tid = threadIdx.x;
    for (int i = tid; i < 256; i += NT) s_bins[i] = 0ull;
    if (tid == 0) s_emax = 0;
    // window from a sample: the first vector per thread
    u32 emax = 0;
    if (first < nvec) {
        const uint4 v = ldg_stream_v4(W + first);
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
            const u32 e = (vec_elem_bits<BF16>(v, j) & 0x7fffffffu) >> 23;
            emax = e > emax ? e : emax;
        }
    }
    emax = warp_max_u32(emax);
    __syncthreads();
    if ((tid & 31) == 0) atomicMax(&s_emax, emax);
    __syncthreads();
    int top = (int)s_emax + 2;
    if (top > 254) top = 254;
    int base = top - WQ_WINDOW;
    if (base < 1) base = 1;
    // 128-bit per-thread sum of m << (e - base) (< 2^49 per term)
    u64 lo = 0ull, hi = 0ull;
    for (long long i = first; i < nvec; i += stride) {
        const uint4 v = ldg_stream_v4(W + i);
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
            const u32 u = vec_elem_bits<BF16>(v, j) & 0x7fffffffu;
            const u32 e = u >> 23;
            const u32 m = (u & 0x7fffffu) | 0x800000u;
            const u32 d = e - (u32)base;
            if (d <= (u32)WQ_WINDOW) {
                const u64 t = (u64)m << d;
                const u64 s2 = lo + t;
                hi += s2 < lo ? 1ull : 0ull;
                lo = s2;
            } else if (u != 0u) {
                atomicAdd(&s_bins[e], (u64)(e ? m : (u & 0x7fffffu)));
            }
        }
    }
    warp_sum_u128(lo, hi);
    if ((tid & 31) == 0) {
        s_wlo[tid >> 5] = lo;
        s_whi[tid >> 5] = hi;
    }
    __syncthreads();
    if (tid == 0) {
#pragma unroll
        for (int k = 0; k < WQ_PART_LIMBS; ++k) L[k] = 0ull;
        for (int w = 0; w < NT / 32; ++w) limbs_add_u128_shl(L, s_wlo[w], s_whi[w], base - 1);
        // term m << (e - base) stands for m * 2^(e - 150) = term * 2^(base - 1) units
        for (int e = 0; e < 256; ++e)
            if (s_bins[e] != 0ull) limbs_add_u128_shl(L, s_bins[e], 0ull, e > 0 ? e - 1 : 0);
    }
}

template <bool BF16>
__global__ void __launch_bounds__(WQ_THREADS, 2) k_absmean_partial(const __grid_constant__ WqParams P) {
    // the next grids may start now (the final grid waits for this one)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int EPV = BF16 ? 8 : 4;
    __shared__ double s_d[WQ_THREADS / 32];
    int ji = 0;
    while (ji + 1 < P.count && (int)blockIdx.x >= P.j[ji + 1].blk0) ++ji;
    const WqJob &job = P.j[ji];
    const uint4 *__restrict__ W = job.W;
    const long long nvec = job.nvec;
    const int tid = threadIdx.x;
    const long long stride = (long long)job.nblk * WQ_THREADS;
    long long i = (long long)((int)blockIdx.x - job.blk0) * WQ_THREADS + tid;
    // two accumulators (even / odd elements of a vector), four vectors in
    // flight while four are summed
    double d0 = 0.0, d1 = 0.0;
    auto add_vec = [&](const uint4 &v) {
#pragma unroll
        for (int j = 0; j < EPV; j += 2) {
            d0 = __dadd_rn(d0, abs_as_double(vec_elem_bits<BF16>(v, j)));
            d1 = __dadd_rn(d1, abs_as_double(vec_elem_bits<BF16>(v, j + 1)));
        }
    };
    uint4 a[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) a[q] = i + q * stride < nvec ? ldg_stream_v4(W + i + q * stride) : make_uint4(0, 0, 0, 0);
    while (i + 4 * stride < nvec) {
        const long long inext = i + 4 * stride;
        uint4 b[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            b[q] = inext + q * stride < nvec ? ldg_stream_v4(W + inext + q * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) add_vec(a[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q) a[q] = b[q];
        i = inext;
    }
    // the last vectors (zeros past the end: 2^-127 each, inside the bound)
#pragma unroll
    for (int q = 0; q < 4; ++q)
        if (i + q * stride < nvec) add_vec(a[q]);
    double d = warp_sum_f64(__dadd_rn(d0, d1));
    if ((tid & 31) == 0) s_d[tid >> 5] = d;
    __syncthreads();
    if (tid == 0) {
        double t = s_d[0];
        for (int w = 1; w < WQ_THREADS / 32; ++w) t = __dadd_rn(t, s_d[w]);
        // read by the final grid after its griddepcontrol.wait
        P.partials[(size_t)blockIdx.x * WQ_PART_LIMBS] = (u64)__double_as_longlong(t);
    }
}

// Block j derives gamma and T of matrix j: from the reduction blocks'
// double sums when their bound decides gamma, else from the exact sum
// (read after the reduction grid has completed).
template <bool BF16>
__global__ void __launch_bounds__(WQ_PACK_THREADS) k_absmean_final(const __grid_constant__ WqParams P) {
    // the pack grid may start loading W now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ double s_d[WQ_PACK_THREADS / 32];
    __shared__ int s_decided;
    __shared__ float s_g;
    __shared__ u32 s_t;
    const WqJob &jb = P.j[blockIdx.x];
    const int tid = threadIdx.x;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    double d = 0.0;
    for (int b = tid; b < jb.nblk; b += WQ_PACK_THREADS)
        d = __dadd_rn(d, __longlong_as_double((long long)__ldcg(P.partials + (size_t)(jb.blk0 + b) * WQ_PART_LIMBS)));
    d = warp_sum_f64(d);
    if ((tid & 31) == 0) s_d[tid >> 5] = d;
    __syncthreads();
    if (tid == 0) {
        double sh = s_d[0];
        for (int w = 1; w < WQ_PACK_THREADS / 32; ++w) sh = __dadd_rn(sh, s_d[w]);
        int decided = 0;
        if (sh < 0x1p127) {
            const double beta = 2.0 * (double)jb.depth * 0x1p-53;
            const double A = (double)jb.n * 0x1p-126;
            double lo = __dsub_rd(__dmul_rd(sh, 1.0 - beta), A);
            lo = lo > 0.0 ? lo : 0.0;
            const double hi = __dmul_ru(sh, 1.0 + beta);
            float glo, ghi;
            u32 tlo, thi;
            wq_gamma_threshold_of(lo, jb.n, &glo, &tlo);
            wq_gamma_threshold_of(hi, jb.n, &ghi, &thi);
            if (__float_as_uint(glo) == __float_as_uint(ghi)) {
                s_g = glo;
                s_t = tlo;
                decided = 1;
            }
        }
        s_decided = decided;
    }
    __syncthreads();
    if (!s_decided) {
        u64 L[WQ_PART_LIMBS];
        wq_exact_block_sum<BF16, WQ_PACK_THREADS>(jb.W, tid, WQ_PACK_THREADS, jb.nvec, L);
        if (tid == 0) {
            u64 L2[WQ_PART_LIMBS + 2];
#pragma unroll
            for (int k = 0; k < WQ_PART_LIMBS; ++k) L2[k] = L[k];
            L2[WQ_PART_LIMBS] = L2[WQ_PART_LIMBS + 1] = 0ull;
            float g;
            u32 t;
            wq_gamma_threshold_of(limbs_to_double_rn(L2, -149), jb.n, &g, &t);
            s_g = g;
            s_t = t;
        }
    }
    if (tid == 0) {
        jb.gamma[0] = s_g;
        P.thresh[blockIdx.x] = s_t;
    }
}

// A CTA packs words of one matrix (grid-stride over its block range); each
// thread packs 16 consecutive weights into one 32-bit word per step, the
// next word's vectors in flight while it packs the current one.  T is read
// after the final grid has completed (griddepcontrol.wait).
template <bool BF16>
__global__ void __launch_bounds__(WQ_PACK_THREADS) k_ternary_pack(const __grid_constant__ WqParams P) {
    constexpr int VPW = BF16 ? 2 : 4;  // 16-byte vectors per 16 weights
    constexpr int EPV = BF16 ? 8 : 4;
    // a programmatically dependent launch after this one (bl_linear's act
    // quant, which does not read the packed weights) may start now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    int ji = 0;
    while (ji + 1 < P.count && (int)blockIdx.x >= P.j[ji + 1].pblk0) ++ji;
    const WqJob &jb = P.j[ji];
    const long long stride = (long long)jb.pnblk * WQ_PACK_THREADS;
    long long wl = (long long)((int)blockIdx.x - jb.pblk0) * WQ_PACK_THREADS + threadIdx.x;
    const long long nwords = jb.nwords;
    // the first words of W are requested before waiting for the reduction grid
    uint4 v[VPW];
#pragma unroll
    for (int q = 0; q < VPW; ++q) v[q] = wl < nwords ? ldg_stream_v4(jb.W + wl * VPW + q) : make_uint4(0, 0, 0, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const u32 T = __ldcg(P.thresh + ji);  // written by the final grid
    // bf16: |w| >= T <=> the magnitude's 15 bits >= T16 = ceil(T / 2^16),
    // tested on both halves of a word at once: (w & 0x7fff7fff) + C with
    // C = (0x8000 - T16) per half has bit 15 (31) set exactly when the low
    // (high) half is >= T16, and no carry crosses the halves (T16 >= 1, as
    // gamma >= 1e-5)
    const u32 T16 = (T + 0xffffu) >> 16;
    const u32 C = (0x8000u - T16) * 0x00010001u;
    for (; wl < nwords; wl += stride) {
        const long long wn = wl + stride;
        uint4 nx[VPW];
#pragma unroll
        for (int q = 0; q < VPW; ++q) nx[q] = wn < nwords ? ldg_stream_v4(jb.W + wn * VPW + q) : make_uint4(0, 0, 0, 0);
        u32 word = 0;
        if (BF16) {
            // pair p = weights 2p (low half) and 2p + 1: j = p / 2, i = 2 (p & 1) + half
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
                u32 t[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int p = 2 * jp + h;
                    const u32 w = (&v[p >> 2].x)[p & 3];
                    const u32 nz = ((w & 0x7fff7fffu) + C) & 0x80008000u;
                    // code 1 - W_q at bits 14-15 (low weight) and 30-31: bit 0 = zero, bit 1 = negative
                    t[h] = ((nz ^ 0x80008000u) >> 1) | (nz & w);
                }
                // bytes 1 and 3 of t[0] (i = 0, 1) and of t[1] (i = 2, 3) hold the codes in
                // their top two bits; word byte i takes code (4 jp + i) at bits 2 jp
                const u32 b = __byte_perm(t[0], t[1], 0x7531u);
                word |= (b >> (6 - 2 * jp)) & (0x03030303u << (2 * jp));
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                u32 bits = vec_elem_bits<BF16>(v[k / EPV], k % EPV);
                u32 nz = (bits & 0x7fffffffu) >= T ? 1u : 0u;
                u32 code = (nz ^ 1u) | ((bits >> 30) & 2u & (nz << 1));  // 1 - W_q: 00 = +1, 01 = 0, 10 = -1
                int i = k & 3, j = k >> 2;
                word |= code << (8 * i + 2 * j);
            }
        }
        jb.packed[wl] = word;
#pragma unroll
        for (int q = 0; q < VPW; ++q) v[q] = nx[q];
    }
}

}  // namespace bl
