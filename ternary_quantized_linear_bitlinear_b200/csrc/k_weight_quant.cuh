// Step 1 of the BitLinear forward: absmean ternary weight quantization and
// 2-bit packing ("Distillix" README, 1. BitNet b1.58 Core; "bitone" README,
// Forward pass; "SLM750-Edge" section 3.1).
//
// Three launches on the caller's stream, each over one or several weight
// matrices (up to WQ_MAX_JOBS: e.g. the projections of a layer, so their
// reduction latency chains overlap), chained as programmatic dependents:
//   k_absmean_partial  one pass over W: exact per-block sum of |w| as a
//                      384-bit fixed-point integer in units of 2^-149,
//                      written to the workspace
//   k_absmean_final    one CTA per matrix: sums its block partials, rounds
//                      once to double, gamma = float(S / n) + 1e-5f, and the
//                      float threshold T with
//                        |w| >= T  <=>  float(|w|/gamma) > 0.5
//   k_ternary_pack     second pass over W (its first words requested before
//                      the wait for T): W_q = sign(w) * (|w| >= T), stored
//                      as the code 1 - W_q, four codes per byte in the
//                      packed word layout
// No CTA waits on another CTA of its own launch, and nothing in the
// workspace needs clearing: every word a launch reads there was written by
// the launch before it.
//
// Exactness: every finite float is an integer multiple of 2^-149, so sum|w|
// is an integer in those units.  Each thread accumulates m << (e - base) in a
// 64-bit register for exponents inside a 26-binade window chosen per block
// from a sample of its data (term < 2^49, at most 2^14 terms per thread).
// Anything outside the window (tiny, huge or subnormal values) is added
// exactly into per-block shared-memory bins indexed by exponent.  The result
// does not depend on the window, the grid or the order of the additions.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int WQ_THREADS = 512;
constexpr int WQ_PACK_THREADS = 256;
constexpr int WQ_WINDOW = 25;       // fast path: base <= e <= base + 25
constexpr int WQ_PART_LIMBS = 6;    // per-block partial, 384 bits
constexpr int WQ_MAX_BLOCKS = 1024; // over all matrices of a launch
constexpr int WQ_MAX_JOBS = 8;      // weight matrices per launch
constexpr size_t WQ_WS_PARTIALS = (size_t)WQ_MAX_BLOCKS * WQ_PART_LIMBS * 8;
constexpr size_t WQ_WS_BYTES = WQ_WS_PARTIALS + 256;  // + threshold words

// One weight matrix of a (grouped) quantization launch: blocks
// [blk0, blk0 + nblk) of the reduction grid sum it, block j of the final
// grid derives its gamma and T, blocks [pblk0, pblk0 + pnblk) of the pack
// grid pack it.
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
};

struct WqParams {
    WqJob j[WQ_MAX_JOBS];
    int count;
    u64 *partials;    // [WQ_MAX_BLOCKS][WQ_PART_LIMBS]
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

// Sums a matrix's block partials (one limb position per pass, 128 bits per
// limb across the block), rounds the total to double and derives gamma and
// T.  Whole block of NT threads; every thread returns with s_out[0] = gamma
// bits and s_out[1] = T bits.
template <int NT>
__device__ void wq_gamma_threshold(const u64 *partials, int nblocks, long long n, u32 *s_out) {
    constexpr int NL = WQ_PART_LIMBS;
    constexpr int NW = NT / 32;
    __shared__ u64 f_lo[NL][NW], f_hi[NL][NW];
    __shared__ u64 f_sum[NL][2];
    const int tid = threadIdx.x;
    u64 slo[NL], shi[NL];
#pragma unroll
    for (int k = 0; k < NL; ++k) slo[k] = shi[k] = 0ull;
    for (int b = tid; b < nblocks; b += NT) {
#pragma unroll
        for (int k = 0; k < NL; ++k) {
            // written by the reduction grid: bypass L1
            const u64 v = __ldcg(partials + (size_t)b * NL + k);
            const u64 t = slo[k] + v;
            shi[k] += t < v ? 1ull : 0ull;
            slo[k] = t;
        }
    }
#pragma unroll
    for (int k = 0; k < NL; ++k) {
        warp_sum_u128(slo[k], shi[k]);
        if ((tid & 31) == 0) {
            f_lo[k][tid >> 5] = slo[k];
            f_hi[k][tid >> 5] = shi[k];
        }
    }
    __syncthreads();
    // limb position k summed over the warps by lane k of warp 0 (128 bits:
    // a thread adds at most four 64-bit limbs, the block's sum is below 2^74)
    if (tid < NL) {
        u64 lo = 0ull, hi = 0ull;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const u64 t = lo + f_lo[tid][w];
            hi += f_hi[tid][w] + (t < lo ? 1ull : 0ull);
            lo = t;
        }
        f_sum[tid][0] = lo;
        f_sum[tid][1] = hi;
    }
    __syncwarp();
    if (tid == 0) {
        // S = sum_k (hi:lo)_k << 64k, folded into NL + 2 limbs
        u64 L[NL + 2];
#pragma unroll
        for (int k = 0; k < NL + 2; ++k) L[k] = 0ull;
#pragma unroll
        for (int k = 0; k < NL; ++k) limbs_add_u128_shl(L, f_sum[k][0], f_sum[k][1], 64 * k);
        double S = limbs_to_double_rn(L, -149);
        float mean = __double2float_rn(__ddiv_rn(S, (double)n));
        float g = __fadd_rn(mean, 1e-5f);
        // smallest t with float(t / g) > 0.5: start at g/2 (exact, quotient 0.5)
        float t = __fmul_rn(0.5f, g);
        for (int it = 0; it < 64 && !(__fdiv_rn(t, g) > 0.5f); ++it)
            t = __uint_as_float(__float_as_uint(t) + 1u);
        s_out[0] = __float_as_uint(g);
        s_out[1] = __float_as_uint(t);
    }
    __syncthreads();
}

template <bool BF16>
__global__ void __launch_bounds__(WQ_THREADS, 2) k_absmean_partial(const __grid_constant__ WqParams P) {
    // the pack kernel may start loading W while this grid runs
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int EPV = BF16 ? 8 : 4;  // elements per 16-byte vector
    __shared__ u64 s_bins[256];
    __shared__ u32 s_emax;
    __shared__ u64 s_wlo[WQ_THREADS / 32], s_whi[WQ_THREADS / 32];

    // the matrix this block sums
    int ji = 0;
    while (ji + 1 < P.count && (int)blockIdx.x >= P.j[ji + 1].blk0) ++ji;
    const WqJob &job = P.j[ji];
    const uint4 *__restrict__ W = job.W;
    const long long nvec = job.nvec;

    const int tid = threadIdx.x;
    for (int i = tid; i < 256; i += WQ_THREADS) s_bins[i] = 0ull;
    if (tid == 0) s_emax = 0;

    const long long stride = (long long)job.nblk * WQ_THREADS;
    const long long first = (long long)((int)blockIdx.x - job.blk0) * WQ_THREADS + tid;

    // Window from a sample: the block's first vector per thread.  The next
    // four vectors are requested before the block reduction, so their
    // latency overlaps it.
    u32 emax = 0;
    uint4 v0 = make_uint4(0, 0, 0, 0);
    if (first < nvec) {
        v0 = ldg_stream_v4(W + first);
    }
    uint4 a[4];
    long long i = first + stride;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        a[q] = i + q * stride < nvec ? ldg_stream_v4(W + i + q * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < EPV; ++j) {
        u32 e = (vec_elem_bits<BF16>(v0, j) & 0x7fffffffu) >> 23;
        emax = e > emax ? e : emax;
    }
    emax = warp_max_u32(emax);
    __syncthreads();
    if ((tid & 31) == 0) atomicMax(&s_emax, emax);
    __syncthreads();
    int top = (int)s_emax + 2;
    if (top > 254) top = 254;
    int base = top - WQ_WINDOW;
    if (base < 1) base = 1;

    u64 acc = 0ull;
    auto add_vec = [&](const uint4 &v) {
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
            u32 u = vec_elem_bits<BF16>(v, j) & 0x7fffffffu;
            u32 e = u >> 23;
            u32 m = (u & 0x7fffffu) | 0x800000u;
            u32 d = e - (u32)base;
            if (d <= (u32)WQ_WINDOW) {
                acc = mad_wide_u32(m, 1u << d, acc);
            } else if (u != 0u) {
                atomicAdd(&s_bins[e], (u64)(e ? m : (u & 0x7fffffu)));
            }
        }
    };
    add_vec(v0);  // zero when first >= nvec
    // Two stages of four vectors: the next four are in flight while the
    // current four are summed.  a[] holds vectors i + q * stride (zero where
    // past the end; zeros add nothing).
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
#pragma unroll
    for (int q = 0; q < 4; ++q) add_vec(a[q]);

    // Block sum of the 64-bit window accumulators as 128 bits.
    u64 lo = acc, hi = 0ull;
    warp_sum_u128(lo, hi);
    if ((tid & 31) == 0) {
        s_wlo[tid >> 5] = lo;
        s_whi[tid >> 5] = hi;
    }
    __syncthreads();
    if (tid < 32) {
        // warp 0: which exponent bins are non-empty (usually none)
        u32 nz[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) nz[q] = __ballot_sync(0xffffffffu, s_bins[q * 32 + tid] != 0ull);
        if (tid == 0) {
            u64 L[WQ_PART_LIMBS] = {0, 0, 0, 0, 0, 0};
            u64 blo = 0, bhi = 0;
            for (int w = 0; w < WQ_THREADS / 32; ++w) {
                u64 sl = blo + s_wlo[w];
                bhi += s_whi[w] + (sl < blo ? 1ull : 0ull);
                blo = sl;
            }
            // term m << (e - base) stands for m * 2^(e - 150) = term * 2^(base - 1) units
            limbs_add_u128_shl(L, blo, bhi, base - 1);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                u32 bits = nz[q];
                while (bits) {
                    const int e = q * 32 + __ffs(bits) - 1;
                    bits &= bits - 1;
                    limbs_add_u128_shl(L, s_bins[e], 0ull, e > 0 ? e - 1 : 0);
                }
            }
            // read by the pack grid after its griddepcontrol.wait (which
            // returns once this grid has completed and its writes are visible)
#pragma unroll
            for (int k = 0; k < WQ_PART_LIMBS; ++k) P.partials[(size_t)blockIdx.x * WQ_PART_LIMBS + k] = L[k];
        }
    }
}

// Block j derives gamma and T of matrix j from its reduction blocks'
// partials (read after the reduction grid has completed).
__global__ void __launch_bounds__(WQ_PACK_THREADS) k_absmean_final(const __grid_constant__ WqParams P) {
    // the pack grid may start loading W now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ u32 s_gt[2];
    const WqJob &jb = P.j[blockIdx.x];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    wq_gamma_threshold<WQ_PACK_THREADS>(P.partials + (size_t)jb.blk0 * WQ_PART_LIMBS, jb.nblk, jb.n, s_gt);
    if (threadIdx.x == 0) {
        jb.gamma[0] = __uint_as_float(s_gt[0]);
        P.thresh[blockIdx.x] = s_gt[1];
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
