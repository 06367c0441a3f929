// Shared device helpers for libbitlinear (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bitlinear.h"

namespace bl {

typedef unsigned long long u64;
typedef unsigned int u32;

// Sticky device error word: bounded waits that give up OR a code in here and
// return; the host reads it with bl_check_device_error.
enum : u32 {
    DEVERR_NONE = 0,
    DEVERR_TIMEOUT_PRODUCER = 1u << 0,
    DEVERR_TIMEOUT_MMA = 1u << 1,
    DEVERR_TIMEOUT_EXPAND = 1u << 2,
    DEVERR_TIMEOUT_EPILOGUE = 1u << 3,
    DEVERR_TMEM_ALLOC = 1u << 4,
};

__device__ u32 g_device_error;

__device__ __forceinline__ void raise_device_error(u32 code) { atomicOr(&g_device_error, code); }

// Float bits of element i of a 16-byte vector of the given dtype.
__device__ __forceinline__ u32 bf16_bits_to_f32_bits(uint16_t h) { return (u32)h << 16; }

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Streamed once: do not keep in L1.
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ u64 mad_wide_u32(u32 a, u32 b, u64 c) {
    u64 d;
    asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(d) : "r"(a), "r"(b), "l"(c));
    return d;
}

// INT8 activation codes of four finite values whose |x * s| is at most 127
// (s = 127 / max|x| of their row): p = float(x * s), then p + 1.5 * 2^23
// rounds p to the nearest integer, ties to even (the addend is even and
// its ulp is 1), and leaves that integer in two's complement in the low
// byte of the sum's bits (|p| < 2^22); the four bytes are packed first in
// the low byte.  Equal to clamp(rne(float(x * s)), -128, 127), which needs
// no clamp there.
__device__ __forceinline__ u32 pack4_s8_rne(float a, float b, float c, float d, float s) {
    constexpr float RND = 12582912.0f;  // 1.5 * 2^23
    const u32 ra = __float_as_uint(__fadd_rn(__fmul_rn(a, s), RND));
    const u32 rb = __float_as_uint(__fadd_rn(__fmul_rn(b, s), RND));
    const u32 rc = __float_as_uint(__fadd_rn(__fmul_rn(c, s), RND));
    const u32 rd = __float_as_uint(__fadd_rn(__fmul_rn(d, s), RND));
    return __byte_perm(__byte_perm(ra, rb, 0x0040u), __byte_perm(rc, rd, 0x0040u), 0x5410u);
}

// |x| of a float's bits as a double: exponent rebiased, mantissa moved;
// exact for normal x, in [2^-127, 2^-126) for zero and subnormal x (also the
// weight absmean's terms).
__device__ __forceinline__ double abs_as_double(u32 bits) {
    const u32 a = bits & 0x7fffffffu;
    return __hiloint2double((int)((a >> 3) + 0x38000000u), (int)(a << 29));
}

// SubLN's f = float(double(S) / K) for S = sum x^2 from a double estimate.
// The square of a float is exact in double and cannot over- or underflow
// there; abs_as_double gives |x| for the estimate (exact for normal x, below
// 2^-126 for zero and subnormal x, so no per-element test).  An estimate
// S_hat summed from those squares with at most K + 256 roundings of a
// non-negative sum lies within beta * S_hat of their sum, beta = 2 (K + 256)
// 2^-53, and their sum within K 2^-250 above S: S lies in
// [S_hat (1 - beta) - K 2^-250, S_hat (1 + beta)].  f is monotone in S, so
// when both ends give the same f it is f(S) bit for bit: returns true with
// *f set.  False (the caller sums exactly) when they differ -- S / K within
// about 10^-12 of a float rounding boundary -- or when amax_bits (max |x|
// of the row as float bits) says the row holds inf / NaN.
__device__ __forceinline__ bool subln_mean_sq_from_estimate(double s_hat, int K, u32 amax_bits, float *f) {
    if (amax_bits >= 0x7f800000u) return false;
    const double beta = 2.0 * (double)(K + 256) * 0x1p-53;
    const double A = (double)K * 0x1p-250;
    double lo = __dsub_rd(__dmul_rd(s_hat, 1.0 - beta), A);
    lo = lo > 0.0 ? lo : 0.0;
    const double hi = __dmul_ru(s_hat, 1.0 + beta);
    const float flo = __double2float_rn(__ddiv_rn(lo, (double)K));
    const float fhi = __double2float_rn(__ddiv_rn(hi, (double)K));
    *f = flo;
    return flo == fhi;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// ---------------------------------------------------------------------------
// Exact multi-limb fixed point (little-endian u64 limbs).

// L += (hi:lo) << sh, 0 <= sh; bits shifted past the last limb are dropped
// (callers size L so that never happens).
template <int NL>
__device__ __forceinline__ void limbs_add_u128_shl(u64 (&L)[NL], u64 lo, u64 hi, int sh) {
    int w = sh >> 6, b = sh & 63;
    u64 p0 = lo << b;
    u64 p1 = b ? ((hi << b) | (lo >> (64 - b))) : hi;
    u64 p2 = b ? (hi >> (64 - b)) : 0ull;
    u64 carry = 0;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        u64 add = (i == w) ? p0 : (i == w + 1) ? p1 : (i == w + 2) ? p2 : 0ull;
        if (i < w) continue;
        u64 s = L[i] + add;
        u64 c1 = s < add;
        u64 s2 = s + carry;
        u64 c2 = s2 < carry;
        L[i] = s2;
        carry = c1 | c2;
    }
}

template <int NL>
__device__ __forceinline__ void limbs_add(u64 (&L)[NL], const u64 (&R)[NL]) {
    u64 carry = 0;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
        u64 s = L[i] + R[i];
        u64 c1 = s < R[i];
        u64 s2 = s + carry;
        u64 c2 = s2 < carry;
        L[i] = s2;
        carry = c1 | c2;
    }
}

// 2^e as a double, -1022 <= e <= 1023.
__device__ __forceinline__ double pow2_double(int e) {
    return __longlong_as_double((long long)(e + 1023) << 52);
}

// Round the non-negative integer in L to the nearest double (ties to even)
// and scale by 2^scale_exp.
template <int NL>
__device__ double limbs_to_double_rn(const u64 (&L)[NL], int scale_exp) {
    int top = -1;
#pragma unroll
    for (int i = NL - 1; i >= 0; --i) {
        if (top < 0 && L[i] != 0ull) top = i * 64 + 63 - __clzll((long long)L[i]);
    }
    if (top < 0) return 0.0;
    int lo = top - 63;  // bit index of window bit 0
    u64 w;
    bool sticky = false;
    if (lo >= 0) {
        int wi = lo >> 6, s = lo & 63;
        u64 cur = 0, nxt = 0;
#pragma unroll
        for (int i = 0; i < NL; ++i) {
            if (i == wi) cur = L[i];
            if (i == wi + 1) nxt = L[i];
            if (i < wi && L[i] != 0ull) sticky = true;
        }
        w = s ? ((cur >> s) | (nxt << (64 - s))) : cur;
        if (s && (cur & ((1ull << s) - 1ull))) sticky = true;
    } else {
        w = L[0] << (-lo);
    }
    u64 mant = w >> 11;
    bool rb = (w >> 10) & 1ull;
    if (w & 0x3ffull) sticky = true;
    int e = lo + 11 + scale_exp;
    if (rb && (sticky || (mant & 1ull))) {
        mant += 1ull;
        if (mant == (1ull << 53)) {
            mant >>= 1;
            e += 1;
        }
    }
    return __ll2double_rn((long long)mant) * pow2_double(e);
}

// ---------------------------------------------------------------------------
// Block-wide reductions (blockDim.x multiple of 32, <= 1024).

__device__ __forceinline__ u32 warp_max_u32(u32 v) { return __reduce_max_sync(0xffffffffu, v); }

__device__ __forceinline__ void warp_sum_u128(u64 &lo, u64 &hi) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        u64 olo = __shfl_down_sync(0xffffffffu, lo, off);
        u64 ohi = __shfl_down_sync(0xffffffffu, hi, off);
        u64 s = lo + olo;
        hi += ohi + (s < lo ? 1ull : 0ull);
        lo = s;
    }
}

// ---------------------------------------------------------------------------
// mbarriers, bulk copies, bounded waits

__device__ __forceinline__ u32 smem_u32(const void *p) { return (u32)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(u32 bar, u32 count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(u32 bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(u32 bar, u32 bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// try_wait may suspend the thread up to the hint (ns) until the phase
// completes, so waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait(u32 bar, u32 parity) {
    u32 ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(200000u)
        : "memory");
    return ok != 0;
}

// Bounded wait: false when the phase did not complete within timeout_ns or
// (abort_flag != nullptr) the CTA abort flag was raised.
__device__ __forceinline__ bool mbar_wait(u32 bar, u32 parity, unsigned long long timeout_ns,
                                          const volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (int it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 7) == 0) {
            if (abort_flag != nullptr && *abort_flag) return false;
            if (globaltimer() - t0 > timeout_ns) return false;
        }
    }
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier.  dst,
// src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(u32 dst, const void *src, u32 bytes, u32 bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Same, with an L2 eviction-priority policy (from l2_policy_evict_first) for
// data that is read exactly once, so it does not displace reused lines.
__device__ __forceinline__ void bulk_g2s_hint(u32 dst, const void *src, u32 bytes, u32 bar, u64 policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ u64 l2_policy_evict_first() {
    u64 p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

}  // namespace bl
