// Step 2 of the BitLinear forward: per-token absmax INT8 activation
// quantization ("BitDistill" article, Evaluation and results), optionally
// fused with the SubLN RMSNorm that precedes the o_proj / down_proj inputs
// ("BitDistill", Stage 1; "SLM750-Edge" section 2.1, eps 1e-6 from its Key
// Architectural Features).
//
// One CTA per token row; the row lives in registers (VPT values per thread),
// so X is read from HBM exactly once and x_q written once.
//   s   = float(127 / max(max|y|, 1e-5f))
//   x_q = clamp(round_half_even(float(y * s)), -128, 127)
// with y = x, or y = float(float(x / r) * g) and
//   r = sqrtf(float(double(sum x^2) / K) + eps),
// the sum of squares exact: x^2 = m^2 * 2^(2e - 300), accumulated as a 128-bit
// integer per thread inside a window of 30 binades below the row's largest
// exponent (m^2 < 2^48, shift <= 60, <= 32 terms per thread, so a warp sum
// stays below 2^118), everything else added exactly into shared-memory bins
// by exponent.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int AQ_MAX_GROUP = BL_MAX_GROUP;

struct ActProblem {
    const void *X;
    const float *gain;
    int8_t *xq;
    float *s;
    int K;
    int pad;
    const float *X2;  // GLU: the up projection's output (X is the gate's), f32
};

// The FFN activation between the up and down projections ("SLM750-Edge",
// Key Architectural Features: ReLU2; section 2.3: gate, up, down):
// h = float(float(r * r) * u), r = g > 0 ? g : 0.  With GLU the quantizer's
// input x is this h, computed as the row is loaded.
__device__ __forceinline__ float glu_relu2(float g, float u) {
    const float r = g > 0.f ? g : 0.f;
    return __fmul_rn(__fmul_rn(r, r), u);
}

__device__ __forceinline__ uint4 glu_relu2_v4(const uint4 &g, const uint4 &u) {
    return make_uint4(__float_as_uint(glu_relu2(__uint_as_float(g.x), __uint_as_float(u.x))),
                      __float_as_uint(glu_relu2(__uint_as_float(g.y), __uint_as_float(u.y))),
                      __float_as_uint(glu_relu2(__uint_as_float(g.z), __uint_as_float(u.z))),
                      __float_as_uint(glu_relu2(__uint_as_float(g.w), __uint_as_float(u.w))));
}

struct ActParams {
    ActProblem p[AQ_MAX_GROUP];
    int count;
    int M;
    float eps;
};

__device__ __forceinline__ float block_max_f(float v, float *s_red) {
    // values are non-negative: compare as unsigned bits
    u32 b = warp_max_u32(__float_as_uint(v));
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[w] = __uint_as_float(b);
    __syncthreads();
    u32 r = 0;
    for (int i = 0; i < nw; ++i) r = max(r, __float_as_uint(s_red[i]));
    return __uint_as_float(r);
}

// VEC: 16-byte vectors per thread; EPV elements per vector.
template <bool BF16, int VEC, bool GLU = false>
__global__ void __launch_bounds__(1024, 1) k_act_quant(const __grid_constant__ ActParams P) {
    static_assert(!(GLU && BF16), "GLU inputs are float32 projection outputs");
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int VPT = VEC * EPV;
    __shared__ float s_red[32];
    __shared__ u64 s_bins[256];
    __shared__ u64 s_lo[32], s_hi[32];
    __shared__ float s_r;

    // let a programmatically dependent launch (the GEMV) start streaming its
    // weights; it waits for this grid to finish before it reads x_q
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int pi = blockIdx.x / P.M;
    const int m = blockIdx.x - pi * P.M;
    const ActProblem &pr = P.p[pi];
    const int K = pr.K;
    const int nvec = K / EPV;
    const int tid = threadIdx.x, T = blockDim.x;

    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.X) + (size_t)m * nvec;
    float x[VPT];
    float amax = 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        int vi = tid + v * T;
        uint4 raw = vi < nvec ? ldg_stream_v4(xr + vi) : make_uint4(0, 0, 0, 0);
        if (GLU && vi < nvec)
            raw = glu_relu2_v4(raw, ldg_stream_v4(reinterpret_cast<const uint4 *>(pr.X2) + (size_t)m * nvec + vi));
        const u32 w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
            u32 bits = BF16 ? ((j & 1) ? (w4[j >> 1] & 0xffff0000u) : (w4[j >> 1] << 16)) : w4[j];
            float f = __uint_as_float(bits);
            x[v * EPV + j] = f;
            amax = fmaxf(amax, fabsf(f));
        }
    }

    if (pr.gain != nullptr) {
        // ---- exact sum of squares ------------------------------------------
        for (int i = tid; i < 256; i += T) s_bins[i] = 0ull;
        amax = block_max_f(amax, s_red);  // also orders the bin clear
        int emax = (int)(__float_as_uint(amax) >> 23);
        int elo = emax - 30;
        if (elo < 1) elo = 1;
        u64 lo = 0ull, hi = 0ull;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            u32 u = __float_as_uint(x[i]) & 0x7fffffffu;
            int e = (int)(u >> 23);
            u64 mm = (u64)((u & 0x7fffffu) | 0x800000u);
            mm *= mm;  // < 2^48
            int d = e - elo;
            if (d >= 0) {
                int sh = 2 * d;  // <= 60
                u64 plo = sh < 64 ? (mm << sh) : 0ull;
                u64 phi = sh == 0 ? 0ull : (sh < 64 ? (mm >> (64 - sh)) : (mm << (sh - 64)));
                u64 s = lo + plo;
                hi += phi + (s < lo ? 1ull : 0ull);
                lo = s;
            } else if (u != 0u) {
                u64 mr = e ? mm : (u64)(u & 0x7fffffu) * (u64)(u & 0x7fffffu);
                atomicAdd(&s_bins[e], mr);
            }
        }
        warp_sum_u128(lo, hi);
        if ((tid & 31) == 0) {
            s_lo[tid >> 5] = lo;
            s_hi[tid >> 5] = hi;
        }
        __syncthreads();
        if (tid == 0) {
            u64 L[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
            for (int w = 0; w < (T >> 5); ++w) limbs_add_u128_shl(L, s_lo[w], s_hi[w], 2 * (elo - 1));
            for (int e = 0; e < 256; ++e) {
                u64 b = s_bins[e];
                if (b) limbs_add_u128_shl(L, b, 0ull, e > 0 ? 2 * (e - 1) : 0);
            }
            double S2 = limbs_to_double_rn(L, -298);
            float ms = __double2float_rn(__ddiv_rn(S2, (double)K));
            s_r = __fsqrt_rn(__fadd_rn(ms, P.eps));
        }
        __syncthreads();
        const float r = s_r;
        const float4 *g4 = reinterpret_cast<const float4 *>(pr.gain);
        amax = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
            int vi = tid + v * T;
#pragma unroll
            for (int q = 0; q < EPV / 4; ++q) {
                float4 g = vi < nvec ? __ldg(g4 + vi * (EPV / 4) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float &xv = x[v * EPV + q * 4 + j];
                    xv = __fmul_rn(__fdiv_rn(xv, r), gg[j]);
                    amax = fmaxf(amax, fabsf(xv));
                }
            }
        }
    }

    amax = block_max_f(amax, s_red);
    const float s = __fdiv_rn(127.f, fmaxf(amax, 1e-5f));
    if (tid == 0) pr.s[m] = s;

    // x_q: EPV bytes per vector
    int8_t *qr = pr.xq + (size_t)m * K;
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
        int vi = tid + v * T;
        if (vi >= nvec) continue;
        u32 out[EPV / 4];
#pragma unroll
        for (int q = 0; q < EPV / 4; ++q) {
            u32 word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int qi = __float2int_rn(__fmul_rn(x[v * EPV + q * 4 + j], s));
                qi = max(-128, min(127, qi));
                word |= ((u32)qi & 0xffu) << (8 * j);
            }
            out[q] = word;
        }
        if (BF16) {
            *reinterpret_cast<uint2 *>(qr + (size_t)vi * 8) = make_uint2(out[0], out[EPV / 4 - 1]);
        } else {
            *reinterpret_cast<u32 *>(qr + (size_t)vi * 4) = out[0];
        }
    }
}

// One warp per row, no SubLN (short rows): VPL 16-byte vectors per lane, the
// row in registers, absmax by a warp reduction -- no block barrier at all.
constexpr int AQW_WARPS = 8;

template <bool BF16, int VPL, bool GLU = false>
__global__ void __launch_bounds__(AQW_WARPS * 32) k_act_quant_warp(const __grid_constant__ ActParams P) {
    static_assert(!(GLU && BF16), "GLU inputs are float32 projection outputs");
    constexpr int EPV = BF16 ? 8 : 4;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int gw = blockIdx.x * AQW_WARPS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (gw >= P.count * P.M) return;
    const int pi = gw / P.M, m = gw - pi * P.M;
    const ActProblem &pr = P.p[pi];
    const int K = pr.K, nvec = K / EPV;
    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.X) + (size_t)m * nvec;
    uint4 raw[VPL];
    u32 amax = 0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vi = lane + v * 32;
        raw[v] = vi < nvec ? ldg_stream_v4(xr + vi) : make_uint4(0, 0, 0, 0);
        if (GLU && vi < nvec)
            raw[v] = glu_relu2_v4(raw[v], ldg_stream_v4(reinterpret_cast<const uint4 *>(pr.X2) + (size_t)m * nvec + vi));
        const u32 w4[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
        for (int j = 0; j < EPV; ++j) {
            u32 bits = BF16 ? ((j & 1) ? (w4[j >> 1] & 0xffff0000u) : (w4[j >> 1] << 16)) : w4[j];
            amax = max(amax, bits & 0x7fffffffu);
        }
    }
    amax = warp_max_u32(amax);
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(amax), 1e-5f));
    if (lane == 0) pr.s[m] = s;
    int8_t *qr = pr.xq + (size_t)m * K;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vi = lane + v * 32;
        if (vi >= nvec) continue;
        const u32 w4[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
        u32 out[EPV / 4];
#pragma unroll
        for (int q = 0; q < EPV / 4; ++q) {
            u32 word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int e = q * 4 + j;
                u32 bits = BF16 ? ((e & 1) ? (w4[e >> 1] & 0xffff0000u) : (w4[e >> 1] << 16)) : w4[e];
                int qi = __float2int_rn(__fmul_rn(__uint_as_float(bits), s));
                qi = max(-128, min(127, qi));
                word |= ((u32)qi & 0xffu) << (8 * j);
            }
            out[q] = word;
        }
        if (BF16) {
            *reinterpret_cast<uint2 *>(qr + (size_t)vi * 8) = make_uint2(out[0], out[EPV / 4 - 1]);
        } else {
            *reinterpret_cast<u32 *>(qr + (size_t)vi * 4) = out[0];
        }
    }
}

}  // namespace bl
