// Step 2 of the BitLinear forward: per-token absmax INT8 activation
// quantization ("BitDistill" article, Evaluation and results), optionally
// fused with the SubLN RMSNorm that precedes the o_proj / down_proj inputs
// ("BitDistill", Stage 1; "SLM750-Edge" section 2.1, eps 1e-6 from its Key
// Architectural Features).
//
//   s   = float(127 / max(max|y|, 1e-5f))
//   x_q = clamp(round_half_even(float(y * s)), -128, 127)
// with y = x, or y = float(float(x / r) * g) and
//   r = sqrtf(float(double(sum x^2) / K) + eps),
// the sum of squares exact (see k_act_quant_subln).
//
// Kernels (all read X once from HBM and write x_q once):
//   k_act_quant_warp   one warp per row, row in registers (up to 1024
//                      16-byte vectors), no SubLN
//   k_act_quant        one CTA per row, longer rows, no SubLN
//   k_act_quant_subln  one warp per row, chunked, any length, SubLN
//   k_act_quant_subln_row   one CTA per row cached in shared memory,
//                      SubLN, rows longer than 256 vectors and the gated
//                      FFN input (bl_ffn_act_quant)
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

// One CTA per row (rows longer than a warp holds), no SubLN.  VEC: 16-byte
// vectors per thread; EPV elements per vector.
template <bool BF16, int VEC, bool GLU = false>
__global__ void __launch_bounds__(1024, 1) k_act_quant(const __grid_constant__ ActParams P) {
    static_assert(!(GLU && BF16), "GLU inputs are float32 projection outputs");
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int VPT = VEC * EPV;
    __shared__ float s_red[32];

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
    // as a programmatic dependent launch this grid completes only after the
    // grid before it (no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// One warp per row: VPL 16-byte vectors per lane, the row in registers,
// reductions by warp shuffles -- no block barrier at all.
constexpr int AQW_WARPS = 4;

// Per-half unsigned max of two 16-bit lanes.
__device__ __forceinline__ u32 vmax_u16x2(u32 a, u32 b) {
    u32 r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Per-half unsigned min of two 16-bit lanes.
__device__ __forceinline__ u32 vmin_u16x2(u32 a, u32 b) {
    u32 r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

template <bool BF16>
__device__ __forceinline__ u32 aq_bits(const uint4 &v, int j) {
    const u32 w = j < (BF16 ? 2 : 1) ? v.x : j < (BF16 ? 4 : 2) ? v.y : j < (BF16 ? 6 : 3) ? v.z : v.w;
    return BF16 ? ((j & 1) ? (w & 0xffff0000u) : (w << 16)) : w;
}

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
    }
    if (GLU) {
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const int vi = lane + v * 32;
            if (vi < nvec)
                raw[v] = glu_relu2_v4(raw[v], ldg_stream_v4(reinterpret_cast<const uint4 *>(pr.X2) + (size_t)m * nvec + vi));
        }
    }
    if (BF16) {
        // both halves of a word at once: max of the 15-bit magnitudes
        u32 m2 = 0;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            m2 = vmax_u16x2(m2, raw[v].x & 0x7fff7fffu);
            m2 = vmax_u16x2(m2, raw[v].y & 0x7fff7fffu);
            m2 = vmax_u16x2(m2, raw[v].z & 0x7fff7fffu);
            m2 = vmax_u16x2(m2, raw[v].w & 0x7fff7fffu);
        }
        amax = max(m2 << 16, m2 & 0xffff0000u);
    } else {
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int j = 0; j < EPV; ++j) amax = max(amax, aq_bits<BF16>(raw[v], j) & 0x7fffffffu);
    }
    amax = warp_max_u32(amax);
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(amax), 1e-5f));
    if (lane == 0) pr.s[m] = s;
    int8_t *qr = pr.xq + (size_t)m * K;
    // finite rows: |x * s| <= 127, so rne and the int8 byte come from one
    // addend (aq_pack4) and no clamp applies; a row with inf / NaN takes the
    // converting path
    const bool finite = amax < 0x7f800000u;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const int vi = lane + v * 32;
        if (vi >= nvec) continue;
        u32 out[EPV / 4];
        if (finite) {
#pragma unroll
            for (int q = 0; q < EPV / 4; ++q) {
                const float a = __uint_as_float(aq_bits<BF16>(raw[v], 4 * q + 0));
                const float b = __uint_as_float(aq_bits<BF16>(raw[v], 4 * q + 1));
                const float c = __uint_as_float(aq_bits<BF16>(raw[v], 4 * q + 2));
                const float d = __uint_as_float(aq_bits<BF16>(raw[v], 4 * q + 3));
                out[q] = pack4_s8_rne(a, b, c, d, s);
            }
        } else {
#pragma unroll
            for (int q = 0; q < EPV / 4; ++q) {
                u32 word = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int qi = __float2int_rn(__fmul_rn(__uint_as_float(aq_bits<BF16>(raw[v], 4 * q + j)), s));
                    qi = max(-128, min(127, qi));
                    word |= ((u32)qi & 0xffu) << (8 * j);
                }
                out[q] = word;
            }
        }
        if (BF16) {
            *reinterpret_cast<uint2 *>(qr + (size_t)vi * 8) = make_uint2(out[0], out[EPV / 4 - 1]);
        } else {
            *reinterpret_cast<u32 *>(qr + (size_t)vi * 4) = out[0];
        }
    }
    // as a programmatic dependent launch this grid completes only after the
    // grid before it (no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// One warp per row with SubLN (rows without a gain are quantized plainly):
// the row is processed in chunks of 128 16-byte vectors (AQS_V per lane),
// re-read from L1/L2 for each pass unless it fits one chunk.  Few registers,
// so many warps per SM hide the latency of the per-element divisions.
//   pass 1  max|x| (the window of the exact sum)
//   pass 2  exact sum x^2: each window adds the values with exponent e in
//           [elo, ehi] (31 binades; subnormals count as e = 1 without the
//           hidden bit) as mant^2 << 2(e - elo) into a 128-bit lane
//           accumulator (< 2^108 per term, <= 2^12 terms per lane, warp sum
//           < 2^125); lane 0 adds it into 576-bit limbs in units of 2^-298;
//           the next window, 31 binades lower, runs only while some lane
//           still holds a smaller nonzero value (normally never)
//   pass 3  r = sqrtf(float(double(S) / K) + eps); max|y|, y = float(float(x / r) * g)
//   pass 4  x_q = clamp(rne(float(y * s)), -128, 127), s = float(127 / max(max|y|, 1e-5f))
constexpr int AQS_V = 4;

template <bool BF16, bool GLU>
__global__ void __launch_bounds__(AQW_WARPS * 32) k_act_quant_subln(const __grid_constant__ ActParams P) {
    static_assert(!(GLU && BF16), "GLU inputs are float32 projection outputs");
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int CH = 32 * AQS_V;  // vectors per chunk
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int gw = blockIdx.x * AQW_WARPS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (gw >= P.count * P.M) return;
    const int pi = gw / P.M, m = gw - pi * P.M;
    const ActProblem &pr = P.p[pi];
    const int K = pr.K, nvec = K / EPV;
    const int nch = (nvec + CH - 1) / CH;
    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.X) + (size_t)m * nvec;
    const uint4 *ur = GLU ? reinterpret_cast<const uint4 *>(pr.X2) + (size_t)m * nvec : nullptr;
    const float4 *g4 = reinterpret_cast<const float4 *>(pr.gain);
    uint4 c[AQS_V];
    auto load = [&](int ch) {
#pragma unroll
        for (int i = 0; i < AQS_V; ++i) {
            const int vi = ch * CH + 32 * i + lane;
            c[i] = make_uint4(0, 0, 0, 0);
            if (vi < nvec) {
                c[i] = ldg_nc_v4(xr + vi);
                if (GLU) c[i] = glu_relu2_v4(c[i], ldg_nc_v4(ur + vi));
            }
        }
    };
    // pass 1 (SubLN rows: also the double estimate of sum x^2)
    u32 amax = 0;
    double dsq = 0.0;
    for (int ch = 0; ch < nch; ++ch) {
        load(ch);
#pragma unroll
        for (int i = 0; i < AQS_V; ++i)
#pragma unroll
            for (int j = 0; j < EPV; ++j) {
                const u32 b = aq_bits<BF16>(c[i], j);
                amax = max(amax, b & 0x7fffffffu);
                if (g4 != nullptr) {
                    const double xd = abs_as_double(b);
                    dsq = __fma_rn(xd, xd, dsq);
                }
            }
    }
    amax = warp_max_u32(amax);
    float r = 1.f;
    float fest = 0.f;
    bool decided = false;
    if (g4 != nullptr) {
        dsq = warp_sum_f64(dsq);
        decided = subln_mean_sq_from_estimate(dsq, K, amax, &fest);
        decided = __shfl_sync(0xffffffffu, decided, 0);  // lane 0's sum decides (lanes may round differently)
        fest = __shfl_sync(0xffffffffu, fest, 0);
    }
    if (g4 != nullptr && decided) r = __fsqrt_rn(__fadd_rn(fest, P.eps));
    if (g4 != nullptr && !decided) {
        // pass 2: exact, by windows
        u64 L[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
        int ehi = (int)(amax >> 23);
        if (ehi < 1) ehi = 1;
        for (int pass = 0; pass < 10; ++pass) {
            const int elo = ehi - 30 < 1 ? 1 : ehi - 30;
            u64 lo = 0ull, hi = 0ull;
            bool below = false;
            for (int ch = 0; ch < nch; ++ch) {
                if (nch > 1 || pass > 0) load(ch);
#pragma unroll
                for (int i = 0; i < AQS_V; ++i) {
#pragma unroll
                    for (int j = 0; j < EPV; ++j) {
                        const u32 u = aq_bits<BF16>(c[i], j) & 0x7fffffffu;
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
        if (lane == 0)
            r = __fsqrt_rn(__fadd_rn(__double2float_rn(__ddiv_rn(limbs_to_double_rn(L, -298), (double)K)), P.eps));
        r = __shfl_sync(0xffffffffu, r, 0);
    }
    if (g4 != nullptr) {
        // pass 3
        amax = 0;
        for (int ch = 0; ch < nch; ++ch) {
            if (nch > 1) load(ch);
#pragma unroll
            for (int i = 0; i < AQS_V; ++i) {
                const int vi = ch * CH + 32 * i + lane;
                if (vi >= nvec) continue;
#pragma unroll
                for (int q = 0; q < EPV / 4; ++q) {
                    const float4 g = __ldg(g4 + vi * (EPV / 4) + q);
                    const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float y = __fmul_rn(__fdiv_rn(__uint_as_float(aq_bits<BF16>(c[i], 4 * q + j)), r), gg[j]);
                        amax = max(amax, __float_as_uint(y) & 0x7fffffffu);
                    }
                }
            }
        }
        amax = warp_max_u32(amax);
    }
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(amax), 1e-5f));
    if (lane == 0) pr.s[m] = s;
    // pass 4
    int8_t *qr = pr.xq + (size_t)m * K;
    for (int ch = 0; ch < nch; ++ch) {
        if (nch > 1) load(ch);
#pragma unroll
        for (int i = 0; i < AQS_V; ++i) {
            const int vi = ch * CH + 32 * i + lane;
            if (vi >= nvec) continue;
            u32 out[EPV / 4];
#pragma unroll
            for (int q = 0; q < EPV / 4; ++q) {
                float gg[4] = {1.f, 1.f, 1.f, 1.f};
                if (g4 != nullptr) {
                    const float4 g = __ldg(g4 + vi * (EPV / 4) + q);
                    gg[0] = g.x;
                    gg[1] = g.y;
                    gg[2] = g.z;
                    gg[3] = g.w;
                }
                u32 word = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float y = __uint_as_float(aq_bits<BF16>(c[i], 4 * q + j));
                    if (g4 != nullptr) y = __fmul_rn(__fdiv_rn(y, r), gg[j]);
                    int qi = __float2int_rn(__fmul_rn(y, s));
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
    // as a programmatic dependent launch this grid completes only after the
    // grid before it (no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// One CTA (AQR_THREADS threads) per row with SubLN, the row cached in shared
// memory as float32: the same result as k_act_quant_subln, with the row's
// elements spread over four warps and the reductions combined through
// shared memory.  A warp per row left too few independent chains per SM to
// hide the latency of the arithmetic.
//
// r needs f = float(double(S) / K) for the exact S = sum x^2: pass 1 also
// sums the squares in double as it loads the row (abs_as_double), and
// subln_mean_sq_from_estimate decides f from that estimate for all but rows
// within about 10^-12 of a float rounding boundary or with inf / NaN, which
// sum the squares exactly by windows over the cached row, as
// k_act_quant_subln does.
constexpr int AQR_THREADS = 128;
constexpr int AQR_WARPS = AQR_THREADS / 32;
constexpr int AQR_MAX_K = 24 * 1024;  // rows cached per CTA: K * 4 bytes of dynamic shared memory

__device__ __forceinline__ u32 aqr_block_max(u32 v, u32 *s_u) {
    v = warp_max_u32(v);
    __syncthreads();  // s_u free (a previous reduction has been read)
    if ((threadIdx.x & 31) == 0) s_u[threadIdx.x >> 5] = v;
    __syncthreads();
    u32 r = s_u[0];
#pragma unroll
    for (int w = 1; w < AQR_WARPS; ++w) r = max(r, s_u[w]);
    return r;
}

template <bool BF16, bool GLU>
__global__ void __launch_bounds__(AQR_THREADS, 8) k_act_quant_subln_row(const __grid_constant__ ActParams P) {
    static_assert(!(GLU && BF16), "GLU inputs are float32 projection outputs");
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int U = 4;  // 16-byte vectors in flight per thread in pass 1
    extern __shared__ __align__(16) float s_row[];
    __shared__ u32 s_u[AQR_WARPS];
    __shared__ u64 s_lo[AQR_WARPS], s_hi[AQR_WARPS];
    __shared__ float s_r;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pi = blockIdx.x / P.M, m = blockIdx.x - pi * P.M;
    const ActProblem &pr = P.p[pi];
    const int K = pr.K, nvec = K / EPV;
    const uint4 *xr = reinterpret_cast<const uint4 *>(pr.X) + (size_t)m * nvec;
    const uint4 *ur = GLU ? reinterpret_cast<const uint4 *>(pr.X2) + (size_t)m * nvec : nullptr;
    const float4 *g4 = reinterpret_cast<const float4 *>(pr.gain);
    // pass 1: load (once), cache as float, max|x|, and (SubLN rows) the
    // double sum of squares S_hat
    // (bf16: also the smallest exponent field, two halves at a time; 0 means
    // the row holds a zero or a subnormal value)
    const bool sub = g4 != nullptr;
    u32 amax = 0, emin2 = 0xffffffffu;
    double dsq = 0.0;
    for (int v0 = 0; v0 < nvec; v0 += AQR_THREADS * U) {
        uint4 c[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int vi = v0 + AQR_THREADS * i + tid;
            c[i] = vi < nvec ? ldg_stream_v4(xr + vi) : make_uint4(0, 0, 0, 0);
        }
        if (GLU) {
#pragma unroll
            for (int i = 0; i < U; ++i) {
                const int vi = v0 + AQR_THREADS * i + tid;
                if (vi < nvec) c[i] = glu_relu2_v4(c[i], ldg_stream_v4(ur + vi));
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int vi = v0 + AQR_THREADS * i + tid;
            if (vi >= nvec) continue;
            if (BF16) {
                emin2 = vmin_u16x2(emin2, c[i].x & 0x7f807f80u);
                emin2 = vmin_u16x2(emin2, c[i].y & 0x7f807f80u);
                emin2 = vmin_u16x2(emin2, c[i].z & 0x7f807f80u);
                emin2 = vmin_u16x2(emin2, c[i].w & 0x7f807f80u);
            }
            float f[EPV];
#pragma unroll
            for (int j = 0; j < EPV; ++j) {
                const u32 b = aq_bits<BF16>(c[i], j);
                amax = max(amax, b & 0x7fffffffu);
                if (sub) {
                    const double xd = abs_as_double(b);
                    dsq = __fma_rn(xd, xd, dsq);
                }
                f[j] = __uint_as_float(b);
            }
#pragma unroll
            for (int j = 0; j < EPV; j += 4)
                reinterpret_cast<float4 *>(s_row)[(vi * EPV + j) >> 2] = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
        }
    }
    amax = aqr_block_max(amax, s_u);  // also orders the row cache writes before the reads below
    // bf16 rows without zero or subnormal values take Markstein's division
    // in pass 3 without a per-element test
    const bool bf16_normal = BF16 && sub && !__syncthreads_or((emin2 & 0xffffu) == 0u || (emin2 >> 16) == 0u);
    if (sub) {
        // f = float(double(S) / K) from S_hat when its bounds agree
        __shared__ double s_d[AQR_WARPS];
        __shared__ float s_f;
        __shared__ int s_exact;
        dsq = warp_sum_f64(dsq);
        if (lane == 0) s_d[warp] = dsq;
        __syncthreads();
        if (tid == 0) {
            double sh = s_d[0];
            for (int w = 1; w < AQR_WARPS; ++w) sh = __dadd_rn(sh, s_d[w]);
            float f;
            const bool ok = subln_mean_sq_from_estimate(sh, K, amax, &f);
            s_f = f;
            s_exact = ok ? 0 : 1;
        }
        __syncthreads();
        if (!s_exact) {
            if (tid == 0) s_r = __fsqrt_rn(__fadd_rn(s_f, P.eps));
        } else {
        // exact sum of squares by windows over the cached row
        u64 L[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
        int ehi = (int)(amax >> 23);
        if (ehi < 1) ehi = 1;
        for (int pass = 0; pass < 10; ++pass) {
            const int elo = ehi - 30 < 1 ? 1 : ehi - 30;
            u64 lo = 0ull, hi = 0ull;
            int below = 0;
            for (int k = tid; k < K; k += AQR_THREADS) {
                const u32 u = __float_as_uint(s_row[k]) & 0x7fffffffu;
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
                    below = 1;
                }
            }
            warp_sum_u128(lo, hi);  // < 2^108 per term, < 2^116 per thread, < 2^123 per CTA
            if (lane == 0) {
                s_lo[warp] = lo;
                s_hi[warp] = hi;
            }
            const int any_below = __syncthreads_or(below);
            if (tid == 0)
                for (int w = 0; w < AQR_WARPS; ++w) limbs_add_u128_shl(L, s_lo[w], s_hi[w], 2 * (elo - 1));
            if (!any_below || elo == 1) break;
            ehi = elo - 1;
            __syncthreads();  // s_lo / s_hi read before the next window writes them
        }
        if (tid == 0)
            s_r = __fsqrt_rn(__fadd_rn(__double2float_rn(__ddiv_rn(limbs_to_double_rn(L, -298), (double)K)), P.eps));
        }
        __syncthreads();
        const float r = s_r;
        // pass 3: y = float(float(x / r) * g) in place, max|y|.  For float32
        // rows (the gated FFN input and h from the gated GEMM), x / r is
        // correctly rounded by Markstein's method from the
        // correctly rounded reciprocal of the row constant r (q0 = x * (1/r),
        // remainder x - r * q0 by FMA, one correction FMA).  The method is
        // exact whenever that remainder is representable, which holds for
        // quotients well above 2^-126 * 2^24 (checked against IEEE division
        // for every dividend mantissa and 2016 divisors); nearer underflow
        // the remainder can need bits below 2^-149 and q1 may be one ulp off.
        // A nonzero subnormal dividend or an r that is not a finite normal
        // number takes the IEEE division.  The underflow band cannot change
        // x_q or s: there |y| < 2^-100, so y * s (s <= 127 / 1e-5 < 2^24)
        // rounds to 0 either way, and such a y is the row maximum only when
        // every |y| of the row is below 1e-5, where s is floored at
        // 127 / 1e-5 whatever the maximum is.
        // Measured 172 -> 136 us for [8192, 4096].  A bf16 row without zero or
        // subnormal values (known from pass 1) takes Markstein for every
        // element without the per-element test (717 -> 638 us for [32768,
        // 9728]); other bf16 rows keep the IEEE division, which with the
        // per-element test was as fast.
        const float ry = __frcp_rn(r);
        const bool mk = (GLU || !BF16) && __float_as_uint(r) >= 0x00800000u && __float_as_uint(r) < 0x7f800000u;
        auto div_r = [&](float x) {
            const u32 ax = __float_as_uint(x) & 0x7fffffffu;
            if (!mk || (ax != 0u && ax < 0x00800000u)) return __fdiv_rn(x, r);
            const float q0 = __fmul_rn(x, ry);
            return __fmaf_rn(__fmaf_rn(-q0, r, x), ry, q0);
        };
        amax = 0;
        if (bf16_normal && __float_as_uint(r) >= 0x00800000u && __float_as_uint(r) < 0x7f800000u) {
            // a bf16 row without zero or subnormal values: Markstein for every element, no branch
            for (int q = tid; q < K / 4; q += AQR_THREADS) {
                const float4 g = __ldg(g4 + q);
                float4 x = reinterpret_cast<float4 *>(s_row)[q];
                float q0 = __fmul_rn(x.x, ry);
                x.x = __fmul_rn(__fmaf_rn(__fmaf_rn(-q0, r, x.x), ry, q0), g.x);
                q0 = __fmul_rn(x.y, ry);
                x.y = __fmul_rn(__fmaf_rn(__fmaf_rn(-q0, r, x.y), ry, q0), g.y);
                q0 = __fmul_rn(x.z, ry);
                x.z = __fmul_rn(__fmaf_rn(__fmaf_rn(-q0, r, x.z), ry, q0), g.z);
                q0 = __fmul_rn(x.w, ry);
                x.w = __fmul_rn(__fmaf_rn(__fmaf_rn(-q0, r, x.w), ry, q0), g.w);
                reinterpret_cast<float4 *>(s_row)[q] = x;
                amax = max(amax, max(max(__float_as_uint(x.x) & 0x7fffffffu, __float_as_uint(x.y) & 0x7fffffffu),
                                     max(__float_as_uint(x.z) & 0x7fffffffu, __float_as_uint(x.w) & 0x7fffffffu)));
            }
        } else
        for (int q = tid; q < K / 4; q += AQR_THREADS) {
            const float4 g = __ldg(g4 + q);
            float4 x = reinterpret_cast<float4 *>(s_row)[q];
            x.x = __fmul_rn(div_r(x.x), g.x);
            x.y = __fmul_rn(div_r(x.y), g.y);
            x.z = __fmul_rn(div_r(x.z), g.z);
            x.w = __fmul_rn(div_r(x.w), g.w);
            reinterpret_cast<float4 *>(s_row)[q] = x;
            amax = max(amax, max(max(__float_as_uint(x.x) & 0x7fffffffu, __float_as_uint(x.y) & 0x7fffffffu),
                                 max(__float_as_uint(x.z) & 0x7fffffffu, __float_as_uint(x.w) & 0x7fffffffu)));
        }
        amax = aqr_block_max(amax, s_u);  // each thread quantizes the elements it wrote: no further barrier
    }
    const float s = __fdiv_rn(127.f, fmaxf(__uint_as_float(amax), 1e-5f));
    if (tid == 0) pr.s[m] = s;
    // pass 4: quantize, four elements -> one 32-bit word
    u32 *qr = reinterpret_cast<u32 *>(pr.xq + (size_t)m * K);
    const bool finite = amax < 0x7f800000u;  // else the converting path (inf / NaN in the row)
    for (int q = tid; q < K / 4; q += AQR_THREADS) {
        const float4 y = reinterpret_cast<const float4 *>(s_row)[q];
        if (finite) {
            qr[q] = pack4_s8_rne(y.x, y.y, y.z, y.w, s);
            continue;
        }
        const float yy[4] = {y.x, y.y, y.z, y.w};
        u32 w = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int qi = __float2int_rn(__fmul_rn(yy[j], s));
            qi = max(-128, min(127, qi));
            w |= ((u32)qi & 0xffu) << (8 * j);
        }
        qr[q] = w;
    }
    // as a programmatic dependent launch this grid completes only after the
    // grid before it (no-op otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace bl
