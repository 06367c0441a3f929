/*
 * BitLinear (BitNet b1.58) forward, and its straight-through backward (at
 * the end of this file) -- plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path never
 * calls it; it shares no code, header, table or constant with the CUDA
 * library.
 *
 * Every step is written as its definition, in the order the source pages give
 * it, with no blocking or reordering:
 *
 *   weight quant   gamma = mean|W| + 1e-5, W_q = clamp(round(W / gamma), -1, 1)
 *                  -- "Distillix" README, "Key Innovations / 1. BitNet b1.58
 *                  Core" (W_q = round(clip(W / mean|W|, -1, 1))); "bitone"
 *                  README, "Forward pass" of the Triton-fused QAT BitLinear
 *                  (gamma = mean(|W|) in one reduction, W_q per tile, then
 *                  Y = X @ W_q^T * gamma); "SLM750-Edge" model card,
 *                  section 3.1 "Ternary Weight Quantization" (round_clip: 0
 *                  when |x| <= 0.5).
 *   act quant      per-token absmax INT8 -- "BitDistill" news article,
 *                  "Evaluation and results" (activations quantized to INT8);
 *                  the constants 127 / max(|x|, 1e-5) and clamp(-128, 127)
 *                  with round-half-even are the plainest reading that the
 *                  pages leave open.
 *   SubLN          RMSNorm (eps from "SLM750-Edge", "Key Architectural
 *                  Features": RMSNorm epsilon = 1e-6) applied before the
 *                  activation quantizer -- "BitDistill", "Stage 1 --
 *                  Architectural refinement with SubLN"; "SLM750-Edge",
 *                  section 2.1 (norm: SubLN = pre-RMSNorm + activation
 *                  quantization).
 *   contraction    acc = sum_k x_q * W_q, exactly (int64 here) -- "bitone"
 *                  README, "How 1.58-bit Works" (add, subtract or skip).
 *   rescale        Y = acc * gamma / s -- "bitone" README, "Forward pass"
 *                  (Y = X @ W_q^T * gamma) combined with the INT8 scale s.
 *
 * Readings where the pages are silent (precision, order, packing) are the
 * ones listed in the repository design notes:
 *   - sum|W| is the EXACT real sum (big-integer accumulation), rounded once to
 *     double; mean = float(double(S) / double(n)); gamma = mean + 1e-5f in
 *     float.  Any summation order therefore gives the same bits.
 *   - W / gamma is an IEEE float division; rounding is half-to-even (rintf).
 *   - x * s and 127 / max(|x|, 1e-5f) are IEEE float operations.
 *   - RMSNorm: S2 = exact sum x^2 rounded once to double; ms = float(S2 / K);
 *     r = sqrtf(ms + eps); y = (x / r) * g, each a float operation.
 *   - the 2-bit packing (a format of this library; the pages only say two
 *     bits or fewer per weight): row n is K/4 bytes = K/16 little-endian
 *     32-bit words; weight k = 16*w + 4*j + i has its code in word w at bits
 *     8*i + 2*j (low) and 8*i + 2*j + 1 (high); the code is 1 - W_q as a
 *     2-bit unsigned number: 00 = +1, 01 = 0, 10 = -1, 11 never written.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared
 *        -fPIC oracle.c -o liboracle.so  (see build.py beside this file).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_NONFINITE 1
#define OR_ERR_SHAPE 2
#define OR_ERR_RANGE 3

/* Threads of the OpenMP loops below (a timing knob; results do not depend
 * on it: each output is computed by one thread in a fixed order). */
void oracle_set_num_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }

/* ------------------------------------------------------------------------ */
/* Exact big-integer helpers (little-endian uint64 limbs).                   */
/* ------------------------------------------------------------------------ */

/* limbs += v << shift, with full carry propagation. */
static void big_add_shifted(uint64_t *limbs, int nlimbs, uint64_t v, int shift) {
    int idx = shift / 64;
    int bit = shift % 64;
    uint64_t lo = v << bit;
    uint64_t hi = bit ? (v >> (64 - bit)) : 0;
    uint64_t carry = 0;
    for (int i = idx; i < nlimbs; ++i) {
        uint64_t add = (i == idx) ? lo : (i == idx + 1 ? hi : 0);
        uint64_t s = limbs[i] + add;
        uint64_t c1 = s < add;
        uint64_t s2 = s + carry;
        uint64_t c2 = s2 < carry;
        limbs[i] = s2;
        carry = c1 | c2;
        if (i > idx + 1 && carry == 0) break;
    }
}

/* Round the non-negative integer held in limbs to the nearest double (ties to
 * even) and scale it by 2^scale_exp.  Returns 0.0 for zero. */
static double big_to_double(const uint64_t *limbs, int nlimbs, int scale_exp) {
    int top = -1;
    for (int i = nlimbs - 1; i >= 0; --i) {
        if (limbs[i]) {
            int b = 63;
            while (!((limbs[i] >> b) & 1u)) --b;
            top = i * 64 + b;
            break;
        }
    }
    if (top < 0) return 0.0;
    uint64_t mant = 0;
    int low = top - 52; /* bit index of the mantissa's least significant bit */
    if (low <= 0) {
        /* fits in 53 bits: the integer is the value */
        for (int b = top; b >= 0; --b)
            mant = (mant << 1) | ((limbs[b / 64] >> (b % 64)) & 1u);
        return ldexp((double)mant, scale_exp);
    }
    for (int b = top; b >= low; --b)
        mant = (mant << 1) | ((limbs[b / 64] >> (b % 64)) & 1u);
    int round_bit = (int)((limbs[(low - 1) / 64] >> ((low - 1) % 64)) & 1u);
    int sticky = 0;
    for (int b = low - 2; b >= 0 && !sticky; --b)
        if ((limbs[b / 64] >> (b % 64)) & 1u) sticky = 1;
    if (round_bit && (sticky || (mant & 1u))) {
        mant += 1;
        if (mant == ((uint64_t)1 << 53)) { mant >>= 1; low += 1; }
    }
    return ldexp((double)mant, low + scale_exp);
}

/* ------------------------------------------------------------------------ */
/* Step 1: absmean scale gamma.                                               */
/* ------------------------------------------------------------------------ */

/* Exact S = sum |w_i| as a 320-bit integer in units of 2^-149 (every finite
 * float is an integer multiple of 2^-149). */
int oracle_abs_sum_exact(const float *w, int64_t n, uint64_t limbs[5]) {
    memset(limbs, 0, 5 * sizeof(uint64_t));
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &w[i], 4);
        u &= 0x7fffffffu;
        uint32_t e = u >> 23, m = u & 0x7fffffu;
        if (e == 255) return OR_ERR_NONFINITE;
        if (e > 0) { m |= 0x800000u; }
        int shift = e > 0 ? (int)e - 1 : 0; /* value = m * 2^(shift - 149) */
        if (m) big_add_shifted(limbs, 5, m, shift);
    }
    return OR_OK;
}

double oracle_limbs_to_double(const uint64_t *limbs, int nlimbs, int scale_exp) {
    return big_to_double(limbs, nlimbs, scale_exp);
}

/* gamma = float(double(S) / double(n)) + 1e-5f. */
int oracle_absmean_gamma(const float *w, int64_t n, float *gamma) {
    if (n <= 0) return OR_ERR_SHAPE;
    uint64_t limbs[5];
    int rc = oracle_abs_sum_exact(w, n, limbs);
    if (rc) return rc;
    double S = big_to_double(limbs, 5, -149);
    double mean_d = S / (double)n;
    float mean_f = (float)mean_d;
    *gamma = mean_f + 1e-5f;
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Step 2: ternarize and pack.                                                */
/* ------------------------------------------------------------------------ */

/* W_q = clamp(round_half_even(W / gamma), -1, 1), division in float. */
void oracle_ternarize(const float *w, int64_t n, float gamma, int8_t *q) {
    for (int64_t i = 0; i < n; ++i) {
        float r = w[i] / gamma;
        float t = rintf(r); /* default rounding mode: to nearest, ties to even */
        if (t > 1.0f) t = 1.0f;
        if (t < -1.0f) t = -1.0f;
        q[i] = (int8_t)t;
    }
}

/* Position of weight k inside its row: byte offset and bit offset. */
static void code_position(int64_t k, int64_t *byte, int *bit) {
    int64_t word = k / 16;
    int within = (int)(k % 16);
    int j = within / 4, i = within % 4;
    *byte = word * 4 + i;  /* little-endian: bits 8i..8i+7 of the word live in byte i */
    *bit = 2 * j;
}

int oracle_pack(const int8_t *q, int64_t N, int64_t K, uint8_t *packed) {
    if (N <= 0 || K <= 0 || K % 16) return OR_ERR_SHAPE;
    memset(packed, 0, (size_t)(N * (K / 4)));
    for (int64_t n = 0; n < N; ++n) {
        uint8_t *row = packed + n * (K / 4);
        for (int64_t k = 0; k < K; ++k) {
            int8_t v = q[n * K + k];
            unsigned code;  /* 1 - v */
            if (v == 1) code = 0u;
            else if (v == 0) code = 1u;
            else if (v == -1) code = 2u;
            else return OR_ERR_RANGE;
            int64_t byte; int bit;
            code_position(k, &byte, &bit);
            row[byte] |= (uint8_t)(code << bit);
        }
    }
    return OR_OK;
}

/* Inverse of oracle_pack; the reserved code 11 is reported as an error. */
int oracle_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *q) {
    if (N <= 0 || K <= 0 || K % 16) return OR_ERR_SHAPE;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = packed + n * (K / 4);
        for (int64_t k = 0; k < K; ++k) {
            int64_t byte; int bit;
            code_position(k, &byte, &bit);
            unsigned code = (row[byte] >> bit) & 3u;
            if (code == 3u) return OR_ERR_RANGE;
            q[n * K + k] = (int8_t)(1 - (int)code);
        }
    }
    return OR_OK;
}

int oracle_quant_weights(const float *W, int64_t N, int64_t K, uint8_t *packed,
                         float *gamma, int8_t *wq_scratch) {
    int rc = oracle_absmean_gamma(W, N * K, gamma);
    if (rc) return rc;
    oracle_ternarize(W, N * K, *gamma, wq_scratch);
    return oracle_pack(wq_scratch, N, K, packed);
}

/* ------------------------------------------------------------------------ */
/* Step 3: per-token INT8 activation quant, optionally after SubLN.           */
/* ------------------------------------------------------------------------ */

/* Exact sum of x_k^2 in units of 2^-298 (9 limbs cover every finite float and
 * K <= 2^17 terms), rounded once to double. */
static int sum_squares_exact(const float *x, int64_t K, double *out) {
    uint64_t limbs[9];
    memset(limbs, 0, sizeof(limbs));
    for (int64_t k = 0; k < K; ++k) {
        uint32_t u;
        memcpy(&u, &x[k], 4);
        u &= 0x7fffffffu;
        uint32_t e = u >> 23;
        uint64_t m = u & 0x7fffffu;
        if (e == 255) return OR_ERR_NONFINITE;
        if (e > 0) m |= 0x800000u;
        int shift = e > 0 ? 2 * ((int)e - 1) : 0; /* x^2 = m^2 * 2^(shift - 298) */
        if (m) big_add_shifted(limbs, 9, m * m, shift);
    }
    *out = big_to_double(limbs, 9, -298);
    return OR_OK;
}

/* SubLN: y = (x / sqrt(mean(x^2) + eps)) * g. */
int oracle_rmsnorm(const float *x, int64_t K, const float *g, float eps, float *y) {
    double S2;
    int rc = sum_squares_exact(x, K, &S2);
    if (rc) return rc;
    float ms = (float)(S2 / (double)K);
    float r = sqrtf(ms + eps);
    for (int64_t k = 0; k < K; ++k) {
        float t = x[k] / r;
        y[k] = t * g[k];
    }
    return OR_OK;
}

/* Absmax quant of one row: s = 127 / max(max|x|, 1e-5f);
 * x_q = clamp(round_half_even(x * s), -128, 127). */
static void quant_row(const float *y, int64_t K, int8_t *xq, float *s_out) {
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = fabsf(y[k]);
        if (v > a) a = v;
    }
    float s = 127.0f / (a > 1e-5f ? a : 1e-5f);
    for (int64_t k = 0; k < K; ++k) {
        float t = rintf(y[k] * s);
        if (t > 127.0f) t = 127.0f;
        if (t < -128.0f) t = -128.0f;
        xq[k] = (int8_t)t;
    }
    *s_out = s;
}

/* X [M, K] row-major.  gain == NULL: plain quant; otherwise SubLN first.
 * y_scratch must hold K floats per thread when gain != NULL (rows are
 * processed independently; OpenMP over rows). */
int oracle_quant_act(const float *X, int64_t M, int64_t K, const float *gain, float eps,
                     int8_t *xq, float *s, float *y_scratch) {
    if (M <= 0 || K <= 0) return OR_ERR_SHAPE;
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(|:bad)
    for (int64_t m = 0; m < M; ++m) {
        const float *row = X + m * K;
        if (gain) {
            float *y = y_scratch + m * K;
            if (oracle_rmsnorm(row, K, gain, eps, y)) { bad |= 1; continue; }
            quant_row(y, K, xq + m * K, s + m);
        } else {
            quant_row(row, K, xq + m * K, s + m);
        }
    }
    return bad ? OR_ERR_NONFINITE : OR_OK;
}

/* ------------------------------------------------------------------------ */
/* FFN activation between the up and down projections: "SLM750-Edge" model  */
/* card, "Key Architectural Features" (FFN activation ReLU2, relu(x)^2) and   */
/* section 2.3 (per-layer FFN gate, up and down projections).  Reading: the   */
/* gated form h = relu(gate)^2 * up, each step a float operation:             */
/*   r = gate > 0 ? gate : 0;  h = float(float(r * r) * up).                  */
/* h is the input of the down projection's SubLN + activation quantizer       */
/* ("BitDistill", Stage 1), i.e. oracle_quant_act on h.                       */
/* ------------------------------------------------------------------------ */
void oracle_ffn_act(const float *gate, const float *up, int64_t n, float *h) {
    for (int64_t i = 0; i < n; ++i) {
        float r = gate[i] > 0.0f ? gate[i] : 0.0f;
        float sq = r * r;
        h[i] = sq * up[i];
    }
}

/* ------------------------------------------------------------------------ */
/* Step 4: exact contraction; step 5: rescale.                                */
/* ------------------------------------------------------------------------ */

/* acc[m, n] = sum_k xq[m, k] * wq[n, k] in int64. */
void oracle_contract(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                     int64_t *acc) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k)
                a += (int64_t)xq[m * K + k] * (int64_t)wq[n * K + k];
            acc[m * N + n] = a;
        }
    }
}

/* Only the listed (m, n) pairs; used where the full product is too large. */
void oracle_contract_pairs(const int8_t *xq, const int8_t *wq, int64_t K,
                           const int64_t *ms, const int64_t *ns, int64_t npairs,
                           int64_t *acc) {
    #pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npairs; ++p) {
        int64_t a = 0;
        for (int64_t k = 0; k < K; ++k)
            a += (int64_t)xq[ms[p] * K + k] * (int64_t)wq[ns[p] * K + k];
        acc[p] = a;
    }
}

/* Y = acc * gamma / s, evaluated in double. */
void oracle_rescale(const int64_t *acc, int64_t count, float gamma, const float *s_per_item,
                    double *Y) {
    for (int64_t i = 0; i < count; ++i)
        Y[i] = (double)acc[i] * (double)gamma / (double)s_per_item[i];
}

/* ------------------------------------------------------------------------
 * Backward of the quantization-aware BitLinear (straight-through estimator).
 *
 * The pages fix only the rule: gradients pass through the quantizers
 * unchanged ("Distillix" README, 1. BitNet b1.58 Core: "STE"; "BitDistill",
 * Evaluation and results: gradients through the activation quantizer use the
 * straight-through estimator), the weight gradient optionally masked by the
 * hard or the soft STE scale of "bitone" README, Soft-STE notes:
 *   hard:  scale = 1 if |w / gamma| <= 1, else 0
 *   soft:  scale = 1 - tanh^2(beta * w / gamma)        (beta = 2 by default)
 * Readings (the plainest ones; listed in the design notes):
 *   - the forward is Y = (x_q / s) @ (gamma W_q)^T, so with both quantizers
 *     passed straight through, dX = dY @ (gamma W_q) and the weight receives
 *     dW = (dY^T @ (x_q / s)) * scale(W / gamma); gamma's own dependence on W
 *     is not differentiated (it is part of the quantizer);
 *   - w / gamma is the float division of the forward (the mask is an integer
 *     decision, taken in the forward's precision); everything else is double.
 * ------------------------------------------------------------------------ */

/* dX [M, K] = dY [M, N] @ (gamma * W_q) [N, K], in double, n ascending. */
void oracle_bwd_dx(const float *dY, const int8_t *wq, float gamma, int64_t M, int64_t N, int64_t K,
                   double *dX) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double a = 0.0;
            for (int64_t n = 0; n < N; ++n)
                a += (double)dY[m * N + n] * (double)wq[n * K + k];
            dX[m * K + k] = a * (double)gamma;
        }
}

/* STE scale of one latent weight: beta <= 0 selects the hard mask. */
static double ste_scale(float w, float gamma, double beta) {
    const float ws = w / gamma; /* float division, as in the forward */
    if (beta <= 0.0) return fabsf(ws) <= 1.0f ? 1.0 : 0.0;
    const double t = tanh(beta * (double)ws);
    return 1.0 - t * t;
}

/* dW [N, K] = (dY^T @ (x_q / s)) * scale(W / gamma), in double, m ascending. */
int oracle_bwd_dw(const float *dY, const int8_t *xq, const float *s, const float *W, float gamma,
                  double beta, int64_t M, int64_t N, int64_t K, double *dW) {
    if (!(gamma > 0.0f)) return OR_ERR_SHAPE;
    for (int64_t m = 0; m < M; ++m)
        if (!(s[m] > 0.0f)) return OR_ERR_SHAPE;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            double a = 0.0;
            for (int64_t m = 0; m < M; ++m)
                a += (double)dY[m * N + n] * ((double)xq[m * K + k] / (double)s[m]);
            dW[n * K + k] = a * ste_scale(W[n * K + k], gamma, beta);
        }
    return OR_OK;
}
