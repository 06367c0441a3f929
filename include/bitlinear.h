/*
 * bitlinear.h -- C ABI of libbitlinear.so: the BitNet b1.58 BitLinear forward
 * on NVIDIA B200 (sm_100a).
 *
 * The forward has four steps; each entry point below names the passage that
 * defines what it computes:
 *   1. absmean weight quantization + 2-bit packing      bl_quant_weights
 *   2. per-token absmax INT8 activation quantization    bl_quant_act
 *      (optionally after a SubLN RMSNorm)
 *   3. exact ternary x INT8 contraction (int32)          bl_forward
 *   4. rescale Y = acc * gamma / s                       bl_forward
 *   all four in one call                                 bl_linear
 *
 * Conventions shared by every entry point
 *   - Shapes: W is [N, K] row-major (out_features x in_features, as a torch
 *     Linear weight), X is [M, K] row-major, Y is [M, N] row-major float32:
 *     Y = X * W^T.
 *   - Every data pointer is a DEVICE pointer on the current CUDA device,
 *     allocated and owned by the caller; the library never allocates, frees
 *     or keeps a pointer after the call returns.  Pointers must be 16-byte
 *     aligned; rows are contiguous (no strides).
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream); a returned BL_OK means "validated and launched".  Outputs are
 *     ready when the stream has reached that point.
 *   - No exception crosses the ABI; errors are returned as bl_status.  Bad
 *     arguments are detected on the host before anything is launched, and
 *     nothing is written then.  Device-side bounded waits that give up set a
 *     sticky device error word, read (and cleared) by bl_check_device_error.
 *   - Inputs must be finite; NaN or Inf input gives unspecified (but memory-
 *     safe) outputs.
 *   - Limits: 1 <= M <= 2^31-1, 1 <= N <= 2^31-1, 64 <= K <= 32768 with
 *     K % 64 == 0; N*K < 2^31 for the weight quantizer.  With |x_q| <= 127
 *     and K <= 32768, |acc| <= 2^22, so acc converts to float exactly.
 *
 * Packed weight format (the pages give no layout; they state ~1.58 bits per
 * weight, "bitone" README, "How 1.58-bit Works", and a memory table at
 * ~1.6 bits): 2 bits per weight, N * K / 4 bytes.  Row n occupies K/4
 * contiguous bytes = K/16 little-endian 32-bit words.  Weight k = 16*w + 4*j
 * + i (0 <= i, j < 4) has its code in word w at bits [8*i + 2*j,
 * 8*i + 2*j + 1].  The code is 1 - W_q as a 2-bit unsigned number: 00 = +1,
 * 01 = 0, 10 = -1; 11 is never written (a zero weight matrix packs to 0x55
 * bytes).  So byte i of a word holds the codes of k = i, i+4,
 * i+8, i+12 of its 16-weight group.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; the header needs no CUDA include. */
typedef struct CUstream_st *bl_stream_t;

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,      /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,     /* M, N, K (or a group count) outside the limits above */
    BL_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned */
    BL_ERR_DTYPE = 4,     /* unknown bl_dtype code */
    BL_ERR_CUDA = 5,      /* a CUDA runtime call or kernel launch failed */
    BL_ERR_TIMEOUT = 6,   /* a bounded device-side wait gave up (see bl_check_device_error) */
    BL_ERR_WORKSPACE = 7, /* workspace NULL or smaller than the *_workspace_bytes query */
    BL_ERR_DEVICE = 8     /* the current device is not a compute capability 10.x GPU */
} bl_status;

typedef enum {
    BL_F32 = 0,  /* IEEE float32 */
    BL_BF16 = 1  /* bfloat16 (upcast to float32 exactly) */
} bl_dtype;

/* Human-readable name of a status code; never NULL. */
const char *bl_status_string(bl_status s);

/* Library ABI version (major * 100 + minor). */
int bl_version(void);

/* Reads and clears the device error word set by bounded device-side waits.
 * Synchronizes `stream` first.  Returns BL_OK, BL_ERR_TIMEOUT or
 * BL_ERR_CUDA. */
bl_status bl_check_device_error(bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 1: absmean ternary weight quantization + 2-bit packing.              */
/*                                                                           */
/* Defined by: "Distillix" README, "Key Innovations / 1. BitNet b1.58 Core"  */
/* (W_q = round(clip(W / mean|W|, -1, 1))); "bitone" README, Triton-fused   */
/* QAT BitLinear "Forward pass" (gamma = mean(|W|) from one reduction over   */
/* W, then W_q per tile); "SLM750-Edge" model card, section 3.1 "Ternary     */
/* Weight Quantization" (round_clip: 0 when |W/gamma| <= 0.5).               */
/*                                                                           */
/*   gamma = float(double(S) / double(N*K)) + 1e-5f, S = sum |W| exactly     */
/*           (order-independent; rounded once to double)                     */
/*   W_q   = clamp(round_half_even(float(W / gamma)), -1, 1)                 */
/*                                                                           */
/* W        [N, K] of dtype wdt (BL_F32 or BL_BF16), device                  */
/* packed   [N, K/4] bytes out, format above, device                         */
/* gamma    1 float out, device                                              */
/* workspace device scratch of at least bl_quant_weights_workspace_bytes();  */
/*          contents on entry are ignored, clobbered on exit                 */
/* Errors: NULL pointer, misalignment, K % 64, N*K >= 2^31, small workspace. */
/* ------------------------------------------------------------------------ */
size_t bl_quant_weights_workspace_bytes(int64_t N, int64_t K);
bl_status bl_quant_weights(const void *W, bl_dtype wdt, int64_t N, int64_t K,
                           uint8_t *packed, float *gamma,
                           void *workspace, size_t workspace_bytes, bl_stream_t stream);

/* Same computation and outputs as bl_quant_weights, for callers that cannot
 * allocate device memory: a plain C host or a runtime that only hands out
 * pointers to tensors it owns, or a program whose device-memory budget is
 * fixed at start-up.  The scratch the reduction needs lives in a static
 * device array inside the library (BL_NOALLOC_SCRATCH_BYTES bytes on every
 * GPU that loads the library, held until process exit); this call never
 * calls cudaMalloc or cudaFree.  No source page has a counterpart: this is
 * an interface convenience of this library.
 *   - Limits: those of bl_quant_weights (N*K < 2^31, K % 64 == 0,
 *     64 <= K <= 32768); the fixed scratch covers every such size.  Other
 *     sizes return BL_ERR_SHAPE.
 *   - The first call on each device looks up the device address of the
 *     static scratch (cudaGetSymbolAddress) with that device current; make
 *     that first call before any stream capture.
 *   - All calls on a device share the one scratch array and it keeps the
 *     previous call's contents (the kernels overwrite every word they read,
 *     so nothing needs clearing).  Calls whose kernels overlap on the GPU --
 *     different streams, or different host threads -- race on it: serialize
 *     them (one stream, or events). */
#define BL_NOALLOC_SCRATCH_BYTES 49408
bl_status bl_quant_weights_noalloc(const void *W, bl_dtype wdt, int64_t N, int64_t K,
                                   uint8_t *packed, float *gamma, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 1 for several weight matrices in three launches (one reduction      */
/* grid, one finalize grid of a block per matrix and one pack grid over all  */
/* of them), e.g. the projections of a layer that are re-quantized every     */
/* call: their reduction latency chains overlap instead of running one       */
/* after the other.  Same definition and the same bits as bl_quant_weights   */
/* for each matrix.                                                          */
/*                                                                           */
/* problems  HOST array of `count` (1 <= count <= BL_MAX_WQ_GROUP) matrices, */
/*           read during the call only; each W of dtype wdt, each with its    */
/*           own packed and gamma outputs (device); limits per matrix as for */
/*           bl_quant_weights                                                */
/* workspace device scratch of at least bl_quant_weights_workspace_bytes()   */
/*           (the same size as for one matrix), clobbered                    */
/* ------------------------------------------------------------------------ */
#define BL_MAX_WQ_GROUP 8

typedef struct {
    const void *W;    /* [N, K] of the call's dtype */
    int64_t N;
    int64_t K;
    uint8_t *packed;  /* [N, K/4] out */
    float *gamma;     /* [1] out */
} bl_weight_problem;

bl_status bl_quant_weights_grouped(const bl_weight_problem *problems, int count, bl_dtype wdt,
                                   void *workspace, size_t workspace_bytes, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 2: per-token absmax INT8 activation quantization, optionally fused  */
/* with a preceding SubLN RMSNorm.                                           */
/*                                                                           */
/* Defined by: "BitDistill" article, "Evaluation and results" (activations   */
/* quantized to INT8); SubLN placement: "BitDistill", "Stage 1 --            */
/* Architectural refinement with SubLN" (before the attention output and    */
/* FFN output projections); "SLM750-Edge" section 2.1 (SubLN = pre-RMSNorm + */
/* activation quantization) and "Key Architectural Features" (RMSNorm eps    */
/* 1e-6).                                                                    */
/*                                                                           */
/*   y   = x                                   if subln_gain == NULL         */
/*   y_k = float(float(x_k / r) * g_k)         otherwise, with               */
/*         r = sqrtf(float(double(sum_k x_k^2) / K) + eps), the sum exact    */
/*   s   = float(127 / max(max_k |y_k|, 1e-5f))                              */
/*   x_q = clamp(round_half_even(float(y * s)), -128, 127)                   */
/*                                                                           */
/* X [M, K] of dtype xdt; subln_gain [K] float or NULL; x_q [M, K] int8 out;  */
/* s [M] float out.  All device.                                             */
/* ------------------------------------------------------------------------ */
bl_status bl_quant_act(const void *X, bl_dtype xdt, int64_t M, int64_t K,
                       const float *subln_gain, float subln_eps,
                       int8_t *x_q, float *s, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Step 2 for the down projection, fused with the FFN activation before it.  */
/*                                                                           */
/* Defined by: "SLM750-Edge" model card, "Key Architectural Features" (FFN   */
/* activation ReLU2, relu(x)^2) and section 2.3 (gate, up and down           */
/* projections per layer); the gated reading h = relu(gate)^2 * up; then the */
/* SubLN + activation quantizer of bl_quant_act on h ("BitDistill", Stage 1: */
/* SubLN before down_proj):                                                  */
/*                                                                           */
/*   h   = float(float(r * r) * up),  r = gate > 0 ? gate : 0                */
/*   x_q, s = bl_quant_act(h, subln_gain, subln_eps)   (h never stored)      */
/*                                                                           */
/* gate, up [M, F] float32 (the gate / up projections' Y); subln_gain [F] or */
/* NULL; x_q [M, F] int8 out; s [M] out.  All device, 16-byte aligned.      */
/* F obeys the K limits (64 <= F <= 32768, F % 64 == 0).                     */
/* ------------------------------------------------------------------------ */
bl_status bl_ffn_act_quant(const float *gate, const float *up, int64_t M, int64_t F,
                           const float *subln_gain, float subln_eps,
                           int8_t *x_q, float *s, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Steps 3 + 4: exact ternary x INT8 contraction and rescale.                */
/*                                                                           */
/* Defined by: "bitone" README, "How 1.58-bit Works" (each weight adds,      */
/* subtracts or skips an input: no multiplication needed) and "Forward      */
/* pass" (Y = X @ W_q^T * gamma), with the INT8 scale s of step 2:           */
/*                                                                           */
/*   acc[m, n] = sum_k x_q[m, k] * W_q[n, k]          (exact, int32)         */
/*   Y[m, n]   = float(float(acc) * float(gamma / s[m]))                     */
/*               (two float roundings: |Y - acc*gamma/s| <= 2^-23 |Y|)       */
/*                                                                           */
/* Engine: the bandwidth-bound decode GEMV when M <= 16 and the staged     */
/* activations fit, M * round_up(K, 256) <= 147456 bytes (M <= 16 for      */
/* K <= 9216, M <= 15 at K = 9728, M <= 9 at K = 16384, M <= 4 at           */
/* K = 32768), otherwise the tcgen05 prefill GEMM.  Both give identical acc. */
/* packed [N, K/4] (format above); gamma [1]; x_q [M, K]; s [M]; Y [M, N]    */
/* out; acc_out [M, N] int32 out or NULL.  All device.                       */
/* ------------------------------------------------------------------------ */
bl_status bl_forward(const uint8_t *packed, const float *gamma, const int8_t *x_q,
                     const float *s, int64_t M, int64_t N, int64_t K, float *Y,
                     int32_t *acc_out, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Steps 3 + 4 of the gate and up projections of an FFN, fused with the FFN  */
/* activation between them and the down projection, in ONE tcgen05 launch:  */
/*                                                                           */
/*   h = float(float(r * r) * Y_up),  r = max(Y_gate, 0)                     */
/*                                                                           */
/* with Y_gate and Y_up the bits bl_forward would give for the two          */
/* projections on the shared x_q, s; only h is written (the gate and up     */
/* outputs never reach memory).  Defined by: "SLM750-Edge" model card, "Key */
/* Architectural Features" (FFN activation ReLU2) and section 2.3 (gate,    */
/* up, down); "bitone" README, Forward pass (Y = X @ W_q^T * gamma).        */
/* h then feeds bl_quant_act (with the down projection's SubLN gain).       */
/*                                                                           */
/* packed_gate, packed_up [F, K/4]; gamma_gate, gamma_up [1]; x_q [M, K];    */
/* s [M]; h [M, F] float32 out.  All device, 16-byte aligned.  F % 64 == 0  */
/* and 64 <= F <= 2^31 - 1 (F is the down projection's K); K as for        */
/* bl_forward.  Any M (the tcgen05 engine; decode-sized calls do better     */
/* with bl_linear_decode_grouped + bl_ffn_act_quant).                        */
/* ------------------------------------------------------------------------ */
bl_status bl_forward_glu(const uint8_t *packed_gate, const float *gamma_gate, const uint8_t *packed_up,
                         const float *gamma_up, const int8_t *x_q, const float *s, int64_t M, int64_t F,
                         int64_t K, float *h, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Backward of the quantization-aware BitLinear, activation gradient, with  */
/* the straight-through estimator ("Distillix" README, 1. BitNet b1.58      */
/* Core: STE; "BitDistill", Evaluation and results: gradients pass the      */
/* activation quantizer unchanged).  With the forward Y = (x_q/s) (gamma    */
/* W_q)^T and both quantizers passed straight through:                       */
/*                                                                           */
/*   dX[m, k] = float(gamma * float(sum_n dY[m, n] * W_q[n, k]))             */
/*                                                                           */
/* the sum in float32 on the tensor cores (bf16 x ternary products are      */
/* exact; the accumulation order is the hardware's, so dX agrees with the   */
/* exact value within about N * 2^-23 of sum_n |dY[m, n] W_q[n, k]| gamma). */
/*                                                                           */
/* dY [M, N] bfloat16 (N % 8 == 0); packed [N, K/4] and gamma [1] as the    */
/* forward's (bl_quant_weights); dX [M, K] float32 out.  All device, 16-byte */
/* aligned.  K as for bl_forward.                                            */
/* ------------------------------------------------------------------------ */
bl_status bl_backward_dx(const void *dY, const uint8_t *packed, const float *gamma, int64_t M, int64_t N,
                         int64_t K, float *dX, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Backward of the quantization-aware BitLinear, weight gradient, with the  */
/* straight-through estimator and the hard or soft STE scale ("Distillix"   */
/* README, 1. BitNet b1.58 Core: STE; "bitone" README, Soft-STE notes:      */
/* hard mask |w / gamma| <= 1, soft scale 1 - tanh^2(beta w / gamma)):      */
/*                                                                           */
/*   dW[n, k] = float(float(sum_m dY[m, n] * xs[m, k]) * scale(r))           */
/*   xs = bf16(float(x_q / s)), r = float(W[n, k] / gamma)                   */
/*   scale(r) = |r| <= 1 ? 1 : 0 (beta <= 0),  1 - tanhf(beta r)^2 otherwise */
/*                                                                           */
/* the sum over the tokens in float32 on the tensor cores after both         */
/* operands are laid out with the tokens contiguous (two transposes into    */
/* the workspace); xs is rounded to bf16 (2^-9 relative), so dW agrees with */
/* the exact value within about (2^-8 + M * 2^-23) of                       */
/* sum_m |dY[m, n] x_q[m, k] / s[m]| * scale.                                */
/*                                                                           */
/* dY [M, N] bfloat16; x_q [M, K], s [M] from the forward's bl_quant_act;    */
/* W [N, K] the latent weights (wdt), gamma [1] their forward scale;         */
/* dW [N, K] float32 out; workspace >= bl_backward_dw_workspace_bytes(M, N,  */
/* K).  All device, 16-byte aligned.  K as for bl_forward, N >= 1.           */
/* ------------------------------------------------------------------------ */
size_t bl_backward_dw_workspace_bytes(int64_t M, int64_t N, int64_t K);
bl_status bl_backward_dw(const void *dY, const int8_t *x_q, const float *s, const void *W, bl_dtype wdt,
                         const float *gamma, float beta, int64_t M, int64_t N, int64_t K, void *workspace,
                         size_t workspace_bytes, float *dW, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* All four steps in one call: bl_quant_weights, bl_quant_act, bl_forward    */
/* (for decode-eligible M, steps 2-4 run as one fused launch, with the same  */
/* results).                                                                 */
/* workspace >= bl_linear_workspace_bytes(M, N, K) holds packed W, gamma,    */
/* x_q and s between the steps.                                              */
/* ------------------------------------------------------------------------ */
size_t bl_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);
bl_status bl_linear(const void *W, bl_dtype wdt, const void *X, bl_dtype xdt,
                    int64_t M, int64_t N, int64_t K,
                    const float *subln_gain, float subln_eps,
                    void *workspace, size_t workspace_bytes, float *Y, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Grouped steps 3+4, ONE kernel launch, same arithmetic as bl_forward:      */
/*  - decode: when every problem is decode-eligible (M <= 16 and the staging */
/*    fits, see bl_forward), up to BL_MAX_GROUP independent problems that    */
/*    share M (e.g. every projection of a decode step);                      */
/*  - prefill: otherwise, up to BL_MAX_PREFILL_GROUP problems that share the */
/*    same x_q, s and K (e.g. the q, k, v or the gate, up projections of one */
/*    layer): their output tiles run in one persistent tcgen05 launch.       */
/*    Problems with different x_q / s / K, or more of them, give             */
/*    BL_ERR_SHAPE.                                                          */
/* `problems` is a HOST array, read during the call only.                    */
/* flags: 0, or BL_FWD_WEIGHTS_READY -- the caller promises that every       */
/* problem's packed weights and gamma were complete before the kernel        */
/* enqueued just before this call began; the engine may then be launched as */
/* a programmatic dependent launch that streams weights while that kernel    */
/* finishes (it still waits for it before reading x_q and s).                */
/* ------------------------------------------------------------------------ */
#define BL_MAX_GROUP 128
#define BL_MAX_PREFILL_GROUP 4
#define BL_FWD_WEIGHTS_READY 1u

typedef struct {
    const uint8_t *packed;  /* [N, K/4] */
    const float *gamma;     /* [1] */
    const int8_t *x_q;      /* [M, K] */
    const float *s;         /* [M] */
    float *Y;               /* [M, N] out */
    int32_t *acc_out;       /* [M, N] out or NULL */
    int64_t N;
    int64_t K;
} bl_problem;

bl_status bl_forward_grouped(const bl_problem *problems, int count, int64_t M, unsigned flags,
                             bl_stream_t stream);

/* Grouped step 2: up to BL_MAX_GROUP activation inputs sharing M and dtype,
 * one launch.  Same arithmetic as bl_quant_act.  `problems` is a HOST
 * array. */
typedef struct {
    const void *X;           /* [M, K] of the call's dtype */
    const float *subln_gain; /* [K] or NULL */
    int8_t *x_q;             /* [M, K] out */
    float *s;                /* [M] out */
    int64_t K;
} bl_act_problem;

bl_status bl_quant_act_grouped(const bl_act_problem *problems, int count, bl_dtype xdt,
                               int64_t M, float subln_eps, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Grouped decode from raw activations: steps 2 + 3 + 4 in ONE launch.       */
/*                                                                           */
/* Defined by the same passages as bl_quant_act and bl_forward: for each     */
/* problem, x_q and s are what bl_quant_act(X, subln_gain, subln_eps) would  */
/* produce (bit for bit), and Y / acc what bl_forward would produce from     */
/* them.  x_q never has to reach global memory: each CTA quantizes the rows  */
/* it needs into on-chip memory while its packed weights stream in.          */
/*                                                                           */
/* X [M, K] of dtype xdt; subln_gain [K] float or NULL (RMSNorm before the   */
/* quantizer, epsilon subln_eps); packed [N, K/4]; gamma [1]; Y [M, N] out.  */
/* Optional outputs (NULL = not written): x_q [M, K] int8, s [M] float,      */
/* acc_out [M, N] int32.  All device pointers, 16-byte aligned; `problems`   */
/* is a HOST array read during the call only.  M <= 16 and every problem    */
/* decode-eligible (see bl_forward), else BL_ERR_SHAPE.  flags: 0 or         */
/* BL_FWD_WEIGHTS_READY (as for bl_forward_grouped; X may still be written  */
/* by the kernel enqueued just before: it is read only after that kernel    */
/* completes).                                                               */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint8_t *packed;    /* [N, K/4] */
    const float *gamma;       /* [1] */
    const void *X;            /* [M, K] of the call's dtype */
    const float *subln_gain;  /* [K] or NULL */
    float *Y;                 /* [M, N] out */
    int8_t *x_q;              /* [M, K] out or NULL */
    float *s;                 /* [M] out or NULL */
    int32_t *acc_out;         /* [M, N] out or NULL */
    int64_t N;
    int64_t K;
} bl_decode_problem;

bl_status bl_linear_decode_grouped(const bl_decode_problem *problems, int count, bl_dtype xdt,
                                   int64_t M, float subln_eps, unsigned flags, bl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* All four steps for up to BL_MAX_PREFILL_GROUP weight matrices that share  */
/* one input X (the q, k, v or the gate, up projections of a layer), every  */
/* weight re-quantized in the call: one grouped weight quantization (two     */
/* launches), ONE activation quantization of X, and one grouped contraction */
/* launch (the tcgen05 GEMM over all matrices' output tiles, or for         */
/* decode-sized M the fused decode launch, which quantizes X itself).  Each  */
/* Y_i carries the bits bl_linear(W_i, X) gives.                             */
/*                                                                           */
/* problems  HOST array of `count` matrices, read during the call only      */
/* X         [M, K] of dtype xdt, device; subln_gain [K] or NULL             */
/* workspace >= bl_linear_grouped_workspace_bytes(problems, count, M, K):    */
/*           packed weights, gammas, x_q and s between the steps             */
/* Errors: as bl_linear; BL_ERR_SHAPE for count outside [1, 4].              */
/* ------------------------------------------------------------------------ */
typedef struct {
    const void *W;  /* [N, K] of the call's weight dtype */
    float *Y;       /* [M, N] out */
    int64_t N;
} bl_linear_problem;

size_t bl_linear_grouped_workspace_bytes(const bl_linear_problem *problems, int count, int64_t M, int64_t K);
bl_status bl_linear_grouped(const bl_linear_problem *problems, int count, bl_dtype wdt, const void *X,
                            bl_dtype xdt, int64_t M, int64_t K, const float *subln_gain, float subln_eps,
                            void *workspace, size_t workspace_bytes, bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
