/*
 * bitlinear_debug.h -- test hooks of libbitlinear.so (not for production use).
 *
 * bl_debug_forward_prefill: steps 3 + 4 exactly as bl_forward defines them
 * ("bitone" README, How 1.58-bit Works and Forward pass), but always through
 * the tcgen05 prefill engine, whatever M (so tests can cover that engine at
 * small M), with every device-side wait limited to `timeout_us`
 * microseconds.  With skip_iter >= 0 the engine's TMA producer never issues
 * its k-iteration number `skip_iter` (counted per CTA), so the consumers'
 * bounded waits run out: the call returns BL_OK, bl_check_device_error then
 * returns BL_ERR_TIMEOUT, Y and acc_out are unspecified, and the CUDA
 * context stays usable.  skip_iter < 0 disables the stall.  Arguments and
 * errors as for bl_forward, plus BL_ERR_SHAPE for timeout_us == 0.
 */
#ifndef BITLINEAR_DEBUG_H
#define BITLINEAR_DEBUG_H

#include "bitlinear.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bl_debug_decode_plan: the launches a decode call (bl_forward_grouped or
 * bl_linear_decode_grouped at M <= 16) over `count` problems of the given
 * shapes (shapes[2i] = N, shapes[2i + 1] = K, host array) would make on a GPU
 * with `sms` SMs, computed on the host without launching anything.  For each
 * launch, out[] receives: CTAs, dynamic shared memory bytes, problems, then
 * per problem: its index in `shapes`, first row, rows, log2 of the warps per
 * 32-row group, K chunks (1 = whole rows), first CTA.  *written = ints
 * written.  Errors: NULL pointer; BL_ERR_SHAPE for count outside [1,
 * BL_MAX_GROUP], M outside [1, 16], sms < 1 or a shape a decode call rejects;
 * BL_ERR_WORKSPACE when out_len is too small.
 */
bl_status bl_debug_decode_plan(const int64_t *shapes, int count, int64_t M, int sms, int *out, int out_len,
                               int *written);

bl_status bl_debug_forward_prefill(const uint8_t *packed, const float *gamma, const int8_t *x_q,
                                   const float *s, int64_t M, int64_t N, int64_t K, float *Y,
                                   int32_t *acc_out, long long skip_iter, uint32_t timeout_us,
                                   bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_DEBUG_H */
