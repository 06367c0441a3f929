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

bl_status bl_debug_forward_prefill(const uint8_t *packed, const float *gamma, const int8_t *x_q,
                                   const float *s, int64_t M, int64_t N, int64_t K, float *Y,
                                   int32_t *acc_out, long long skip_iter, uint32_t timeout_us,
                                   bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_DEBUG_H */
