// Steps 3 + 4 for large M.  Interim engine: the decode GEMV run over token
// chunks small enough for its shared-memory staging.
#pragma once

#include "bl_common.cuh"
#include "k_decode.cuh"

namespace bl {

inline cudaError_t prefill_setup() { return cudaSuccess; }

inline bl_status prefill_launch(const uint8_t *packed, const float *gamma, const int8_t *x_q, const float *s,
                                int64_t M, int64_t N, int64_t K, float *Y, int32_t *acc_out, cudaStream_t st) {
    int rs = dec_row_stride((int)K);
    int64_t chunk = DEC_MAX_XQ_SMEM / rs;
    if (chunk > 16) chunk = 16;
    if (chunk < 1) return BL_ERR_SHAPE;
    for (int64_t m0 = 0; m0 < M; m0 += chunk) {
        int64_t mc = M - m0 < chunk ? M - m0 : chunk;
        DecodeParams P;
        P.count = 1;
        P.M = (int)mc;
        int glog = 0;
        {
            int steps = (int)((K + 255) / 256);
            glog = steps <= 3 ? 0 : steps <= 6 ? 1 : steps <= 12 ? 2 : 3;
        }
        P.p[0] = DecodeProblem{packed, gamma, x_q + m0 * K, s + m0, Y + m0 * N,
                               acc_out ? acc_out + m0 * N : nullptr, (int)N, (int)K, glog, 0};
        int tiles = (int)((N + 15) / 16);
        int per = DEC_WARPS >> glog;
        int ctas = (tiles + per - 1) / per;
        size_t smem = (size_t)mc * rs;
        if (mc <= 8)
            k_decode<1><<<ctas, DEC_THREADS, smem, st>>>(P);
        else
            k_decode<2><<<ctas, DEC_THREADS, smem, st>>>(P);
        if (cudaGetLastError() != cudaSuccess) return BL_ERR_CUDA;
    }
    return BL_OK;
}

}  // namespace bl
