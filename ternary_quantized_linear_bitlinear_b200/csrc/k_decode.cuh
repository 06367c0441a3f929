// Steps 3 + 4 for decode-sized M (<= 16): the ternary x INT8 GEMV engine.
//
// What it computes ("bitone" README, How 1.58-bit Works and Forward pass):
//   acc[m, n] = sum_k x_q[m, k] * W_q[n, k];  Y[m, n] = acc * (gamma / s[m])
//
// The work is bound by streaming the packed weights from HBM (2 bits per
// weight).  Design:
//   - A warp owns a 16-row tile of W; a CTA (8 warps) owns 8/G tiles, with G
//     warps splitting each tile's K range (G picked per problem from K).
//   - Each thread streams 16 bytes of row g and 16 bytes of row g+8 per
//     256-k step with 128-bit non-caching loads; lanes of a quad read one
//     contiguous 64-byte run of a row.
//   - Unpacking costs 1-2 ALU ops per 4 weights: with the packed layout, word
//     (w << (6 - 2j)) & 0xC0C0C0C0 puts the codes of k = 16w' + 4j .. 4j+3 in
//     the top two bits of four bytes, i.e. the int8 values 64 * W_q.
//   - The MACs run on the tensor cores (mma.sync m16n8k32 s8): W tile as A
//     (16 rows), tokens as B (8 columns, zero for m >= M).  Because the
//     int32 sum is exact, the k order inside a step may be permuted as long
//     as A and B use the same permutation: thread t's A fragment for step
//     pair c holds k = 64t + 16c + (0..15), and its B fragment reads exactly
//     those x_q bytes.
//   - x_q is staged once per CTA in shared memory (rows of round_up(K, 256)
//     bytes, 16-byte chunks XOR-swizzled so that the B loads are free of
//     bank conflicts).
//   - acc = (sum of 64 * W_q * x_q) >> 6 exactly; the split-K partials meet
//     in shared memory; the epilogue rescales and stores Y (and acc).
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_MAX_XQ_SMEM = 96 * 1024;

struct DecodeProblem {
    const uint8_t *packed;
    const float *gamma;
    const int8_t *xq;
    const float *s;
    float *Y;
    int32_t *acc;
    int N;
    int K;
    int g_log2;     // log2(G): warps per row tile
    int cta_begin;  // first CTA of this problem in the grouped grid
};

struct DecodeParams {
    DecodeProblem p[BL_MAX_GROUP];
    int count;
    int M;
};

__host__ __device__ inline int dec_row_stride(int K) { return (K + 255) & ~255; }

__device__ __forceinline__ int dec_swz_chunk(int L, int row) {
    int x = (((L >> 3) & 1) << 1) | (row & 1);
    return (L & ~7) | ((L ^ x) & 7);
}

__device__ __forceinline__ u32 dec_unpack(u32 w, int j) {
    // codes of k = 4j .. 4j+3 of this 16-weight word -> int8 lanes holding 64 * W_q
    return (w << (6 - 2 * j)) & 0xC0C0C0C0u;
}

__device__ __forceinline__ void mma_s8_16832(int (&c)[4], u32 a0, u32 a1, u32 a2, u32 a3, u32 b0, u32 b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT: 8-token column tiles (1: M <= 8, 2: M <= 16).
template <int NT>
__global__ void __launch_bounds__(DEC_THREADS) k_decode(const __grid_constant__ DecodeParams P) {
    extern __shared__ __align__(16) uint8_t s_xq[];
    __shared__ int s_red[DEC_WARPS][NT][4][32];

    const int b = blockIdx.x;
    int pi = 0;
    while (pi + 1 < P.count && P.p[pi + 1].cta_begin <= b) ++pi;
    const DecodeProblem &pr = P.p[pi];
    const int M = P.M, N = pr.N, K = pr.K;
    const int glog = pr.g_log2, G = 1 << glog;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_per_cta = DEC_WARPS >> glog;
    const int tile = (b - pr.cta_begin) * tiles_per_cta + (warp >> glog);
    const int kslot = warp & (G - 1);
    const int row0 = tile * 16;
    const int RS = dec_row_stride(K);
    const int Kw = K >> 2;         // packed bytes per row
    const int nchunk64 = K >> 6;   // 64-k chunks (16 packed bytes each)
    const int steps = (K + 255) >> 8;

    // Stage x_q rows [0, M) into shared memory, swizzled, zero-padded to RS.
    {
        const int chunks = RS >> 4;
        for (int idx = threadIdx.x; idx < M * chunks; idx += DEC_THREADS) {
            int r = idx / chunks, L = idx - r * chunks;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (L * 16 < K) v = *reinterpret_cast<const uint4 *>(pr.xq + (size_t)r * K + L * 16);
            *reinterpret_cast<uint4 *>(s_xq + r * RS + dec_swz_chunk(L, r) * 16) = v;
        }
    }
    __syncthreads();

    const int g = lane >> 2, t = lane & 3;
    const bool rowA = row0 + g < N, rowB = row0 + g + 8 < N;
    const uint8_t *wA = pr.packed + (size_t)(row0 + g) * Kw;
    const uint8_t *wB = pr.packed + (size_t)(row0 + g + 8) * Kw;

    int acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0;

    // token rows of the B fragments this lane reads
    const int tr0 = g, tr1 = g + 8;
    const bool tv0 = tr0 < M, tv1 = NT > 1 && tr1 < M;

    for (int st = kslot; st < steps; st += 2 * G) {
        // two steps in flight: st and st + G
        uint4 a[2], bb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            int s2 = st + u * G;
            bool kv = s2 < steps && (s2 * 4 + t) < nchunk64;
            a[u] = (rowA && kv) ? ldg_stream_v4(wA + s2 * 64 + t * 16) : make_uint4(0, 0, 0, 0);
            bb[u] = (rowB && kv) ? ldg_stream_v4(wB + s2 * 64 + t * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            int s2 = st + u * G;
            if (s2 >= steps) break;
            const u32 wa[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
            const u32 wb[4] = {bb[u].x, bb[u].y, bb[u].z, bb[u].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int L = s2 * 16 + t * 4 + c;  // 16-byte chunk of x_q
                uint4 x0 = tv0 ? *reinterpret_cast<const uint4 *>(s_xq + tr0 * RS + dec_swz_chunk(L, tr0) * 16)
                               : make_uint4(0, 0, 0, 0);
                uint4 x1 = make_uint4(0, 0, 0, 0);
                if (NT > 1 && tv1) x1 = *reinterpret_cast<const uint4 *>(s_xq + tr1 * RS + dec_swz_chunk(L, tr1) * 16);
                const u32 xb0[4] = {x0.x, x0.y, x0.z, x0.w};
                const u32 xb1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    u32 a0 = dec_unpack(wa[c], 2 * h), a2 = dec_unpack(wa[c], 2 * h + 1);
                    u32 a1 = dec_unpack(wb[c], 2 * h), a3 = dec_unpack(wb[c], 2 * h + 1);
                    mma_s8_16832(acc[0], a0, a1, a2, a3, xb0[2 * h], xb0[2 * h + 1]);
                    if (NT > 1) mma_s8_16832(acc[NT - 1], a0, a1, a2, a3, xb1[2 * h], xb1[2 * h + 1]);
                }
            }
        }
    }

    // split-K reduction through shared memory
    if (G > 1) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s_red[warp][nt][i][lane] = acc[nt][i];
        __syncthreads();
        if (kslot == 0) {
            for (int q = 1; q < G; ++q)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[nt][i] += s_red[warp + q][nt][i][lane];
        }
    }
    if (kslot != 0) return;

    const float gamma = *pr.gamma;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = nt * 8 + 2 * t + (i & 1);
            const int n = row0 + g + 8 * (i >> 1);
            if (m < M && n < N) {
                const int a = acc[nt][i] >> 6;  // exact: the sum is a multiple of 64
                const float f = __fdiv_rn(gamma, pr.s[m]);
                pr.Y[(size_t)m * N + n] = __fmul_rn(__int2float_rn(a), f);
                if (pr.acc) pr.acc[(size_t)m * N + n] = a;
            }
        }
    }
}

}  // namespace bl
