// Steps 3 + 4 for large M: the tcgen05 prefill engine (sm_100a).
//
// What it computes ("bitone" README, How 1.58-bit Works and Forward pass):
//   acc[m, n] = sum_k x_q[m, k] * W_q[n, k];  Y[m, n] = acc * (gamma / s[m])
//
// Two CTAs (a cluster pair on two SMs) compute one output tile of 256 tokens
// (m) x 256 weight rows (n) with tcgen05.mma.cta_group::2.kind::i8, M = 256,
// N = 256, K = 32 per instruction, issued by one thread of the pair's first
// CTA (the leader).  Each CTA holds its own half of both operands:
//   A = its 128 tokens of x_q, by TMA with 128-byte swizzle, K-major;
//   B = 64 * W_q of its 128 of the 256 weight rows as int8: the packed 2-bit
//     rows arrive by TMA, four expander warps (one weight row per thread)
//     unpack them (((word << (6 - 2j)) & 0xC0C0C0C0) ^ 0x40404040 gives
//     four int8 lanes 64 * W_q from the codes 1 - W_q),
//     store them in the 128-byte-swizzled K-major layout the MMA reads, then
//     fence the async proxy;
//   D = int32 accumulators in each CTA's TMEM (lane = its token, column =
//     weight row of the full 256), two 256-column buffers so the epilogue of
//     one tile overlaps the MMAs of the next.
// The pair reads each B half once for both token halves, so every CTA
// expands, stores and feeds the tensor core half the weight bytes of a
// one-CTA 128 x 256 tile for the same number of MACs per SM: the shared
// memory traffic per MAC (TMA writes, expansion, operand reads), which bounds
// the one-CTA design, drops by about a third.
// Each epilogue thread owns one token (one float(gamma / s[m]) per tile); a
// warp converts a 32 x 32 block into a 128B-swizzled staging buffer and one
// lane writes it to Y with a TMA tensor store (tails clipped by the tensor
// map).  The exact sum is 64 * acc (|64 acc| <= 2^28, exact in int32 and in
// float), so Y = float(float(64 acc) * (f / 64)) with f = float(gamma / s[m])
// (f / 64 is exact) -- the same bits as float(acc) * f.
//
// Pipelines: PF_STAGES shared-memory stages carry x_q and packed tiles from
// TMA (per CTA, own barriers); PF_BSTAGES stages carry the expanded weights
// to the MMA: both CTAs' expanders arrive on the leader's "ready" barrier.
// MMA completion is committed to the barriers of both CTAs at once
// (tcgen05.commit multicast), which frees both kinds of stage and signals the
// epilogues; both CTAs' epilogues arrive on the leader's "accumulator empty"
// barrier.  The leader's "ready" arrival from the peer's expanders also
// implies that the peer's x_q stage has landed (they waited for it).
//
// Warp roles (persistent: one cluster pair per two SMs loops over tiles):
//   warp 0        TMA producer (one thread)
//   warp 1        TMEM allocator (both CTAs) + MMA issuer (leader, one thread)
//   warps 2..5    expanders: weight row 32*(w - 2) + lane of this CTA's half
//   warps 6..13   epilogue: TMEM lanes 32*(w % 4) .. +31 (tokens), columns
//                 128*((w - 6) / 4) .. +127 (weight rows)
// Every mbarrier wait is bounded (globaltimer); a wait that gives up raises
// the device error word, sets the CTA's abort flag and the CTA drains its
// in-flight copies and MMAs (again with bounded waits) before the pair meets
// at a cluster barrier, frees TMEM and exits.  No wait is unbounded and
// nothing traps.  No copy uses cluster multicast.
#pragma once

#include <cuda.h>

#include "bl_common.cuh"

namespace bl {

constexpr int PF_BM = 128;          // tokens per CTA (MMA M = 2 x 128, TMEM lanes)
constexpr int PF_BN = 256;          // weight rows per pair tile (MMA N, TMEM columns)
constexpr int PF_BNH = PF_BN / 2;   // weight rows expanded per CTA
constexpr int PF_BK = 128;          // k per pipeline stage (4 MMAs of K = 32)
constexpr int PF_STAGES = 8;        // TMA stages (x_q + packed)
constexpr int PF_BSTAGES = 2;       // expanded-weight stages (8 + 2 measured best of 5+5, 6+4, 7+3, 8+2)
constexpr int PF_EXP_WARPS = PF_BNH / 32;
constexpr int PF_EPI_WARPS = 8;
constexpr int PF_EPI_WARP0 = 2 + PF_EXP_WARPS;
constexpr int PF_THREADS = 32 * (PF_EPI_WARP0 + PF_EPI_WARPS);
constexpr int PF_A_BYTES = PF_BM * PF_BK;          // x_q stage: 16 KiB
constexpr int PF_P_BYTES = PF_BNH * PF_BK / 4;     // packed stage: 4 KiB
constexpr int PF_B_BYTES = PF_BNH * PF_BK;         // expanded stage: 16 KiB
constexpr int PF_TMEM_COLS = 512;                  // 2 x 256 accumulator columns
constexpr int PF_Y_BYTES = 32 * 32 * 4;            // per-epilogue-warp Y staging block (TMA store)

// shared memory carve-up (offsets from a 1024-byte aligned base; identical in
// both CTAs of a pair, which the pair MMA relies on)
constexpr int PF_OFF_A = 0;
constexpr int PF_OFF_B = PF_OFF_A + PF_STAGES * PF_A_BYTES;
constexpr int PF_OFF_P = PF_OFF_B + PF_BSTAGES * PF_B_BYTES;
constexpr int PF_OFF_Y = PF_OFF_P + PF_STAGES * PF_P_BYTES;             // [8 warps][32 x 32] float, 128B-swizzled
constexpr int PF_OFF_BAR = PF_OFF_Y + PF_EPI_WARPS * PF_Y_BYTES;
constexpr int PF_NBAR = 2 * PF_STAGES + 2 * PF_BSTAGES + 4;  // full, empty, bready, bempty, accfull x2, accempty x2
constexpr int PF_OFF_MISC = PF_OFF_BAR + PF_NBAR * 8;
constexpr int PF_SMEM_USED = PF_OFF_MISC + 16;
constexpr int PF_SMEM_BYTES = PF_SMEM_USED + 1024;                     // + alignment slack
static_assert(PF_SMEM_BYTES > 116 * 1024, "keeps one CTA per SM, so the TMEM allocation never waits");
static_assert(PF_SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(PF_OFF_B % 1024 == 0 && PF_OFF_Y % 1024 == 0 && PF_A_BYTES % 1024 == 0 && PF_B_BYTES % 1024 == 0,
              "128-byte swizzled stages start on 1024-byte boundaries");

// Up to PF_MAX_PROB weight matrices that share one activation (e.g. the q,
// k, v or the gate, up projections of a layer) in one launch: their output
// tiles are numbered consecutively along N (problem p owns global n-tiles
// nt_begin .. nt_begin + ceil(N / PF_BN) - 1).
constexpr int PF_MAX_PROB = BL_MAX_PREFILL_GROUP;

struct PrefillProb {
    const float *gamma;
    float *Y;
    int32_t *acc;
    int N;
    int nt_begin;
};

// TMA descriptors: the shared x_q and, per problem, packed weights and Y.
struct PrefillMaps {
    CUtensorMap x;
    CUtensorMap w[PF_MAX_PROB];
    CUtensorMap y[PF_MAX_PROB];
};

struct PrefillParams {
    PrefillProb prob[PF_MAX_PROB];
    int nprob;
    const float *s;
    int M, K;
    int n_tiles, m_tiles, k_stages;  // n_tiles: over all problems; m_tiles: 256-token pair tiles
    unsigned long long timeout_ns;
    long long dbg_skip_iter;  // >= 0: the producers never issue this k-iteration (bounded-wait test)
    int y_tma;                // 1: Y written by TMA stores (every N % 4 == 0 and no acc output)
    int glu;                  // 1: gated FFN tiles (below): problem 0 = gate, 1 = up, output h
};

// ---------------------------------------------------------------------------
// PTX wrappers

__device__ __forceinline__ void tma_load_2d(u32 dst, const CUtensorMap *map, int x, int y, u32 bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Y block store: shared (128B-swizzled 32 x 32 floats) -> global through the
// tensor map; out-of-range rows / columns of the box are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, u32 src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(map), "r"(x), "r"(y), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ u32 cluster_ctarank() {
    u32 r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ u32 cluster_idx() {
    u32 r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ u32 cluster_count() {
    u32 r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// every thread of both CTAs; orders the barrier initialisation (release) before
// any arrival from the peer, and at the end keeps a CTA resident while its peer
// may still touch its shared memory
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// arrive on the barrier at the same shared-memory offset in CTA `rank` of the
// cluster (this CTA included).  Default (CTA-scope release) semantics: what the
// arrival publishes is shared memory for the tensor core, ordered by the
// async-proxy fence before it, or TMEM reads ordered by tcgen05.fence; a
// cluster-scope release here (a fence per expander warp per k block) measured
// 40 % slower.
__device__ __forceinline__ void mbar_arrive_cluster(u32 bar, u32 rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.shared::cluster.b64 _, [ra];\n\t}"
        ::"r"(bar), "r"(rank)
        : "memory");
}

// D[tmem of both CTAs] (+)= A[smem desc, each CTA's half] * B[smem desc, each
// CTA's half of N], kind::i8, cta_group::2
__device__ __forceinline__ void tc2_mma_i8_ss(u32 d_tmem, unsigned long long a_desc, unsigned long long b_desc,
                                              u32 idesc, u32 accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Same with bf16 operands and f32 accumulation (kind::f16): the backward
// product dX = dY (gamma W_q).
__device__ __forceinline__ void tc2_mma_f16_ss(u32 d_tmem, unsigned long long a_desc, unsigned long long b_desc,
                                               u32 idesc, u32 accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive (once the MMAs issued so far complete) on the barrier at this
// shared-memory offset in both CTAs of the pair
__device__ __forceinline__ void tc2_commit_pair(u32 bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(bar), "h"((unsigned short)3)
        : "memory");
}

__device__ __forceinline__ void tc_ld_32x32b_x32(u32 taddr, u32 (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), version 1 (sm_100), base offset 0 (stage bases are
// 1024-byte aligned).
__device__ __forceinline__ unsigned long long smem_desc_k_sw128(u32 saddr) {
    unsigned long long d = 0;
    d |= (unsigned long long)((saddr >> 4) & 0x3FFFu);
    d |= (unsigned long long)1u << 16;            // leading byte offset (unused for swizzled K-major) = 16 B
    d |= (unsigned long long)(1024u >> 4) << 32;  // stride byte offset
    d |= (unsigned long long)1u << 46;            // descriptor version
    d |= (unsigned long long)2u << 61;            // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::i8: D s32, A s8, B s8, both K-major,
// N = PF_BN, M = 2 x PF_BM (the pair).  BWD (kind::f16): D f32, A bf16,
// B bf16, same shape.
template <bool BWD>
__host__ __device__ constexpr u32 pf_idesc() {
    return (BWD ? (1u << 4) : (2u << 4))      // D format: f32 / s32
           | (1u << 7)                        // A format: bf16 / signed 8-bit
           | (1u << 10)                       // B format: bf16 / signed 8-bit
           | ((u32)(PF_BN >> 3) << 17)        // N >> 3
           | ((u32)((2 * PF_BM) >> 4) << 24); // M >> 4
}

// Backward mode: a pipeline stage covers 64 of the reduction index n (bf16:
// the same 128 bytes per operand row as 128 int8); its packed stage holds
// 64 rows n x 128 k of the forward's packed matrix (32 bytes per row).
constexpr int PF_BWD_BK = 64;
constexpr int PF_BWD_P_BYTES = PF_BWD_BK * PF_BNH / 4;  // 2 KiB

// ---------------------------------------------------------------------------

// problem that owns global n-tile nt
__device__ __forceinline__ int pf_prob_of(const PrefillParams &p, int nt) {
    int pi = 0;
    while (pi + 1 < p.nprob && nt >= p.prob[pi + 1].nt_begin) ++pi;
    return pi;
}

// BWD = false: the forward (int8 x_q against expanded 64 * W_q, acc int32).
// BWD = true: the backward product dX = dY (gamma W_q): A = dY bf16 [M, N]
// (the reduction index n contiguous), B = W_q^T as bf16 +-1 / 0, expanded
// from the forward's packed rows (each B row is an input feature k, read
// across 64 packed rows n per stage), f32 accumulators; epilogue dX =
// float(acc * gamma).  Everything else (pairs, pipelines, TMEM, waits) is
// shared.
template <bool BWD>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PF_THREADS, 1)
    k_prefill_tc(const __grid_constant__ PrefillMaps maps, const __grid_constant__ PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const u32 sbase = smem_u32(sm);
    const u32 bar0 = sbase + PF_OFF_BAR;
    auto BAR_FULL = [&](int s) { return bar0 + 8u * s; };
    auto BAR_EMPTY = [&](int s) { return bar0 + 8u * (PF_STAGES + s); };
    auto BAR_BREADY = [&](int a) { return bar0 + 8u * (2 * PF_STAGES + a); };
    auto BAR_BEMPTY = [&](int a) { return bar0 + 8u * (2 * PF_STAGES + PF_BSTAGES + a); };
    auto BAR_ACCFULL = [&](int b) { return bar0 + 8u * (2 * PF_STAGES + 2 * PF_BSTAGES + b); };
    auto BAR_ACCEMPTY = [&](int b) { return bar0 + 8u * (2 * PF_STAGES + 2 * PF_BSTAGES + 2 + b); };
    u32 *s_tmem = reinterpret_cast<u32 *>(sm + PF_OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + PF_OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const u32 rank = cluster_ctarank();  // 0: the leader, which issues the pair's MMAs
    if (threadIdx.x == 0) {
        for (int s = 0; s < PF_STAGES; ++s) {
            mbar_init(BAR_FULL(s), 1);
            mbar_init(BAR_EMPTY(s), 1);
        }
        for (int a = 0; a < PF_BSTAGES; ++a) {
            mbar_init(BAR_BREADY(a), 2 * PF_EXP_WARPS);  // used in the leader: both CTAs' expanders
            mbar_init(BAR_BEMPTY(a), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR_ACCFULL(b), 1);
            mbar_init(BAR_ACCEMPTY(b), 2 * PF_EPI_WARPS);  // used in the leader: both CTAs' epilogues
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.x) : "memory");
        for (int i = 0; i < p.nprob; ++i) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.w[i]) : "memory");
            if (p.y_tma) asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.y[i]) : "memory");
        }
    }
    if (warp == 1) {
        // both CTAs, same warp: the pair's columns are allocated in both TMEMs
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(PF_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const u32 tmem = *s_tmem;

    const int total_tiles = p.n_tiles * p.m_tiles;
    const int KS = p.k_stages;
    const unsigned long long TO = p.timeout_ns;
    const int cid = (int)cluster_idx(), ncl = (int)cluster_count();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // x_q and the packed weights may come from the kernel before this
            // one (programmatic dependent launch; a no-op otherwise)
            asm volatile("griddepcontrol.wait;" ::: "memory");
            long long it = 0;
            bool failed = false;
            for (int tile = cid; tile < total_tiles && !failed; tile += ncl) {
                const int nt = tile % p.n_tiles, mt = tile / p.n_tiles;
                // gated tiles: the leader's half of B is 128 gate rows, the
                // peer's the same 128 rows of up
                const int pi = (!BWD && p.glu) ? (int)rank : pf_prob_of(p, nt);
                const CUtensorMap *tmw = &maps.w[pi];
                const int ntl = (!BWD && p.glu) ? nt : nt - p.prob[pi].nt_begin;
                const int arow = mt * (2 * PF_BM) + (int)rank * PF_BM;   // this CTA's tokens
                const int brow = (!BWD && p.glu) ? ntl * PF_BNH : ntl * PF_BN + (int)rank * PF_BNH;  // this CTA's B rows
                for (int ks = 0; ks < KS; ++ks, ++it) {
                    const int s = (int)(it % PF_STAGES);
                    const u32 ph = (u32)((it / PF_STAGES) & 1);
                    if (!mbar_wait(BAR_EMPTY(s), ph ^ 1u, TO, s_abort)) {
                        failed = true;
                        break;
                    }
                    if (it == p.dbg_skip_iter) continue;  // test hook: this stage never arrives
                    if (BWD) {
                        // dY columns n = 64 ks ..; packed rows n = 64 ks .., bytes of k = brow .. brow + 127
                        mbar_arrive_expect_tx(BAR_FULL(s), PF_A_BYTES + PF_BWD_P_BYTES);
                        tma_load_2d(sbase + PF_OFF_A + s * PF_A_BYTES, &maps.x, ks * PF_BWD_BK, arow, BAR_FULL(s));
                        tma_load_2d(sbase + PF_OFF_P + s * PF_P_BYTES, tmw, brow / 4, ks * PF_BWD_BK, BAR_FULL(s));
                    } else {
                        mbar_arrive_expect_tx(BAR_FULL(s), PF_A_BYTES + PF_P_BYTES);
                        tma_load_2d(sbase + PF_OFF_A + s * PF_A_BYTES, &maps.x, ks * PF_BK, arow, BAR_FULL(s));
                        tma_load_2d(sbase + PF_OFF_P + s * PF_P_BYTES, tmw, ks * (PF_BK / 4), brow, BAR_FULL(s));
                    }
                }
            }
            if (failed) {
                raise_device_error(DEVERR_TIMEOUT_PRODUCER);
                *s_abort = 1;
            }
            // drain: the last PF_STAGES issued loads must have landed before exit
            // (time-bounded only; the abort flag does not cut this wait short)
            for (long long j = it - PF_STAGES; j < it; ++j) {
                if (j < 0 || j == p.dbg_skip_iter) continue;
                mbar_wait(BAR_FULL((int)(j % PF_STAGES)), (u32)((j / PF_STAGES) & 1), TO, nullptr);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0 && rank == 0) {
            const u32 idesc = pf_idesc<BWD>();
            long long it = 0;
            int tc = 0;
            bool failed = false, issued = false;
            u32 last_bar = 0, last_ph = 0;
            for (int tile = cid; tile < total_tiles && !failed; tile += ncl, ++tc) {
                const int b = tc & 1;
                const u32 cph = (u32)((tc >> 1) & 1);
                // both CTAs' epilogues have drained this accumulator buffer
                if (!mbar_wait(BAR_ACCEMPTY(b), cph ^ 1u, TO, s_abort)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const u32 d_tmem = tmem + b * PF_BN;
                for (int ks = 0; ks < KS; ++ks, ++it) {
                    const int s = (int)(it % PF_STAGES);
                    const u32 ph = (u32)((it / PF_STAGES) & 1);
                    const int a = (int)(it % PF_BSTAGES);
                    const u32 aph = (u32)((it / PF_BSTAGES) & 1);
                    // own x_q stage landed; both CTAs' expanded halves ready
                    // (the peer's expanders waited for the peer's x_q stage)
                    if (!mbar_wait(BAR_FULL(s), ph, TO, s_abort) ||
                        !mbar_wait(BAR_BREADY(a), aph, TO, s_abort)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    const u32 astage = sbase + PF_OFF_A + s * PF_A_BYTES;
                    const u32 bstage = sbase + PF_OFF_B + a * PF_B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < PF_BK / 32; ++kk) {
                        if (BWD)
                            tc2_mma_f16_ss(d_tmem, smem_desc_k_sw128(astage + kk * 32),
                                           smem_desc_k_sw128(bstage + kk * 32), idesc, (ks | kk) != 0 ? 1u : 0u);
                        else
                            tc2_mma_i8_ss(d_tmem, smem_desc_k_sw128(astage + kk * 32),
                                          smem_desc_k_sw128(bstage + kk * 32), idesc, (ks | kk) != 0 ? 1u : 0u);
                    }
                    tc2_commit_pair(BAR_EMPTY(s));
                    tc2_commit_pair(BAR_BEMPTY(a));
                    issued = true;
                    last_bar = BAR_EMPTY(s);
                    last_ph = ph;
                }
                if (failed) break;
                tc2_commit_pair(BAR_ACCFULL(b));
            }
            if (failed) {
                raise_device_error(DEVERR_TIMEOUT_MMA);
                *s_abort = 1;
                // drain: every MMA issued so far completes before TMEM is freed
                if (issued) mbar_wait(last_bar, last_ph, TO, nullptr);
            }
        }
    } else if (warp < PF_EPI_WARP0) {
        // ------------------------------------------------------------ expanders
        const int row = (warp - 2) * 32 + lane;  // weight row within this CTA's half
        const int rsw = row & 7;                 // 128-byte swizzle phase of this row
        long long it = 0;
        bool failed = false;
        for (int tile = cid; tile < total_tiles && !failed; tile += ncl) {
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int s = (int)(it % PF_STAGES);
                const u32 ph = (u32)((it / PF_STAGES) & 1);
                const int a = (int)(it % PF_BSTAGES);
                const u32 aph = (u32)((it / PF_BSTAGES) & 1);
                // the packed stage has landed and the MMAs that read this B stage before are done
                bool ok = mbar_wait(BAR_FULL(s), ph, TO, s_abort) && mbar_wait(BAR_BEMPTY(a), aph ^ 1u, TO, s_abort);
                if (!__all_sync(0xffffffffu, ok)) {
                    failed = true;
                    break;
                }
                uint8_t *brow = sm + PF_OFF_B + a * PF_B_BYTES + row * 128;
                if (BWD) {
                    // B row = input feature k (this thread's `row` of the tile's
                    // 128): the codes of (n, k) for the stage's 64 n, from word
                    // k / 16 of each packed row n (32 bytes per row in the
                    // stage; the warp's 32 rows share two words: broadcasts),
                    // as bf16 0 / +1 / -1, 8 n per 16-byte chunk
                    const u32 *pw = reinterpret_cast<const u32 *>(sm + PF_OFF_P + s * PF_P_BYTES) + (row >> 4);
                    const int sh = 8 * (row & 3) + 2 * ((row >> 2) & 3);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        u32 o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const u32 c0 = (pw[8 * (8 * c + 2 * e)] >> sh) & 3u;
                            const u32 c1 = (pw[8 * (8 * c + 2 * e + 1)] >> sh) & 3u;
                            // code 1 - W_q -> bf16: 00 -> +1 (0x3F80), 01 -> 0, 10 -> -1 (0xBF80)
                            const u32 b0 = ((c0 & 1u) ^ 1u) * 0x3F80u | ((c0 & 2u) << 14);
                            const u32 b1 = ((c1 & 1u) ^ 1u) * 0x3F80u | ((c1 & 2u) << 14);
                            o[e] = b0 | (b1 << 16);
                        }
                        *reinterpret_cast<uint4 *>(brow + ((c ^ rsw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(BAR_BREADY(a), 0);
                    continue;
                }
                const uint4 *src = reinterpret_cast<const uint4 *>(sm + PF_OFF_P + s * PF_P_BYTES + row * (PF_BK / 4));
                const uint4 v0 = src[0], v1 = src[1];
                const u32 w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // packed word i = k 16i .. 16i+15 = 16-byte chunk i of the row.
                    // Code c = 1 - W_q moved to the top two bits of a byte, its
                    // low bit flipped, is W_q in two's complement there, i.e.
                    // the int8 64 * W_q (one AND and XOR, one LOP3, per four)
                    uint4 o;
                    o.x = ((w[i] << 6) & 0xC0C0C0C0u) ^ 0x40404040u;
                    o.y = ((w[i] << 4) & 0xC0C0C0C0u) ^ 0x40404040u;
                    o.z = ((w[i] << 2) & 0xC0C0C0C0u) ^ 0x40404040u;
                    o.w = (w[i] & 0xC0C0C0C0u) ^ 0x40404040u;
                    *reinterpret_cast<uint4 *>(brow + ((i ^ rsw) << 4)) = o;
                }
                // make the generic-proxy stores visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(BAR_BREADY(a), 0);
            }
        }
        if (failed && lane == 0) {
            raise_device_error(DEVERR_TIMEOUT_EXPAND);
            *s_abort = 1;
        }
    } else {
        // ------------------------------------------------------------- epilogue
        asm volatile("griddepcontrol.wait;" ::: "memory");  // s and gamma, as above
        const int q = warp & 3;                           // TMEM lane quarter = token block
        const int ew = warp - PF_EPI_WARP0;               // 0..7
        const int half = ew >> 2;                         // weight-row half of the tile

        uint8_t *ystage = sm + PF_OFF_Y + ew * PF_Y_BYTES;
        const u32 ystage_s = smem_u32(ystage);
        int tc = 0;
        bool failed = false;
        for (int tile = cid; tile < total_tiles && !failed; tile += ncl, ++tc) {
            const int nt = tile % p.n_tiles, mt = tile / p.n_tiles;
            if (!BWD && p.glu) {
                // Gated FFN tile: TMEM columns 0..127 hold gate, 128..255 up,
                // for the same 128 rows (n).  Each thread owns one token:
                //   h = float(float(r * r) * u), r = max(g, 0), with
                //   g = float(float(acc_g) * float(gamma_g / s)), u likewise,
                // the bits the plain epilogue would store for gate and up.
                // This warp writes h columns 64 * half .. + 63 of the tile.
                const int b = tc & 1;
                const u32 cph = (u32)((tc >> 1) & 1);
                const int mrow0 = mt * (2 * PF_BM) + (int)rank * PF_BM + q * 32;
                const int m = mrow0 + lane;
                const float sm_ = m < p.M ? p.s[m] : 1.f;
                const float fg = __fmul_rn(__fdiv_rn(*p.prob[0].gamma, sm_), 0.015625f);
                const float fu = __fmul_rn(__fdiv_rn(*p.prob[1].gamma, sm_), 0.015625f);
                bool ok = mbar_wait(BAR_ACCFULL(b), cph, TO, s_abort);
                if (!__all_sync(0xffffffffu, ok)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const int n0 = nt * PF_BNH + half * (PF_BNH / 2);
#pragma unroll 1
                for (int c0 = 0; c0 < PF_BNH / 2; c0 += 32) {
                    u32 rg[32], ru[32];
                    const u32 ta = tmem + ((u32)(q * 32) << 16) + b * PF_BN + half * (PF_BNH / 2) + c0;
                    tc_ld_32x32b_x32(ta, rg);
                    tc_ld_32x32b_x32(ta + PF_BNH, ru);
                    tc_wait_ld();
                    if (c0 + 32 == PF_BNH / 2) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(BAR_ACCEMPTY(b), 0);
                    }
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float hv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float g = __fmul_rn(__int2float_rn((int)rg[4 * c + e]), fg);
                            const float u = __fmul_rn(__int2float_rn((int)ru[4 * c + e]), fu);
                            const float r = g > 0.f ? g : 0.f;
                            hv[e] = __fmul_rn(__fmul_rn(r, r), u);
                        }
                        *reinterpret_cast<float4 *>(ystage + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_float4(hv[0], hv[1], hv[2], hv[3]);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&maps.y[0], n0 + c0, mrow0, ystage_s);
                    __syncwarp();
                }
                continue;
            }
            const PrefillProb &pp = p.prob[pf_prob_of(p, nt)];
            const int pN = pp.N;
            const int ntl = nt - pp.nt_begin;
            const float gamma = *pp.gamma;
            const bool vec_ok = (pN & 3) == 0;            // rows of Y 16-byte aligned
            const int b = tc & 1;
            const u32 cph = (u32)((tc >> 1) & 1);
            const int mrow0 = mt * (2 * PF_BM) + (int)rank * PF_BM + q * 32;  // this warp's first token
            const int m = mrow0 + lane;                   // this thread's token
            const bool mvalid = m < p.M;
            // forward: float(gamma / s[m]) / 64 (exact); backward: gamma
            const float f = BWD ? gamma : (mvalid ? __fmul_rn(__fdiv_rn(gamma, p.s[m]), 0.015625f) : 0.f);
            auto cvt = [&](u32 v) {
                return BWD ? __fmul_rn(__uint_as_float(v), f) : __fmul_rn(__int2float_rn((int)v), f);
            };
            bool ok = mbar_wait(BAR_ACCFULL(b), cph, TO, s_abort);
            if (!__all_sync(0xffffffffu, ok)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const int n0 = ntl * PF_BN + half * (PF_BN / 2);  // within this problem
            const bool full = vec_ok && n0 + PF_BN / 2 <= pN;
            float *yrow = pp.Y + (size_t)m * pN + n0;
            int32_t *arow = pp.acc ? pp.acc + (size_t)m * pN + n0 : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < PF_BN / 2; c0 += 32) {
                u32 r[32];
                tc_ld_32x32b_x32(tmem + ((u32)(q * 32) << 16) + b * PF_BN + half * (PF_BN / 2) + c0, r);
                tc_wait_ld();
                if (c0 + 32 == PF_BN / 2) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(BAR_ACCEMPTY(b), 0);
                }
                if (p.y_tma) {
                    // the previous TMA store from this block has finished reading it
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float4 o;
                        o.x = cvt(r[4 * c + 0]);
                        o.y = cvt(r[4 * c + 1]);
                        o.z = cvt(r[4 * c + 2]);
                        o.w = cvt(r[4 * c + 3]);
                        *reinterpret_cast<float4 *>(ystage + lane * 128 + ((c ^ (lane & 7)) << 4)) = o;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&maps.y[pf_prob_of(p, nt)], n0 + c0, mrow0, ystage_s);
                } else if (mvalid) {
                    if (full) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            float4 o;
                            o.x = cvt(r[j + 0]);
                            o.y = cvt(r[j + 1]);
                            o.z = cvt(r[j + 2]);
                            o.w = cvt(r[j + 3]);
                            *reinterpret_cast<float4 *>(yrow + c0 + j) = o;
                            if (arow) {
                                // exact: the sums are multiples of 64
                                *reinterpret_cast<int4 *>(arow + c0 + j) =
                                    make_int4((int)r[j] >> 6, (int)r[j + 1] >> 6, (int)r[j + 2] >> 6, (int)r[j + 3] >> 6);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (n0 + c0 + j < pN) {
                                yrow[c0 + j] = cvt(r[j]);
                                if (arow) arow[c0 + j] = (int)r[j] >> 6;
                            }
                        }
                    }
                }
                __syncwarp();  // converged before the next tcgen05.ld
            }
        }
        // every TMA store of this warp has completed before the CTA exits
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
        if (failed && lane == 0) {
            raise_device_error(DEVERR_TIMEOUT_EPILOGUE);
            *s_abort = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA leaves (or frees TMEM) while its peer may still arrive on its
    // barriers, read its shared memory through the pair MMA or write its TMEM
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(PF_TMEM_COLS)
                     : "memory");
    }
}

}  // namespace bl

// ===========================================================================
// Host side: tensor maps and launch.

#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

namespace bl {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

inline cudaError_t prefill_setup() {
    if (encode_tiled_fn() == nullptr) return cudaErrorNotSupported;
    if (cudaFuncSetAttribute(k_prefill_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM_BYTES) !=
        cudaSuccess)
        return cudaErrorUnknown;
    return cudaFuncSetAttribute(k_prefill_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM_BYTES);
}

// Cluster pairs that can be resident at once on the current device (the
// persistent grid never exceeds it, so every pair runs in the first wave).
inline int prefill_max_pairs(int sms) {
    static std::atomic<int> cache[64];  // per device; 0 = not queried yet (a race only repeats the query)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sms / 2;
    const int known = cache[dev].load(std::memory_order_relaxed);
    if (known > 0) return known;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * (sms / 2)));
    cfg.blockDim = dim3(PF_THREADS);
    cfg.dynamicSmemBytes = PF_SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_prefill_tc<false>, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = sms / 2;
    }
    if (n > sms / 2) n = sms / 2;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

constexpr unsigned long long PF_DEFAULT_TIMEOUT_NS = 2000000000ull;  // 2 s per wait

// One weight matrix of a grouped prefill launch (all share x_q, s, M, K).
struct PrefillJob {
    const uint8_t *packed;
    const float *gamma;
    float *Y;
    int32_t *acc_out;
    int64_t N;
};

// pdl: launch as a programmatic dependent of the kernel before it (its
// set-up -- barriers, TMEM, descriptor prefetch -- overlaps that kernel's
// tail; the producer and the epilogue wait for it before touching inputs).
inline bl_status prefill_launch_group(int sms, const PrefillJob *jobs, int count, const int8_t *x_q, const float *s,
                                      int64_t M, int64_t K, cudaStream_t st,
                                      unsigned long long timeout_ns = PF_DEFAULT_TIMEOUT_NS,
                                      long long dbg_skip_iter = -1, bool pdl = false) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return BL_ERR_CUDA;
    if (count < 1 || count > PF_MAX_PROB) return BL_ERR_SHAPE;
    PrefillMaps maps;
    memset(&maps, 0, sizeof(maps));
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {(cuuint32_t)PF_BK, (cuuint32_t)PF_BM};
        if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(x_q), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    // Y through TMA stores when every Y row is a 16-byte multiple and no acc output is requested
    int y_tma = 1;
    for (int i = 0; i < count; ++i) y_tma &= (jobs[i].N % 4 == 0 && jobs[i].acc_out == nullptr) ? 1 : 0;
    int64_t n_tiles = 0;
    for (int i = 0; i < count; ++i) {
        const PrefillJob &j = jobs[i];
        {
            const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)j.N};
            const cuuint64_t gstride[1] = {(cuuint64_t)(K / 4)};
            const cuuint32_t box[2] = {(cuuint32_t)(PF_BK / 4), (cuuint32_t)PF_BNH};  // one CTA's half of a tile
            if (enc(&maps.w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(j.packed), gdim, gstride, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return BL_ERR_CUDA;
        }
        if (y_tma) {
            const cuuint64_t gdim[2] = {(cuuint64_t)j.N, (cuuint64_t)M};
            const cuuint64_t gstride[1] = {(cuuint64_t)j.N * 4};
            const cuuint32_t box[2] = {32, 32};
            if (enc(&maps.y[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, j.Y, gdim, gstride, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return BL_ERR_CUDA;
        }
        p.prob[i] = PrefillProb{j.gamma, j.Y, j.acc_out, (int)j.N, (int)n_tiles};
        n_tiles += (j.N + PF_BN - 1) / PF_BN;
    }
    const int64_t m_tiles = (M + 2 * PF_BM - 1) / (2 * PF_BM);  // 256-token pair tiles
    if (n_tiles * m_tiles > 0x7fffffffLL) return BL_ERR_SHAPE;
    p.nprob = count;
    p.y_tma = y_tma;
    p.s = s;
    p.M = (int)M;
    p.K = (int)K;
    p.n_tiles = (int)n_tiles;
    p.m_tiles = (int)m_tiles;
    p.k_stages = (int)((K + PF_BK - 1) / PF_BK);
    p.timeout_ns = timeout_ns;
    p.dbg_skip_iter = dbg_skip_iter;
    const int64_t tiles = n_tiles * m_tiles;
    const int pairs = prefill_max_pairs(sms);
    const unsigned grid = 2u * (unsigned)(tiles < pairs ? tiles : pairs);  // cluster pairs (__cluster_dims__)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(PF_THREADS);
    cfg.dynamicSmemBytes = PF_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_prefill_tc<false>, maps, p) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

// Gated FFN: h [M, F] = relu(Y_gate)^2 * Y_up from one launch whose pair
// tiles hold 128 gate and the same 128 up rows (F % 64 == 0: every h row is
// a multiple of 16 bytes, stored by TMA).
inline bl_status prefill_launch_glu(int sms, const uint8_t *packed_gate, const float *gamma_gate,
                                    const uint8_t *packed_up, const float *gamma_up, const int8_t *x_q,
                                    const float *s, int64_t M, int64_t F, int64_t K, float *h, cudaStream_t st,
                                    bool pdl = false) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return BL_ERR_CUDA;
    PrefillMaps maps;
    memset(&maps, 0, sizeof(maps));
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {(cuuint32_t)PF_BK, (cuuint32_t)PF_BM};
        if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(x_q), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    const uint8_t *pk[2] = {packed_gate, packed_up};
    for (int i = 0; i < 2; ++i) {
        const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)F};
        const cuuint64_t gstride[1] = {(cuuint64_t)(K / 4)};
        const cuuint32_t box[2] = {(cuuint32_t)(PF_BK / 4), (cuuint32_t)PF_BNH};
        if (enc(&maps.w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(pk[i]), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)F, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)F * 4};
        const cuuint32_t box[2] = {32, 32};
        if (enc(&maps.y[0], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, h, gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
            CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    p.prob[0] = PrefillProb{gamma_gate, h, nullptr, (int)F, 0};
    p.prob[1] = PrefillProb{gamma_up, h, nullptr, (int)F, 0};
    p.nprob = 2;
    p.glu = 1;
    p.y_tma = 1;
    p.s = s;
    p.M = (int)M;
    p.K = (int)K;
    const int64_t n_tiles = (F + PF_BNH - 1) / PF_BNH;
    const int64_t m_tiles = (M + 2 * PF_BM - 1) / (2 * PF_BM);
    if (n_tiles * m_tiles > 0x7fffffffLL) return BL_ERR_SHAPE;
    p.n_tiles = (int)n_tiles;
    p.m_tiles = (int)m_tiles;
    p.k_stages = (int)((K + PF_BK - 1) / PF_BK);
    p.timeout_ns = PF_DEFAULT_TIMEOUT_NS;
    p.dbg_skip_iter = -1;
    const int64_t tiles = n_tiles * m_tiles;
    const int pairs = prefill_max_pairs(sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * (unsigned)(tiles < pairs ? tiles : pairs));
    cfg.blockDim = dim3(PF_THREADS);
    cfg.dynamicSmemBytes = PF_SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_prefill_tc<false>, maps, p) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

// Backward dX [M, K] = dY [M, N] (gamma W_q) on the tensor cores: bf16 dY,
// the forward's packed W [N, K/4], f32 accumulation (N % 8 == 0: the dY
// rows are multiples of 16 bytes for TMA).
inline bl_status prefill_launch_bwd(int sms, const void *dY, const uint8_t *packed, const float *gamma, int64_t M,
                                    int64_t N, int64_t K, float *dX, cudaStream_t st) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return BL_ERR_CUDA;
    PrefillMaps maps;
    memset(&maps, 0, sizeof(maps));
    PrefillParams p;
    memset(&p, 0, sizeof(p));
    const cuuint32_t es[2] = {1, 1};
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)N, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)N * 2};
        const cuuint32_t box[2] = {(cuuint32_t)PF_BWD_BK, (cuuint32_t)PF_BM};
        if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(dY), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)(K / 4)};
        const cuuint32_t box[2] = {(cuuint32_t)(PF_BNH / 4), (cuuint32_t)PF_BWD_BK};  // 128 k x 64 n
        if (enc(&maps.w[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(packed), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)K * 4};
        const cuuint32_t box[2] = {32, 32};
        if (enc(&maps.y[0], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dX, gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return BL_ERR_CUDA;
    }
    p.prob[0] = PrefillProb{gamma, dX, nullptr, (int)K, 0};
    p.nprob = 1;
    p.y_tma = 1;
    p.M = (int)M;
    p.K = (int)N;
    const int64_t n_tiles = (K + PF_BN - 1) / PF_BN;
    const int64_t m_tiles = (M + 2 * PF_BM - 1) / (2 * PF_BM);
    if (n_tiles * m_tiles > 0x7fffffffLL) return BL_ERR_SHAPE;
    p.n_tiles = (int)n_tiles;
    p.m_tiles = (int)m_tiles;
    p.k_stages = (int)((N + PF_BWD_BK - 1) / PF_BWD_BK);
    p.timeout_ns = PF_DEFAULT_TIMEOUT_NS;
    p.dbg_skip_iter = -1;
    const int64_t tiles = n_tiles * m_tiles;
    const int pairs = prefill_max_pairs(sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * (unsigned)(tiles < pairs ? tiles : pairs));
    cfg.blockDim = dim3(PF_THREADS);
    cfg.dynamicSmemBytes = PF_SMEM_BYTES;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, k_prefill_tc<true>, maps, p) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

inline bl_status prefill_launch(int sms, const uint8_t *packed, const float *gamma, const int8_t *x_q, const float *s,
                                int64_t M, int64_t N, int64_t K, float *Y, int32_t *acc_out, cudaStream_t st,
                                unsigned long long timeout_ns = PF_DEFAULT_TIMEOUT_NS, long long dbg_skip_iter = -1,
                                bool pdl = false) {
    const PrefillJob job{packed, gamma, Y, acc_out, N};
    return prefill_launch_group(sms, &job, 1, x_q, s, M, K, st, timeout_ns, dbg_skip_iter, pdl);
}

}  // namespace bl
