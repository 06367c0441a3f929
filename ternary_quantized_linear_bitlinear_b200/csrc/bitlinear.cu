// libbitlinear.so: the C ABI declared in include/bitlinear.h.
//
// Host side only validates, picks an engine and enqueues kernels on the
// caller's stream; it never allocates device memory and never synchronizes
// (except bl_check_device_error, which is documented to).
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "bitlinear.h"
#include "bitlinear_debug.h"
#include "bl_common.cuh"
#include "k_act_quant.cuh"
#include "k_decode.cuh"
#include "k_prefill_tc.cuh"
#include "k_dense_tc.cuh"
#include "k_weight_quant.cuh"

using namespace bl;

namespace {

constexpr int BL_VERSION = 100;
constexpr int64_t K_MAX = 32768;
constexpr int MAX_DEVICES = 64;
// dynamic shared memory a decode launch may use: the CTA's weights (whole
// groups, or a 32 x DEC_KCH_B chunk) plus padding, x_q and the sums; a
// problem whose whole group does not fit beside its x_q is chunked, and
// problems whose combined layout would not fit go to separate launches
constexpr size_t DEC_SMEM_ATTR = (size_t)DEC_ROWS * DEC_KCH_B + DEC_W_PAD + DEC_X_MAX + DEC_WARPS * DEC_ROWS * 16 * 4 + 512;
// ... within the 227 KiB opt-in limit with the kernel's static shared memory (under 1 KiB)
static_assert(DEC_SMEM_ATTR + 1024 <= 227 * 1024, "decode engine shared memory");
// dynamic shared memory of a CTA that still fits three to an SM (228 KiB,
// 1 KiB reserved per CTA, static shared memory under 1 KiB)
constexpr size_t DEC_SMEM_3 = 228 * 1024 / 3 - 2 * 1024;

static_assert(sizeof(DecodeParams) <= 32764, "decode parameters exceed the kernel parameter limit");

struct DeviceInfo {
    bool init = false;
    bool ok = false;
    int sms = 0;
};
DeviceInfo g_dev[MAX_DEVICES];
std::mutex g_dev_mu;

bl_status device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return BL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.init) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BL_ERR_CUDA;
        d.ok = (major == 10);
        d.sms = sms;
        if (d.ok) {
            // opt in to large dynamic shared memory once per device
            bool fail = false;
            for (auto fn : {k_decode<1, DEC_SRC_XQ>, k_decode<2, DEC_SRC_XQ>, k_decode<1, DEC_SRC_BF16>,
                            k_decode<2, DEC_SRC_BF16>, k_decode<1, DEC_SRC_F32>, k_decode<2, DEC_SRC_F32>})
                fail |= cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DEC_SMEM_ATTR) !=
                        cudaSuccess;
            fail |= prefill_setup() != cudaSuccess;
            fail |= dense_setup() != cudaSuccess;
            for (auto fn : {k_act_quant_subln_row<false, true>, k_act_quant_subln_row<true, false>,
                            k_act_quant_subln_row<false, false>})
                fail |= cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, AQR_MAX_K * 4) !=
                        cudaSuccess;
            if (fail) return BL_ERR_CUDA;
        }
        d.init = true;
    }
    if (!d.ok) return BL_ERR_DEVICE;
    *out = &d;
    return BL_OK;
}

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bl_status check_k(int64_t K) {
    if (K < 64 || K > K_MAX || (K % 64) != 0) return BL_ERR_SHAPE;
    return BL_OK;
}

// N * K < 2^31 without forming the product (N may be anything up to
// INT64_MAX; K has passed check_k, so 64 <= K <= K_MAX).
bool nk_fits(int64_t N, int64_t K) { return N <= ((1LL << 31) - 1) / K; }

// ---------------------------------------------------------------------------
// Step 1

// One weight matrix to quantize (all matrices of a launch share the dtype).
struct WqIn {
    const void *W;
    int64_t N, K;
    uint8_t *packed;
    float *gamma;
};

// Reduction blocks per matrix: a share of 2 x SMs proportional to its size,
// at least enough that no thread sums more than 2^14 terms (which keeps each
// 64-bit window accumulator exact), at most one vector per thread, and at
// most WQ_MAX_BLOCKS over the launch.  Pack blocks: a share of 8 x SMs (at
// most one word per thread), at least one per matrix.
bl_status quant_weights_impl(const DeviceInfo &d, const WqIn *in, int count, bl_dtype wdt, void *ws,
                             cudaStream_t st) {
    if (count < 1 || count > WQ_MAX_JOBS) return BL_ERR_SHAPE;
    const bool bf16 = wdt == BL_BF16;
    const int epv = bf16 ? 8 : 4;
    const long long vec_cap = 16384 / epv;  // vectors per thread
    WqParams P;
    memset(&P, 0, sizeof(P));
    P.count = count;
    P.partials = reinterpret_cast<u64 *>(ws);
    P.thresh = reinterpret_cast<u32 *>(reinterpret_cast<uint8_t *>(ws) + WQ_WS_PARTIALS);
    double total = 0.0;
    for (int i = 0; i < count; ++i) total += (double)in[i].N * (double)in[i].K;
    long long blocks = 0, words = 0;
    long long mins = 0;
    for (int i = 0; i < count; ++i) {
        const long long n = (long long)in[i].N * in[i].K;
        const long long nvec = n / epv;
        const long long need = (nvec + WQ_THREADS - 1) / WQ_THREADS;
        const long long minb = (nvec + (long long)WQ_THREADS * vec_cap - 1) / ((long long)WQ_THREADS * vec_cap);
        long long nb = (long long)std::llround(2.0 * d.sms * ((double)n / total));
        if (nb > need) nb = need;
        if (nb < minb) nb = minb;
        if (nb < 1) nb = 1;
        mins += minb;
        P.j[i] = WqJob{reinterpret_cast<const uint4 *>(in[i].W), nvec, n, in[i].gamma,
                       reinterpret_cast<u32 *>(in[i].packed), n / 16, (int)blocks, (int)nb, 0, 0, 0};
        blocks += nb;
        words += n / 16;
    }
    if (mins > WQ_MAX_BLOCKS) return BL_ERR_SHAPE;
    if (blocks > WQ_MAX_BLOCKS) {
        // scale the shares down (never below a matrix's minimum)
        blocks = 0;
        for (int i = 0; i < count; ++i) {
            const long long minb = (P.j[i].nvec + (long long)WQ_THREADS * vec_cap - 1) / ((long long)WQ_THREADS * vec_cap);
            long long nb = (long long)((double)P.j[i].nblk * (WQ_MAX_BLOCKS - mins) / (double)WQ_MAX_BLOCKS);
            if (nb < minb) nb = minb;
            if (nb < 1) nb = 1;
            P.j[i].blk0 = (int)blocks;
            P.j[i].nblk = (int)nb;
            blocks += nb;
        }
        if (blocks > WQ_MAX_BLOCKS) return BL_ERR_SHAPE;
    }
    // roundings a term of a matrix's double sum passes through: its thread's
    // chain (half of its elements per accumulator) plus the reduction trees
    for (int i = 0; i < count; ++i) {
        const long long per = (long long)P.j[i].nblk * WQ_THREADS;
        const long long vpt = (P.j[i].nvec + per - 1) / per;
        P.j[i].depth = (int)(vpt * epv / 2 + 64 + (P.j[i].nblk + WQ_PACK_THREADS - 1) / WQ_PACK_THREADS);
    }
    const long long pcap = 8LL * d.sms;
    long long pblocks = 0;
    for (int i = 0; i < count; ++i) {
        const long long need = (P.j[i].nwords + WQ_PACK_THREADS - 1) / WQ_PACK_THREADS;
        long long nb = (long long)std::llround((double)pcap * ((double)P.j[i].nwords / (double)words));
        if (nb > need) nb = need;
        if (nb < 1) nb = 1;
        P.j[i].pblk0 = (int)pblocks;
        P.j[i].pnblk = (int)nb;
        pblocks += nb;
    }
    if (bf16)
        k_absmean_partial<true><<<(unsigned)blocks, WQ_THREADS, 0, st>>>(P);
    else
        k_absmean_partial<false><<<(unsigned)blocks, WQ_THREADS, 0, st>>>(P);
    if (cudaGetLastError() != cudaSuccess) return BL_ERR_CUDA;
    // programmatic dependent launches: the final grid waits for the
    // reduction (griddepcontrol.wait) before it reads the partials; the pack
    // grid starts loading W while both run and waits for T
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(WQ_PACK_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)count);
    if ((bf16 ? cudaLaunchKernelEx(&cfg, k_absmean_final<true>, P) : cudaLaunchKernelEx(&cfg, k_absmean_final<false>, P)) !=
        cudaSuccess)
        return BL_ERR_CUDA;
    cfg.gridDim = dim3((unsigned)pblocks);
    cudaError_t e = bf16 ? cudaLaunchKernelEx(&cfg, k_ternary_pack<true>, P)
                         : cudaLaunchKernelEx(&cfg, k_ternary_pack<false>, P);
    return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

bl_status quant_weights_one(const DeviceInfo &d, const void *W, bl_dtype wdt, int64_t N, int64_t K, uint8_t *packed,
                            float *gamma, void *ws, cudaStream_t st) {
    const WqIn in{W, N, K, packed, gamma};
    return quant_weights_impl(d, &in, 1, wdt, ws, st);
}

// ---------------------------------------------------------------------------
// Step 2

// Kernel launch, optionally as a programmatic dependent launch (it may
// start while the kernel before it runs; the act-quant kernels end with
// griddepcontrol.wait, so their completion still implies that kernel's).
template <typename Kern>
bl_status launch_act(Kern kernel, unsigned grid, unsigned block, cudaStream_t st, bool pdl, const ActParams &P) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, P) == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

bl_status quant_act_impl(const ActParams &P, bl_dtype xdt, int64_t Kmax, cudaStream_t st, bool pdl = false) {
    const bool bf16 = xdt == BL_BF16;
    const bool glu = P.p[0].X2 != nullptr;  // all problems of a call alike (f32 only)
    const int epv = bf16 ? 8 : 4;
    const long long nvec = Kmax / epv;
    bool subln = false;
    for (int i = 0; i < P.count; ++i) subln |= P.p[i].gain != nullptr;
    const long long rows = (long long)P.count * P.M;
    const unsigned wgrid = (unsigned)((rows + AQW_WARPS - 1) / AQW_WARPS);
    if (subln && nvec > (glu ? 32 * AQS_V : 256) && Kmax <= AQR_MAX_K) {
        // SubLN rows (gated FFN rows longer than one chunk, plain rows longer
        // than 256 vectors): one CTA per row, the row cached in shared memory
        // as float (read once, each element divided once), four warps per
        // row.  Measured 1.9x faster than a warp per row for the gated
        // [8192, 4096] input, 2-10 % faster for bf16 rows of 2560 and 9728,
        // slower for bf16 rows of 1536 (which the chunked warp kernel keeps).
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)rows);
        cfg.blockDim = dim3(AQR_THREADS);
        cfg.dynamicSmemBytes = (size_t)Kmax * 4;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 1 : 0;
        cudaError_t e;
        if (glu) e = cudaLaunchKernelEx(&cfg, k_act_quant_subln_row<false, true>, P);
        else if (bf16) e = cudaLaunchKernelEx(&cfg, k_act_quant_subln_row<true, false>, P);
        else e = cudaLaunchKernelEx(&cfg, k_act_quant_subln_row<false, false>, P);
        return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
    }
    if (subln) {
        // one warp per row, chunked, any K (rows without a gain: plain)
        if (glu) return launch_act(k_act_quant_subln<false, true>, wgrid, AQW_WARPS * 32, st, pdl, P);
        if (bf16) return launch_act(k_act_quant_subln<true, false>, wgrid, AQW_WARPS * 32, st, pdl, P);
        return launch_act(k_act_quant_subln<false, false>, wgrid, AQW_WARPS * 32, st, pdl, P);
    }
    if (nvec <= 32 * 32) {
        // rows up to 1024 16-byte vectors: one warp per row, row in registers
        int vpl = 1;
        while (vpl * 32 < nvec) vpl *= 2;
        const unsigned grid = wgrid;
#define BL_AQW_CASE(B, V)                                                                       \
        if (bf16 == B && vpl == V) {                                                            \
            if (glu) return launch_act(k_act_quant_warp<false, V, true>, grid, AQW_WARPS * 32, st, pdl, P); \
            return launch_act(k_act_quant_warp<B, V>, grid, AQW_WARPS * 32, st, pdl, P);       \
        }
        BL_AQW_CASE(true, 1)
        BL_AQW_CASE(true, 2)
        BL_AQW_CASE(true, 4)
        BL_AQW_CASE(true, 8)
        BL_AQW_CASE(true, 16)
        BL_AQW_CASE(true, 32)
        BL_AQW_CASE(false, 1)
        BL_AQW_CASE(false, 2)
        BL_AQW_CASE(false, 4)
        BL_AQW_CASE(false, 8)
        BL_AQW_CASE(false, 16)
        BL_AQW_CASE(false, 32)
#undef BL_AQW_CASE
    }
    int vec = 1;
    while ((nvec + vec - 1) / vec > 1024) vec *= 2;
    int T = (int)(((nvec + vec - 1) / vec + 31) / 32 * 32);
    const unsigned grid = (unsigned)(P.count * P.M);
#define BL_AQ_CASE(B, V)                                                            \
    if (bf16 == B && vec == V) {                                                    \
        if (glu) return launch_act(k_act_quant<false, V, true>, grid, T, st, pdl, P); \
        return launch_act(k_act_quant<B, V>, grid, T, st, pdl, P);                  \
    }
    // at most 32 values per thread (bf16: 4 vectors, f32: 8 vectors)
    BL_AQ_CASE(true, 1)
    BL_AQ_CASE(true, 2)
    BL_AQ_CASE(true, 4)
    BL_AQ_CASE(false, 1)
    BL_AQ_CASE(false, 2)
    BL_AQ_CASE(false, 4)
    BL_AQ_CASE(false, 8)
    return BL_ERR_SHAPE;
#undef BL_AQ_CASE
}

// ---------------------------------------------------------------------------
// Steps 3 + 4

bool decode_eligible(int64_t M, int64_t K) { return M <= 16 && M * dec_row_stride((int)K) <= DEC_X_MAX; }


// One problem of a decode launch, as the entry points receive it.
struct DecodeJob {
    const uint8_t *packed;
    const float *gamma;
    const void *x;        // x_q (DEC_SRC_XQ) or X
    float *s;
    float *Y;
    int32_t *acc;
    const float *gain;
    int8_t *xq_out;
    int64_t N, K;
};

// Decode launches: each problem's 32-row groups cut into CTAs of T = 8 / G
// groups (G from K, raised to 8 when the problems are too few to fill the
// GPU); a CTA table maps each CTA to its problem.  A call with more CTAs or
// problems than one launch holds is split into several launches (a problem
// by row ranges).
// With `plan` set nothing is launched: each launch the call would make is
// appended to it as {CTAs, dynamic shared memory bytes, problems, then per
// problem: job index, first row, rows, glog, K chunks, first CTA}.
bl_status decode_launch(const DecodeJob *jobs, int count, int M, float eps, bool pdl, cudaStream_t st, int src,
                        int sms, std::vector<int> *plan = nullptr) {
    thread_local DecodeParams P;
    int pjob[BL_MAX_GROUP];
    int glog[BL_MAX_GROUP], kchs[BL_MAX_GROUP];
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        kchs[i] = dec_kch((int)jobs[i].K, M, DEC_SMEM_ATTR);
        glog[i] = kchs[i] > 1 ? 3 : dec_glog((int)jobs[i].K);
        const int64_t ng = (jobs[i].N + DEC_ROWS - 1) / DEC_ROWS;
        total += (ng + (DEC_WARPS >> glog[i]) - 1) / (DEC_WARPS >> glog[i]);
    }
    if (total < sms)
        for (int i = 0; i < count; ++i) glog[i] = 3;
    const int NT = M <= 8 ? 1 : 2;
    P.M = M;
    P.eps = eps;
    P.count = 0;
    int nc = 0, w_max = 0, rs_max = 0, t_max = 0;
    bool first = true;
    auto flush = [&]() -> bl_status {
        if (P.count == 0) return BL_OK;
        P.x_off = (w_max + DEC_W_PAD + 127) & ~127;
        P.acc_off = P.x_off + ((M * rs_max + 127) & ~127);
        const size_t smem = (size_t)P.acc_off + (size_t)t_max * DEC_ROWS * M * 4;
        if (M * rs_max > DEC_X_MAX || smem > DEC_SMEM_ATTR) return BL_ERR_SHAPE;
        if (plan != nullptr) {
            plan->insert(plan->end(), {nc, (int)smem, P.count});
            for (int q = 0; q < P.count; ++q)
                plan->insert(plan->end(), {pjob[q], P.p[q].row0, P.p[q].rows, P.p[q].glog, P.p[q].kch, P.p[q].cta_begin});
            P.count = 0;
            nc = w_max = rs_max = t_max = 0;
            return BL_OK;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)nc);
        cfg.blockDim = dim3(DEC_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl || !first ? 1 : 0;
        cudaError_t e;
        if (src == DEC_SRC_BF16)
            e = NT == 1 ? cudaLaunchKernelEx(&cfg, k_decode<1, DEC_SRC_BF16>, P)
                        : cudaLaunchKernelEx(&cfg, k_decode<2, DEC_SRC_BF16>, P);
        else if (src == DEC_SRC_F32)
            e = NT == 1 ? cudaLaunchKernelEx(&cfg, k_decode<1, DEC_SRC_F32>, P)
                        : cudaLaunchKernelEx(&cfg, k_decode<2, DEC_SRC_F32>, P);
        else
            e = NT == 1 ? cudaLaunchKernelEx(&cfg, k_decode<1, DEC_SRC_XQ>, P)
                        : cudaLaunchKernelEx(&cfg, k_decode<2, DEC_SRC_XQ>, P);
        if (e != cudaSuccess) return BL_ERR_CUDA;
        first = false;
        P.count = 0;
        nc = w_max = rs_max = t_max = 0;
        return BL_OK;
    };
    for (int i = 0; i < count; ++i) {
        const DecodeJob &j = jobs[i];
        const int N = (int)j.N, K = (int)j.K;
        const int T = DEC_WARPS >> glog[i];
        const int kch = kchs[i];
        const int wb = kch > 1 ? DEC_ROWS * DEC_KCH_B : T * DEC_ROWS * (K >> 2);
        for (int row = 0; row < N;) {
            // the launch's layout with this problem in it must fit
            const int w2 = wb > w_max ? wb : w_max;
            const int r2 = dec_row_stride(K) > rs_max ? dec_row_stride(K) : rs_max;
            const int t2 = T > t_max ? T : t_max;
            const size_t need_smem = (size_t)((w2 + DEC_W_PAD + 127) & ~127) + (size_t)((M * r2 + 127) & ~127) +
                                     (size_t)t2 * DEC_ROWS * M * 4;
            // (and a launch whose CTAs fit three to an SM is not given a
            // problem that would take that away from all of them)
            const size_t cur_smem = (size_t)((w_max + DEC_W_PAD + 127) & ~127) +
                                    (size_t)((M * rs_max + 127) & ~127) + (size_t)t_max * DEC_ROWS * M * 4;
            const bool lose3 = cur_smem <= DEC_SMEM_3 && need_smem > DEC_SMEM_3;
            if (P.count == BL_MAX_GROUP || nc == DEC_MAX_CTAS ||
                (P.count > 0 && (need_smem > DEC_SMEM_ATTR || lose3))) {
                bl_status rc = flush();
                if (rc) return rc;
            }
            const int need = (N - row + T * DEC_ROWS - 1) / (T * DEC_ROWS);
            const int cn = need < DEC_MAX_CTAS - nc ? need : DEC_MAX_CTAS - nc;
            const int nrows = cn * T * DEC_ROWS < N - row ? cn * T * DEC_ROWS : N - row;
            P.p[P.count] = DecodeProblem{j.packed, j.gamma, j.x, j.s, j.Y, j.acc, j.gain, j.xq_out,
                                         N, K, row, nrows, glog[i], nc, kch};
            for (int c = 0; c < cn; ++c) P.cta_problem[nc + c] = (unsigned char)P.count;
            pjob[P.count] = i;
            nc += cn;
            ++P.count;
            row += nrows;
            w_max = wb > w_max ? wb : w_max;
            rs_max = dec_row_stride(K) > rs_max ? dec_row_stride(K) : rs_max;
            t_max = T > t_max ? T : t_max;
        }
    }
    return flush();
}

bl_status forward_impl(const DeviceInfo &d, const uint8_t *packed, const float *gamma, const int8_t *x_q,
                       const float *s, int64_t M, int64_t N, int64_t K, float *Y, int32_t *acc_out, cudaStream_t st,
                       bool pdl = false) {
    if (decode_eligible(M, K)) {
        const DecodeJob job{packed, gamma, x_q, const_cast<float *>(s), Y, acc_out, nullptr, nullptr, N, K};
        return decode_launch(&job, 1, (int)M, 0.f, false, st, DEC_SRC_XQ, d.sms);
    }
    return prefill_launch(d.sms, packed, gamma, x_q, s, M, N, K, Y, acc_out, st, PF_DEFAULT_TIMEOUT_NS, -1, pdl);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Prefill-sized groups: problems sharing one activation (x_q, s, K) in one
// tcgen05 launch.
bl_status forward_grouped_prefill(const bl_problem *problems, int count, int64_t M, cudaStream_t st) {
    if (count > PF_MAX_PROB || M < 1 || M > 0x7fffffffLL) return BL_ERR_SHAPE;
    const bl_problem &q0 = problems[0];
    PrefillJob jobs[PF_MAX_PROB];
    for (int i = 0; i < count; ++i) {
        const bl_problem &q = problems[i];
        if (!q.packed || !q.gamma || !q.x_q || !q.s || !q.Y) return BL_ERR_NULL;
        if (q.x_q != q0.x_q || q.s != q0.s || q.K != q0.K) return BL_ERR_SHAPE;
        if (q.N < 1 || q.N > 0x7fffffffLL || check_k(q.K) != BL_OK) return BL_ERR_SHAPE;
        if (!aligned16(q.packed) || !aligned16(q.gamma) || !aligned16(q.x_q) || !aligned16(q.s) || !aligned16(q.Y) ||
            (q.acc_out && !aligned16(q.acc_out)))
            return BL_ERR_ALIGN;
        jobs[i] = PrefillJob{q.packed, q.gamma, q.Y, q.acc_out, q.N};
    }
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return prefill_launch_group(d->sms, jobs, count, q0.x_q, q0.s, M, q0.K, st);
}

}  // namespace

// ===========================================================================
// C ABI

extern "C" {

const char *bl_status_string(bl_status s) {
    switch (s) {
        case BL_OK: return "BL_OK";
        case BL_ERR_NULL: return "BL_ERR_NULL: a required pointer is NULL";
        case BL_ERR_SHAPE: return "BL_ERR_SHAPE: M, N, K or count outside the supported range";
        case BL_ERR_ALIGN: return "BL_ERR_ALIGN: a pointer is not 16-byte aligned";
        case BL_ERR_DTYPE: return "BL_ERR_DTYPE: unknown dtype code";
        case BL_ERR_CUDA: return "BL_ERR_CUDA: a CUDA runtime call or launch failed";
        case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a bounded device-side wait gave up";
        case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace missing or too small";
        case BL_ERR_DEVICE: return "BL_ERR_DEVICE: current device is not compute capability 10.x";
    }
    return "BL_ERR_UNKNOWN";
}

int bl_version(void) { return BL_VERSION; }

bl_status bl_check_device_error(bl_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return BL_ERR_CUDA;
    u32 v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return BL_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return BL_ERR_CUDA;
    return v ? BL_ERR_TIMEOUT : BL_OK;
}

size_t bl_quant_weights_workspace_bytes(int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return align256(WQ_WS_BYTES);
}

bl_status bl_quant_weights(const void *W, bl_dtype wdt, int64_t N, int64_t K, uint8_t *packed, float *gamma,
                           void *workspace, size_t workspace_bytes, bl_stream_t stream) {
    if (!W || !packed || !gamma) return BL_ERR_NULL;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    if (N < 1 || check_k(K) != BL_OK || !nk_fits(N, K)) return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(gamma)) return BL_ERR_ALIGN;
    if (!workspace || workspace_bytes < bl_quant_weights_workspace_bytes(N, K)) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return quant_weights_one(*d, W, wdt, N, K, packed, gamma, workspace, (cudaStream_t)stream);
}

bl_status bl_quant_weights_grouped(const bl_weight_problem *problems, int count, bl_dtype wdt, void *workspace,
                                   size_t workspace_bytes, bl_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_WQ_GROUP) return BL_ERR_SHAPE;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    WqIn in[BL_MAX_WQ_GROUP];
    for (int i = 0; i < count; ++i) {
        const bl_weight_problem &q = problems[i];
        if (!q.W || !q.packed || !q.gamma) return BL_ERR_NULL;
        if (q.N < 1 || check_k(q.K) != BL_OK || !nk_fits(q.N, q.K)) return BL_ERR_SHAPE;
        if (!aligned16(q.W) || !aligned16(q.packed) || !aligned16(q.gamma)) return BL_ERR_ALIGN;
        in[i] = WqIn{q.W, q.N, q.K, q.packed, q.gamma};
    }
    if (!workspace || workspace_bytes < bl_quant_weights_workspace_bytes(1, 64)) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return quant_weights_impl(*d, in, count, wdt, workspace, (cudaStream_t)stream);
}

bl_status bl_quant_act_grouped(const bl_act_problem *problems, int count, bl_dtype xdt, int64_t M, float subln_eps,
                               bl_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_GROUP || M < 1 || M * (int64_t)count > 0x7fffffffLL) return BL_ERR_SHAPE;
    if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_DTYPE;
    ActParams P;
    P.count = count;
    P.M = (int)M;
    P.eps = subln_eps;
    int64_t kmax = 0;
    for (int i = 0; i < count; ++i) {
        const bl_act_problem &q = problems[i];
        if (!q.X || !q.x_q || !q.s) return BL_ERR_NULL;
        if (check_k(q.K) != BL_OK) return BL_ERR_SHAPE;
        if (!aligned16(q.X) || !aligned16(q.x_q) || !aligned16(q.s) || (q.subln_gain && !aligned16(q.subln_gain)))
            return BL_ERR_ALIGN;
        P.p[i] = ActProblem{q.X, q.subln_gain, q.x_q, q.s, (int)q.K, 0};
        kmax = q.K > kmax ? q.K : kmax;
    }
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return quant_act_impl(P, xdt, kmax, (cudaStream_t)stream);
}

bl_status bl_ffn_act_quant(const float *gate, const float *up, int64_t M, int64_t F, const float *subln_gain,
                           float subln_eps, int8_t *x_q, float *s, bl_stream_t stream) {
    if (!gate || !up || !x_q || !s) return BL_ERR_NULL;
    if (M < 1 || M > 0x7fffffffLL || check_k(F) != BL_OK) return BL_ERR_SHAPE;
    if (!aligned16(gate) || !aligned16(up) || !aligned16(x_q) || !aligned16(s) ||
        (subln_gain && !aligned16(subln_gain)))
        return BL_ERR_ALIGN;
    ActParams P;
    P.count = 1;
    P.M = (int)M;
    P.eps = subln_eps;
    P.p[0] = ActProblem{gate, subln_gain, x_q, s, (int)F, 0, up};
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return quant_act_impl(P, BL_F32, F, (cudaStream_t)stream);
}

bl_status bl_quant_act(const void *X, bl_dtype xdt, int64_t M, int64_t K, const float *subln_gain, float subln_eps,
                       int8_t *x_q, float *s, bl_stream_t stream) {
    bl_act_problem q{X, subln_gain, x_q, s, K};
    return bl_quant_act_grouped(&q, 1, xdt, M, subln_eps, stream);
}

bl_status bl_forward(const uint8_t *packed, const float *gamma, const int8_t *x_q, const float *s, int64_t M,
                     int64_t N, int64_t K, float *Y, int32_t *acc_out, bl_stream_t stream) {
    if (!packed || !gamma || !x_q || !s || !Y) return BL_ERR_NULL;
    if (M < 1 || N < 1 || M > 0x7fffffffLL || N > 0x7fffffffLL || check_k(K) != BL_OK) return BL_ERR_SHAPE;
    if (!aligned16(packed) || !aligned16(gamma) || !aligned16(x_q) || !aligned16(s) || !aligned16(Y) ||
        (acc_out && !aligned16(acc_out)))
        return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return forward_impl(*d, packed, gamma, x_q, s, M, N, K, Y, acc_out, (cudaStream_t)stream);
}

bl_status bl_forward_glu(const uint8_t *packed_gate, const float *gamma_gate, const uint8_t *packed_up,
                         const float *gamma_up, const int8_t *x_q, const float *s, int64_t M, int64_t F, int64_t K,
                         float *h, bl_stream_t stream) {
    if (!packed_gate || !gamma_gate || !packed_up || !gamma_up || !x_q || !s || !h) return BL_ERR_NULL;
    if (M < 1 || M > 0x7fffffffLL || F < 64 || F > 0x7fffffffLL || (F % 64) != 0 || check_k(K) != BL_OK)
        return BL_ERR_SHAPE;
    if (!aligned16(packed_gate) || !aligned16(gamma_gate) || !aligned16(packed_up) || !aligned16(gamma_up) ||
        !aligned16(x_q) || !aligned16(s) || !aligned16(h))
        return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return prefill_launch_glu(d->sms, packed_gate, gamma_gate, packed_up, gamma_up, x_q, s, M, F, K, h,
                              (cudaStream_t)stream);
}

bl_status bl_backward_dx(const void *dY, const uint8_t *packed, const float *gamma, int64_t M, int64_t N, int64_t K,
                         float *dX, bl_stream_t stream) {
    if (!dY || !packed || !gamma || !dX) return BL_ERR_NULL;
    if (M < 1 || M > 0x7fffffffLL || N < 8 || N > 0x7fffffffLL || (N % 8) != 0 || check_k(K) != BL_OK)
        return BL_ERR_SHAPE;
    if (!aligned16(dY) || !aligned16(packed) || !aligned16(gamma) || !aligned16(dX)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return prefill_launch_bwd(d->sms, dY, packed, gamma, M, N, K, dX, (cudaStream_t)stream);
}

size_t bl_backward_dw_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || N < 1 || K < 1) return 0;
    return dw_workspace_bytes(M, N, K);
}

bl_status bl_backward_dw(const void *dY, const int8_t *x_q, const float *s, const void *W, bl_dtype wdt,
                         const float *gamma, float beta, int64_t M, int64_t N, int64_t K, void *workspace,
                         size_t workspace_bytes, float *dW, bl_stream_t stream) {
    if (!dY || !x_q || !s || !W || !gamma || !dW) return BL_ERR_NULL;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || M > 0x7fffffffLL - 64 || N < 1 || check_k(K) != BL_OK || !nk_fits(N, K)) return BL_ERR_SHAPE;
    if (!aligned16(dY) || !aligned16(x_q) || !aligned16(s) || !aligned16(W) || !aligned16(gamma) || !aligned16(dW))
        return BL_ERR_ALIGN;
    if (!workspace || workspace_bytes < dw_workspace_bytes(M, N, K)) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    EncodeTiledFn enc = encode_tiled_fn();
    if (enc == nullptr) return BL_ERR_CUDA;
    return dw_launch(enc, dY, x_q, s, W, wdt == BL_BF16, gamma, beta, M, N, K, workspace, dW, (cudaStream_t)stream);
}

bl_status bl_forward_grouped(const bl_problem *problems, int count, int64_t M, unsigned flags,
                             bl_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_GROUP || M < 1) return BL_ERR_SHAPE;
    bool decode = M <= 16;
    for (int i = 0; i < count && decode; ++i) decode = check_k(problems[i].K) == BL_OK && decode_eligible(M, problems[i].K);
    if (!decode) return forward_grouped_prefill(problems, count, M, (cudaStream_t)stream);
    DecodeJob jobs[BL_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        const bl_problem &q = problems[i];
        if (!q.packed || !q.gamma || !q.x_q || !q.s || !q.Y) return BL_ERR_NULL;
        if (q.N < 1 || q.N > 0x7fffffffLL || check_k(q.K) != BL_OK || !decode_eligible(M, q.K)) return BL_ERR_SHAPE;
        if (!aligned16(q.packed) || !aligned16(q.gamma) || !aligned16(q.x_q) || !aligned16(q.s) || !aligned16(q.Y) ||
            (q.acc_out && !aligned16(q.acc_out)))
            return BL_ERR_ALIGN;
        jobs[i] = DecodeJob{q.packed, q.gamma, q.x_q, const_cast<float *>(q.s), q.Y, q.acc_out, nullptr, nullptr,
                            q.N, q.K};
    }
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return decode_launch(jobs, count, (int)M, 0.f, (flags & BL_FWD_WEIGHTS_READY) != 0, (cudaStream_t)stream,
                         DEC_SRC_XQ, d->sms);
}

bl_status bl_linear_decode_grouped(const bl_decode_problem *problems, int count, bl_dtype xdt, int64_t M,
                                   float subln_eps, unsigned flags, bl_stream_t stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_GROUP || M < 1 || M > 16) return BL_ERR_SHAPE;
    if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_DTYPE;
    DecodeJob jobs[BL_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        const bl_decode_problem &q = problems[i];
        if (!q.packed || !q.gamma || !q.X || !q.Y) return BL_ERR_NULL;
        if (q.N < 1 || q.N > 0x7fffffffLL || check_k(q.K) != BL_OK || !decode_eligible(M, q.K)) return BL_ERR_SHAPE;
        if (!aligned16(q.packed) || !aligned16(q.gamma) || !aligned16(q.X) || !aligned16(q.Y) ||
            (q.subln_gain && !aligned16(q.subln_gain)) || (q.x_q && !aligned16(q.x_q)) ||
            (q.s && !aligned16(q.s)) || (q.acc_out && !aligned16(q.acc_out)))
            return BL_ERR_ALIGN;
        jobs[i] = DecodeJob{q.packed, q.gamma, q.X, q.s, q.Y, q.acc_out, q.subln_gain, q.x_q, q.N, q.K};
    }
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return decode_launch(jobs, count, (int)M, subln_eps, (flags & BL_FWD_WEIGHTS_READY) != 0, (cudaStream_t)stream,
                         xdt == BL_BF16 ? DEC_SRC_BF16 : DEC_SRC_F32, d->sms);
}

size_t bl_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || N < 1 || K < 1) return 0;
    return align256(WQ_WS_BYTES) + align256((size_t)N * (size_t)K / 4) + 256 + align256((size_t)M * (size_t)K) +
           align256((size_t)M * 4);
}

bl_status bl_linear(const void *W, bl_dtype wdt, const void *X, bl_dtype xdt, int64_t M, int64_t N, int64_t K,
                    const float *subln_gain, float subln_eps, void *workspace, size_t workspace_bytes, float *Y,
                    bl_stream_t stream) {
    if (!W || !X || !Y) return BL_ERR_NULL;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || N < 1 || M > 0x7fffffffLL || check_k(K) != BL_OK || !nk_fits(N, K)) return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(X) || !aligned16(Y) || (subln_gain && !aligned16(subln_gain)))
        return BL_ERR_ALIGN;
    if (!workspace || workspace_bytes < bl_linear_workspace_bytes(M, N, K)) return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    uint8_t *p = reinterpret_cast<uint8_t *>(workspace);
    void *wq_ws = p;
    p += align256(WQ_WS_BYTES);
    uint8_t *packed = p;
    p += align256((size_t)N * (size_t)K / 4);
    float *gamma = reinterpret_cast<float *>(p);
    p += 256;
    int8_t *x_q = reinterpret_cast<int8_t *>(p);
    p += align256((size_t)M * (size_t)K);
    float *s = reinterpret_cast<float *>(p);
    cudaStream_t st = (cudaStream_t)stream;
    rc = quant_weights_one(*d, W, wdt, N, K, packed, gamma, wq_ws, st);
    if (rc) return rc;
    if (decode_eligible(M, K)) {
        // decode-sized: activation quant fused into the GEMV launch (x_q and s
        // still land in the workspace)
        const DecodeJob job{packed, gamma, X, s, Y, nullptr, subln_gain, x_q, N, K};
        return decode_launch(&job, 1, (int)M, subln_eps, false, st, xdt == BL_BF16 ? DEC_SRC_BF16 : DEC_SRC_F32,
                             d->sms);
    }
    ActParams P;
    P.count = 1;
    P.M = (int)M;
    P.eps = subln_eps;
    P.p[0] = ActProblem{X, subln_gain, x_q, s, (int)K, 0};
    // the act quant depends only on X: it may run while the weight pack
    // finishes (programmatic dependent launch); the GEMM waits for both
    rc = quant_act_impl(P, xdt, K, st, true);
    if (rc) return rc;
    return forward_impl(*d, packed, gamma, x_q, s, M, N, K, Y, nullptr, st, true);
}

size_t bl_linear_grouped_workspace_bytes(const bl_linear_problem *problems, int count, int64_t M, int64_t K) {
    if (!problems || count < 1 || count > BL_MAX_PREFILL_GROUP || M < 1 || K < 1) return 0;
    size_t b = align256(WQ_WS_BYTES) + 256 + align256((size_t)M * (size_t)K) + align256((size_t)M * 4);
    for (int i = 0; i < count; ++i) {
        if (problems[i].N < 1) return 0;
        b += align256((size_t)problems[i].N * (size_t)K / 4);
    }
    return b;
}

bl_status bl_linear_grouped(const bl_linear_problem *problems, int count, bl_dtype wdt, const void *X, bl_dtype xdt,
                            int64_t M, int64_t K, const float *subln_gain, float subln_eps, void *workspace,
                            size_t workspace_bytes, bl_stream_t stream) {
    if (!problems || !X) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_PREFILL_GROUP) return BL_ERR_SHAPE;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    if (xdt != BL_F32 && xdt != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || M > 0x7fffffffLL || check_k(K) != BL_OK) return BL_ERR_SHAPE;
    if (!aligned16(X) || (subln_gain && !aligned16(subln_gain))) return BL_ERR_ALIGN;
    for (int i = 0; i < count; ++i) {
        const bl_linear_problem &q = problems[i];
        if (!q.W || !q.Y) return BL_ERR_NULL;
        if (q.N < 1 || !nk_fits(q.N, K)) return BL_ERR_SHAPE;
        if (!aligned16(q.W) || !aligned16(q.Y)) return BL_ERR_ALIGN;
    }
    if (!workspace || workspace_bytes < bl_linear_grouped_workspace_bytes(problems, count, M, K))
        return BL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    // workspace: [weight-quant scratch | gammas (16 B apart) | x_q | s | packed_0 | packed_1 ...]
    uint8_t *p = reinterpret_cast<uint8_t *>(workspace);
    void *wq_ws = p;
    p += align256(WQ_WS_BYTES);
    float *gammas = reinterpret_cast<float *>(p);
    p += 256;
    int8_t *x_q = reinterpret_cast<int8_t *>(p);
    p += align256((size_t)M * (size_t)K);
    float *s = reinterpret_cast<float *>(p);
    p += align256((size_t)M * 4);
    WqIn in[BL_MAX_PREFILL_GROUP];
    for (int i = 0; i < count; ++i) {
        in[i] = WqIn{problems[i].W, problems[i].N, K, p, gammas + 4 * i};
        p += align256((size_t)problems[i].N * (size_t)K / 4);
    }
    cudaStream_t st = (cudaStream_t)stream;
    rc = quant_weights_impl(*d, in, count, wdt, wq_ws, st);
    if (rc) return rc;
    if (decode_eligible(M, K)) {
        // decode-sized: the fused launch quantizes X itself (per CTA)
        DecodeJob jobs[BL_MAX_PREFILL_GROUP];
        for (int i = 0; i < count; ++i)
            jobs[i] = DecodeJob{in[i].packed, in[i].gamma, X, nullptr, problems[i].Y, nullptr, subln_gain, nullptr,
                                problems[i].N, K};
        return decode_launch(jobs, count, (int)M, subln_eps, false, st, xdt == BL_BF16 ? DEC_SRC_BF16 : DEC_SRC_F32,
                             d->sms);
    }
    ActParams P;
    P.count = 1;
    P.M = (int)M;
    P.eps = subln_eps;
    P.p[0] = ActProblem{X, subln_gain, x_q, s, (int)K, 0};
    // the act quant depends only on X: it may run while the weight pack
    // finishes (programmatic dependent launch); the GEMM waits for both
    rc = quant_act_impl(P, xdt, K, st, true);
    if (rc) return rc;
    PrefillJob jobs[BL_MAX_PREFILL_GROUP];
    for (int i = 0; i < count; ++i) jobs[i] = PrefillJob{in[i].packed, in[i].gamma, problems[i].Y, nullptr, problems[i].N};
    return prefill_launch_group(d->sms, jobs, count, x_q, s, M, K, st, PF_DEFAULT_TIMEOUT_NS, -1, true);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Weight quantization without caller-provided scratch (see the header): the
// reduction's per-block partials live in this static array.  Host code must
// not hand the symbol itself to a kernel -- in host code it names a
// host-side stand-in -- so the device address is looked up
// once per device with cudaGetSymbolAddress.

namespace {

static_assert(WQ_WS_BYTES <= BL_NOALLOC_SCRATCH_BYTES, "static weight-quant scratch too small");
static __device__ __align__(256) unsigned char g_noalloc_scratch[BL_NOALLOC_SCRATCH_BYTES];

void *g_noalloc_ptr[MAX_DEVICES];
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (set up on the
// first call per device, with that device current).
bl_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return BL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BL_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return BL_OK;
}

}  // namespace

extern "C" bl_status bl_quant_weights_noalloc(const void *W, bl_dtype wdt, int64_t N, int64_t K, uint8_t *packed,
                                              float *gamma, bl_stream_t stream) {
    if (!W || !packed || !gamma) return BL_ERR_NULL;
    if (wdt != BL_F32 && wdt != BL_BF16) return BL_ERR_DTYPE;
    if (N < 1 || check_k(K) != BL_OK || !nk_fits(N, K)) return BL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(packed) || !aligned16(gamma)) return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    return quant_weights_one(*d, W, wdt, N, K, packed, gamma, scratch, (cudaStream_t)stream);
}

extern "C" bl_status bl_debug_forward_prefill(const uint8_t *packed, const float *gamma, const int8_t *x_q,
                                              const float *s, int64_t M, int64_t N, int64_t K, float *Y,
                                              int32_t *acc_out, long long skip_iter, uint32_t timeout_us,
                                              bl_stream_t stream) {
    if (!packed || !gamma || !x_q || !s || !Y) return BL_ERR_NULL;
    if (M < 1 || N < 1 || M > 0x7fffffffLL || N > 0x7fffffffLL || check_k(K) != BL_OK || timeout_us == 0)
        return BL_ERR_SHAPE;
    if (!aligned16(packed) || !aligned16(gamma) || !aligned16(x_q) || !aligned16(s) || !aligned16(Y) ||
        (acc_out && !aligned16(acc_out)))
        return BL_ERR_ALIGN;
    DeviceInfo *d;
    bl_status rc = device_info(&d);
    if (rc) return rc;
    return prefill_launch(d->sms, packed, gamma, x_q, s, M, N, K, Y, acc_out, (cudaStream_t)stream,
                          (unsigned long long)timeout_us * 1000ull, skip_iter < 0 ? -1 : skip_iter);
}

extern "C" bl_status bl_debug_decode_plan(const int64_t *shapes, int count, int64_t M, int sms, int *out,
                                          int out_len, int *written) {
    if (!shapes || !out || !written) return BL_ERR_NULL;
    if (count < 1 || count > BL_MAX_GROUP || M < 1 || M > 16 || sms < 1 || out_len < 1) return BL_ERR_SHAPE;
    DecodeJob jobs[BL_MAX_GROUP];
    // placeholder addresses: the plan reads only the shapes
    static const float dummy[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < count; ++i) {
        const int64_t N = shapes[2 * i], K = shapes[2 * i + 1];
        if (N < 1 || N > 0x7fffffffLL || check_k(K) != BL_OK || !nk_fits(N, K) || !decode_eligible(M, K))
            return BL_ERR_SHAPE;
        jobs[i] = DecodeJob{reinterpret_cast<const uint8_t *>(dummy), dummy, dummy, nullptr, nullptr, nullptr,
                            nullptr, nullptr, N, K};
    }
    std::vector<int> plan;
    bl_status rc = decode_launch(jobs, count, (int)M, 0.f, false, nullptr, DEC_SRC_XQ, sms, &plan);
    if (rc) return rc;
    if ((int)plan.size() > out_len) return BL_ERR_WORKSPACE;
    std::memcpy(out, plan.data(), plan.size() * sizeof(int));
    *written = (int)plan.size();
    return BL_OK;
}

