"""GPU path vs CPU oracle, element by element, through the C ABI.

Bit-exact: packed weights, gamma, x_q, s, acc.  Y: |Y - Y_ref| <= 1e-6 |Y_ref|.
Small cases cover several tiles plus ragged tails; the full-size cases run
the workloads' shapes in the launch configuration the benchmark times and
compare sampled outputs (all outputs where the oracle is fast enough).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import (check_act, check_forward_full, check_forward_sampled, check_weights, check_y, gpu_quant_weights,
                     np32)

pytestmark = pytest.mark.gpu


def chain(W_cpu, X_cpu, gain_cpu=None, eps=1e-6, want_acc=True):
    """GPU: quant weights, quant act, forward.  Returns device tensors."""
    W = W_cpu.cuda()
    X = X_cpu.cuda()
    packed, gamma = api.bl_quant_weights(W)
    x_q, s = api.bl_quant_act(X, None if gain_cpu is None else gain_cpu.cuda(), eps)
    M, N = X.shape[0], W.shape[0]
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda") if want_acc else None
    Y = api.bl_forward(packed, gamma, x_q, s, N, acc_out=acc)
    api.bl_check_device_error()
    return packed, gamma, x_q, s, Y, acc


# -- step 1 --------------------------------------------------------------------

@pytest.mark.parametrize("N,K,dtype,kind", [
    (2048, 768, torch.float32, "normal"),
    (37, 192, torch.float32, "normal"),
    (37, 192, torch.bfloat16, "normal"),
    (1, 64, torch.float32, "normal"),
    (300, 4096, torch.bfloat16, "normal"),
    (64, 1024, torch.float32, "wide"),
    (48, 512, torch.float32, "zeros"),
    (33, 320, torch.bfloat16, "ternary"),
    (9728, 2560, torch.bfloat16, "normal"),
    (64, 1024, torch.bfloat16, "wide"),
    (48, 512, torch.bfloat16, "zeros"),
    (512, 2048, torch.bfloat16, "outliers"),
    # sum |W| / n exactly halfway between two floats: the double estimate
    # cannot decide gamma, the exact sum in the final block does
    (1, 64, torch.bfloat16, "midpoint"),
    (4, 64, torch.float32, "midpoint"),
    (64, 4096, torch.bfloat16, "midpoint"),
])
def test_quant_weights(N, K, dtype, kind):
    if kind == "normal":
        W = workloads.normal((N, K), 0.02, 100 + N, dtype)
    elif kind == "wide":
        # exponents spread over ~230 binades, subnormals and zeros: every
        # exact-sum path (window, bins, subnormal) is exercised
        g = torch.Generator().manual_seed(5)
        mant = torch.randn(N, K, generator=g, dtype=torch.float64)
        ex = torch.randint(-150, 80, (N, K), generator=g).double()
        W = (mant * torch.pow(2.0, ex)).float()
        W[0, :17] = 0.0
        W[1, :5] = torch.tensor([1e-45, -3e-44, 1e-39, 3e38, -2e38])
        W = W.to(dtype)
    elif kind == "zeros":
        W = torch.zeros(N, K, dtype=dtype)
    elif kind == "midpoint":
        # n / 2 - 1 entries of 2, one of 1, one of -1 and one of -2^-24 n, the
        # rest zero: sum |W| = n (1 + 2^-24)
        n = N * K
        W = torch.zeros(n, dtype=torch.float32)
        W[: n // 2 - 1] = 2.0
        W[n // 2 - 1] = 1.0
        W[n // 2] = -1.0
        W[n // 2 + 1] = -(2.0 ** -24) * n
        W = W.reshape(N, K).to(dtype)
    elif kind == "outliers":
        # a few values outside the summing window of their block (tiny, a
        # subnormal, huge) among normal ones: only the threads that meet
        # them take the exact slow path
        W = workloads.normal((N, K), 0.02, 7, torch.float32)
        W[3, 7] = 1e-30
        W[100, 5] = -(2.0 ** -130)
        W[200, 1000] = 1e20
        W[511, 2047] = 0.0
        W = W.to(dtype)
    else:
        W = workloads.ternary_weights(N, K, seed=3, dtype=dtype)
    packed, gamma = gpu_quant_weights(W)
    check_weights(W, packed, gamma)
    if kind == "zeros":
        assert gamma.item() == np.float32(1e-5)
        assert bool(torch.all(packed == 0x55))  # code 01 = 0 for every weight


def test_quant_weights_workspace_contents_ignored_and_reused():
    """The workspace may hold anything on entry (here all 0xFF bytes), and back-to-back
    calls on one workspace and stream (the second launched while the first may still
    run) give each tensor's own result."""
    Ws = [workloads.normal((300, 4096), 0.02, 31, torch.bfloat16), workloads.normal((37, 192), 0.03, 32),
          workloads.normal((2048, 768), 0.02, 33, torch.bfloat16)]
    ws = torch.full((api.quant_weights_workspace_bytes(2048, 4096),), 255, dtype=torch.uint8, device="cuda")
    outs = []
    for W in Ws:
        Wd = W.cuda()
        outs.append(api.bl_quant_weights(Wd, workspace=ws))
    api.bl_check_device_error()
    for W, (packed, gamma) in zip(Ws, outs):
        check_weights(W, packed, gamma)


# -- step 2 --------------------------------------------------------------------

def _wide_rows(M, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float64)
    x = x * torch.pow(2.0, torch.randint(-90, 20, (M, K), generator=g).double())
    return x.float()


@pytest.mark.parametrize("M,K,dtype,subln,kind", [
    (16, 768, torch.float32, False, "outlier"),
    (5, 3200, torch.bfloat16, False, "outlier"),
    (3, 2048, torch.float32, False, "outlier"),
    (7, 4096, torch.bfloat16, False, "student"),
    (70, 4032, torch.bfloat16, False, "normal"),
    (3, 64, torch.float32, False, "normal"),
    (2, 32768, torch.float32, False, "normal"),
    (2, 32768, torch.bfloat16, True, "normal"),
    (4, 128, torch.float32, False, "tiny"),
    (33, 2560, torch.bfloat16, True, "normal"),
    (4, 9728, torch.float32, True, "normal"),
    (6, 1024, torch.float32, True, "wide"),
    (7, 9728, torch.bfloat16, True, "student"),
    (6, 4096, torch.float32, True, "wide"),
    (3, 2560, torch.bfloat16, True, "wide"),
    # bf16 SubLN rows of the CTA-per-row kernel: its one-accumulator exact
    # sum of squares (nonzero |x| within 19 binades, no subnormal) and the
    # windowed one it falls back to
    (4, 4096, torch.bfloat16, True, "tiny"),
    (3, 24576, torch.bfloat16, True, "normal"),
    (5, 2560, torch.bfloat16, True, "span"),
    # rows whose sum of squares / K lies exactly on, or just off, a float
    # rounding boundary: the double-sum estimate cannot decide them, the
    # exact windowed sum does
    (4, 4096, torch.bfloat16, True, "midpoint"),
    (4, 2048, torch.float32, True, "midpoint"),
    # the same rows short enough for the warp-per-row SubLN quantizer
    (4, 2048, torch.bfloat16, True, "midpoint"),
    (4, 1024, torch.float32, True, "midpoint"),
])
def test_quant_act(M, K, dtype, subln, kind):
    if kind == "outlier":
        X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 7, dtype), max(1, K // 100), 30.0, 8)
    elif kind == "normal":
        X = workloads.normal((M, K), 1.0, 9, dtype)
    elif kind == "student":
        X = workloads.student_t((M, K), 3, 0.5, 10, dtype)
    elif kind == "wide":
        X = _wide_rows(M, K, 11).to(dtype)
    elif kind == "span":
        # rows whose nonzero |x| span exactly 19 binades (the one-accumulator
        # limit), 20 binades, one subnormal, and huge values (2^60)
        X = workloads.normal((M, K), 1.0, 14).to(dtype).float()
        X = X.sign() * (X.abs().clamp(2.0 ** -8, 2.0 ** 8 - 1))
        X[0, 0], X[0, 1] = 2.0 ** 10, 2.0 ** -9          # exponents 10 .. -9: span 19
        X[1, 0], X[1, 1] = 2.0 ** 10, -(2.0 ** -10)      # span 20
        X[2, 5] = 2.0 ** -130                            # a subnormal (bf16 keeps it)
        X[3] = X[3] * 2.0 ** 52                          # up to 2^60
        X = X.to(dtype)
    elif kind == "midpoint":
        # sum x^2 = 64 + 2^-18 with K = 2^12 (or 2^11): S / K = 2^-6 (1 + 2^-24)
        # (or 2^-5 (1 + 2^-24)), halfway between two floats; then a row just
        # above it, its negation, and a normal row
        X = torch.zeros(M, K, dtype=torch.float32)
        X[0, 0], X[0, 1] = 8.0, 2.0 ** -9
        X[1, 0], X[1, 1], X[1, 2] = 8.0, 2.0 ** -9, 2.0 ** -30
        X[2] = -X[0]
        X[3] = workloads.normal((1, K), 1.0, 15)[0]
        X = X.to(dtype)
    else:  # rows below the 1e-5 floor, and an all-zero row
        X = (workloads.normal((M, K), 1.0, 12) * 1e-7).to(dtype)
        X[1] = 0
    gain = workloads.uniform((K,), 0.9, 1.1, 13) if subln else None
    x_q, s = api.bl_quant_act(X.cuda(), None if gain is None else gain.cuda(), 1e-6)
    torch.cuda.synchronize()
    check_act(X, x_q, s, gain)


# -- steps 3 + 4 -------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [
    (1, 2048, 768), (3, 37, 192), (8, 2048, 768), (16, 300, 3200), (1, 8640, 3200),
    (4, 3200, 8640), (1, 17, 64), (16, 64, 6144), (2, 33, 32768),
    (17, 300, 1536), (100, 37, 4096), (257, 130, 768), (64, 256, 64),
])
def test_forward(M, N, K):
    W = workloads.normal((N, K), 0.02, 200 + K)
    X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 300 + M, torch.bfloat16), 2, 20.0, 4)
    packed, gamma, x_q, s, Y, acc = chain(W, X)
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s)
    check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_forward_without_acc_and_zero_rows():
    M, N, K = 9, 50, 256
    W = workloads.normal((N, K), 0.02, 1)
    X = workloads.normal((M, K), 1.0, 2)
    X[3] = 0
    packed, gamma, x_q, s, Y, acc = chain(W, X)
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s)
    check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)
    Y2 = api.bl_forward(packed, gamma, x_q, s, N)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    assert torch.all(Y[3] == 0)


# -- grouped decode: every projection of the 125M decode workload -----------

@pytest.mark.parametrize("M", [1, 4, 8])
def test_grouped_decode_125m(M):
    items = workloads.decode125m(M=M)
    dev, probs, refs = [], [], []
    for name, W, X in items:
        packed, gamma = gpu_quant_weights(W)
        x_q, s = api.bl_quant_act(X.cuda())
        N, K = W.shape
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
        dev.append((packed, gamma, x_q, s, Y, acc, N, K))
        refs.append((W, X))
    arr = api.make_problems(dev)
    api.bl_forward_grouped(arr, len(dev), M)
    api.bl_check_device_error()
    for (packed, gamma, x_q, s, Y, acc, N, K), (W, X) in zip(dev, refs):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        xq_ref, s_ref = check_act(X, x_q, s)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


@pytest.mark.parametrize("M,K,Ns,with_acc", [
    (300, 768, (768, 256, 256), False),       # q, k, v of one layer sharing x_q; ragged M
    (200, 1536, (4096, 4096), False),         # gate, up
    (129, 192, (37, 300, 256, 64), True),     # ragged N, int32 outputs (plain stores)
    (40, 64, (1,), False),                    # a one-problem group, N = 1
])
def test_grouped_prefill_shared_activation(M, K, Ns, with_acc):
    """One tcgen05 launch over several weight matrices that share x_q."""
    X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 700 + M, torch.bfloat16), 2, 20.0, 5)
    x_q, s = api.bl_quant_act(X.cuda())
    probs, refs = [], []
    for i, N in enumerate(Ns):
        W = workloads.normal((N, K), 0.02, 710 + i)
        packed, gamma = gpu_quant_weights(W)
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        acc = torch.empty(M, N, dtype=torch.int32, device="cuda") if with_acc else None
        probs.append((packed, gamma, x_q, s, Y, acc, N, K))
        refs.append(W)
    api.bl_forward_grouped(api.make_problems(probs), len(probs), M)
    api.bl_check_device_error()
    xq_ref, s_ref = check_act(X, x_q, s)
    for (packed, gamma, _, _, Y, acc, N, K_), W in zip(probs, refs):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        if acc is None:
            check_y(Y.cpu().numpy(), oracle.contract(xq_ref, wq_ref), g_ref, s_ref[:, None])
        else:
            check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_grouped_act_quant_matches_single():
    items = workloads.decode125m(M=4, layers=1)
    dev = []
    for name, W, X in items:
        Xd = X.cuda()
        dev.append((Xd, None, torch.empty_like(Xd, dtype=torch.int8), torch.empty(4, device="cuda")))
    api.bl_quant_act_grouped(dev, torch.bfloat16)
    torch.cuda.synchronize()
    for (Xd, _, xq, s), (name, W, X) in zip(dev, items):
        check_act(X, xq, s)


# -- fused bl_linear -----------------------------------------------------------

def test_linear_single_workload():
    W, X = workloads.single()
    Y = api.bl_linear(W.cuda(), X.cuda())
    torch.cuda.synchronize()
    ref = oracle.linear(np32(W), np32(X))
    err = np.abs(Y.cpu().numpy().astype(np.float64) - ref["Y"])
    assert np.all(err <= 1e-6 * np.abs(ref["Y"]))


def test_linear_subln_qat4b_oproj_small():
    name, W, X, gain = workloads.qat4b(M=96, which=("o",))[0]
    Y = api.bl_linear(W.cuda(), X.cuda(), gain.cuda(), workloads.SUBLN_EPS)
    torch.cuda.synchronize()
    ref = oracle.linear(np32(W), np32(X), np32(gain), workloads.SUBLN_EPS)
    err = np.abs(Y.cpu().numpy().astype(np.float64) - ref["Y"])
    assert np.all(err <= 1e-6 * np.abs(ref["Y"]))


def test_linear_back_to_back_calls_share_a_workspace():
    """Prefill-sized bl_linear calls in a row on one stream and one workspace:
    inside a call the act quant overlaps the weight pack (programmatic
    dependent launch); each call must still see only its own inputs."""
    cases = [(300, 130, 768, None), (200, 257, 1536, 21), (300, 64, 768, 22)]
    ws = torch.empty(max(api.linear_workspace_bytes(M, N, K) for M, N, K, _ in cases), dtype=torch.uint8,
                     device="cuda")
    outs, refs = [], []
    for i, (M, N, K, gseed) in enumerate(cases):
        W = workloads.normal((N, K), 0.02, 40 + i, torch.bfloat16)
        X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 50 + i, torch.bfloat16), 2, 20.0, 60 + i)
        gain = None if gseed is None else workloads.uniform((K,), 0.9, 1.1, gseed)
        outs.append(api.bl_linear(W.cuda(), X.cuda(), None if gain is None else gain.cuda(), workloads.SUBLN_EPS,
                                  workspace=ws))
        refs.append((W, X, gain))
    torch.cuda.synchronize()
    for Y, (W, X, gain) in zip(outs, refs):
        ref = oracle.linear(np32(W), np32(X), None if gain is None else np32(gain), workloads.SUBLN_EPS)
        err = np.abs(Y.cpu().numpy().astype(np.float64) - ref["Y"])
        assert np.all(err <= 1e-6 * np.abs(ref["Y"]))


# -- tcgen05 prefill engine at small M, and its bounded waits ----------------

@pytest.mark.parametrize("M,N,K", [
    (128, 128, 128), (1, 37, 64), (5, 300, 192), (16, 128, 1536), (200, 130, 768), (129, 257, 4096),
    (300, 64, 8640),
])
def test_prefill_engine_forced(M, N, K):
    W = workloads.normal((N, K), 0.02, 500 + K)
    X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 600 + M, torch.bfloat16), 2, 20.0, 4)
    packed, gamma = api.bl_quant_weights(W.cuda())
    x_q, s = api.bl_quant_act(X.cuda())
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    Y = api.bl_debug_forward_prefill(packed, gamma, x_q, s, N, acc_out=acc)
    api.bl_check_device_error()
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s)
    check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_prefill_bounded_wait_gives_up_and_context_survives():
    M, N, K = 256, 256, 1024
    W = workloads.normal((N, K), 0.02, 7)
    X = workloads.normal((M, K), 1.0, 8, torch.bfloat16)
    packed, gamma = api.bl_quant_weights(W.cuda())
    x_q, s = api.bl_quant_act(X.cuda())
    api.bl_check_device_error()
    # the producer never issues k-iteration 0: every consumer's wait runs out
    api.bl_debug_forward_prefill(packed, gamma, x_q, s, N, skip_iter=0, timeout_us=2000)
    with pytest.raises(api.BitLinearError) as e:
        api.bl_check_device_error()
    assert e.value.status == 6  # BL_ERR_TIMEOUT
    api.bl_check_device_error()  # the error word was cleared
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    Y = api.bl_forward(packed, gamma, x_q, s, N, acc_out=acc)
    api.bl_check_device_error()
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s)
    check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_grouped_decode_with_programmatic_launch():
    M = 8
    items = workloads.decode125m(M=M, layers=1)
    acts, dev, refs = [], [], []
    for name, W, X in items:
        packed, gamma = gpu_quant_weights(W)
        N, K = W.shape
        Xd = X.cuda()
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        s = torch.empty(M, dtype=torch.float32, device="cuda")
        acts.append((Xd, None, xq, s))
        dev.append((packed, gamma, xq, s, torch.empty(M, N, device="cuda"),
                    torch.empty(M, N, dtype=torch.int32, device="cuda"), N, K))
        refs.append((W, X))
    arr = api.make_problems(dev)
    for _ in range(3):  # act quant immediately followed by the dependent GEMV
        api.bl_quant_act_grouped(acts, torch.bfloat16)
        api.bl_forward_grouped(arr, len(dev), M, flags=api.BL_FWD_WEIGHTS_READY)
    api.bl_check_device_error()
    for (packed, gamma, x_q, s, Y, acc, N, K), (W, X) in zip(dev, refs):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        xq_ref, s_ref = check_act(X, x_q, s)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)
