"""Fused decode (bl_linear_decode_grouped: activation quant + ternary GEMV +
rescale in one launch) vs the CPU oracle.

x_q and s (written by the problem's first CTA on request) must equal the
oracle's bit for bit, acc exactly, Y within 1e-6 relative; Y must also be
bit-identical to the two-launch path (bl_quant_act_grouped +
bl_forward_grouped), since both compute the same x_q and s.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_act, check_forward_full, check_weights, gpu_quant_weights

pytestmark = pytest.mark.gpu


def _wide_rows(M, K, seed):
    # magnitudes spread over ~110 binades: several exact sum-of-squares windows
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float64)
    x = x * torch.pow(2.0, torch.randint(-90, 20, (M, K), generator=g).double())
    return x.float()


def _inputs(M, K, dtype, kind, seed):
    if kind == "outlier":
        return workloads.with_outlier_channels(workloads.normal((M, K), 1.0, seed, dtype), max(1, K // 100), 30.0,
                                               seed + 1)
    if kind == "student":
        return workloads.student_t((M, K), 3, 0.5, seed, dtype)
    if kind == "wide":
        return _wide_rows(M, K, seed).to(dtype)
    if kind == "tiny":  # rows below the 1e-5 floor, an all-zero row, subnormals
        X = (workloads.normal((M, K), 1.0, seed) * 1e-7).to(dtype)
        X[min(1, M - 1)] = 0
        if dtype == torch.float32:
            X[0, :8] = torch.tensor([1e-40, -3e-39, 2e-45, 0.0, 5e-41, -1e-44, 7e-39, 1e-38])
        return X
    if kind == "midpoint":
        # sum x^2 / K exactly halfway between two floats (K a power of two),
        # a row just above it, its negation and a normal row: the double
        # estimate of sum x^2 cannot decide the first and third, the exact sum does
        X = torch.zeros(M, K, dtype=torch.float32)
        X[0, 0], X[0, 1] = 8.0, 2.0 ** -9
        X[1, 0], X[1, 1], X[1, 2] = 8.0, 2.0 ** -9, 2.0 ** -30
        X[2] = -X[0]
        X[3] = workloads.normal((1, K), 1.0, seed)[0]
        return X.to(dtype)
    return workloads.normal((M, K), 1.0, seed, dtype)


def run_fused(items, M, dtype, eps=1e-6, outputs=True, flags=0):
    """items: list of (W cpu, X cpu, gain cpu or None).  Returns per-problem
    device tensors (packed, gamma, x_q, s, Y, acc)."""
    dev = []
    for W, X, gain in items:
        packed, gamma = gpu_quant_weights(W)
        N, K = W.shape
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda") if outputs else None
        s = torch.empty(M, dtype=torch.float32, device="cuda") if outputs else None
        acc = torch.empty(M, N, dtype=torch.int32, device="cuda") if outputs else None
        dev.append((packed, gamma, X.cuda(), None if gain is None else gain.cuda(), Y, xq, s, acc, N, K))
    arr = api.make_decode_problems(dev)
    api.bl_linear_decode_grouped(arr, len(dev), M, dtype, eps, flags)
    api.bl_check_device_error()
    return [(d[0], d[1], d[5], d[6], d[4], d[7]) for d in dev], arr, dev


@pytest.mark.parametrize("M,N,K,dtype,subln,kind", [
    (1, 2048, 768, torch.bfloat16, False, "normal"),
    (3, 37, 192, torch.float32, False, "outlier"),
    (8, 300, 2048, torch.bfloat16, True, "student"),
    (16, 300, 3200, torch.bfloat16, True, "outlier"),
    (5, 130, 9728, torch.float32, True, "normal"),
    (2, 33, 20480, torch.bfloat16, False, "normal"),
    (4, 40, 16384, torch.float32, True, "normal"),
    (13, 24, 9728, torch.bfloat16, True, "outlier"),
    (16, 64, 6144, torch.bfloat16, False, "outlier"),
    (6, 100, 1024, torch.float32, True, "wide"),
    (4, 70, 1024, torch.float32, False, "wide"),
    (4, 17, 128, torch.float32, True, "tiny"),
    (4, 17, 128, torch.float32, False, "tiny"),
    (9, 257, 64, torch.bfloat16, True, "normal"),
    (2, 50, 1024, torch.float32, False, "wide"),
    (1, 40, 4096, torch.bfloat16, False, "outlier"),
    (2, 33, 192, torch.float32, False, "tiny"),
    (4, 64, 4096, torch.bfloat16, True, "midpoint"),
    (4, 64, 2048, torch.float32, True, "midpoint"),
])
def test_fused_decode_matches_oracle(M, N, K, dtype, subln, kind):
    W = workloads.normal((N, K), 0.02, 500 + K)
    X = _inputs(M, K, dtype, kind, 600 + M)
    gain = workloads.uniform((K,), 0.9, 1.1, 700 + K) if subln else None
    (res,), _, _ = run_fused([(W, X, gain)], M, dtype)
    packed, gamma, x_q, s, Y, acc = res
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s, gain)
    check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_fused_decode_125m_all_projections(M):
    """All 84 projections of the 125M decode workload in one launch, with
    SubLN on the o and down projections."""
    items = workloads.decode125m(M=M)
    K_set = sorted({W.shape[1] for _, W, _ in items})
    gains = {K: workloads.uniform((K,), 0.9, 1.1, 800 + K) for K in K_set}
    probs = [(W, X, gains[W.shape[1]] if name.endswith((".o", ".down")) else None) for name, W, X in items]
    results, _, _ = run_fused(probs, M, torch.bfloat16)
    for (W, X, gain), (packed, gamma, x_q, s, Y, acc) in zip(probs, results):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        xq_ref, s_ref = check_act(X, x_q, s, gain)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_fused_equals_two_launch_path_and_optional_outputs():
    M = 8
    items = workloads.decode125m(M=M, layers=1)
    gains = {768: workloads.uniform((768,), 0.9, 1.1, 1), 2048: workloads.uniform((2048,), 0.9, 1.1, 2)}
    probs = [(W, X, gains[W.shape[1]] if name.endswith((".o", ".down")) else None) for name, W, X in items]
    results, _, dev = run_fused(probs, M, torch.bfloat16)
    # same problems without the optional outputs
    bare = [(d[0], d[1], d[2], d[3], torch.empty_like(d[4]), None, None, None, d[8], d[9]) for d in dev]
    api.bl_linear_decode_grouped(api.make_decode_problems(bare), len(bare), M, torch.bfloat16, 1e-6)
    # the two-launch path on the same device inputs
    acts, fwd = [], []
    for d in dev:
        xq = torch.empty_like(d[5])
        s = torch.empty_like(d[6])
        acts.append((d[2], d[3], xq, s))
        fwd.append((d[0], d[1], xq, s, torch.empty_like(d[4]), None, d[8], d[9]))
    api.bl_quant_act_grouped(acts, torch.bfloat16, 1e-6)
    api.bl_forward_grouped(api.make_problems(fwd), len(fwd), M)
    api.bl_check_device_error()
    for r, b, a, f in zip(results, bare, acts, fwd):
        assert torch.equal(r[2], a[2]) and torch.equal(r[3].view(torch.int32), a[3].view(torch.int32))
        assert torch.equal(r[4].view(torch.int32), b[4].view(torch.int32))
        assert torch.equal(r[4].view(torch.int32), f[4].view(torch.int32))


def test_fused_decode_programmatic_launch_sees_fresh_inputs():
    """With BL_FWD_WEIGHTS_READY the launch may overlap the kernel before it,
    but X written by that kernel must be what is quantized."""
    M = 4
    items = workloads.decode125m(M=M, layers=1)
    probs = [(W, X, None) for _, W, X in items]
    results, arr, dev = run_fused(probs, M, torch.bfloat16)
    new_X = [workloads.normal(tuple(d[2].shape), 2.0, 900 + i, torch.bfloat16) for i, d in enumerate(dev)]
    staged = [x.cuda() for x in new_X]
    for _ in range(3):
        for d, x in zip(dev, staged):
            d[2].copy_(x)  # the kernel right before each fused launch writes X
        api.bl_linear_decode_grouped(arr, len(dev), M, torch.bfloat16, 1e-6, api.BL_FWD_WEIGHTS_READY)
    api.bl_check_device_error()
    for (W, _, _), Xn, (packed, gamma, x_q, s, Y, acc) in zip(probs, new_X, results):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        xq_ref, s_ref = check_act(Xn, x_q, s)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)
