"""Pins for the oracle's straight-through backward (the next step of the
path: the QAT backward GEMMs).  Checked against what the pages print (the
STE scale values of "bitone" README, Soft-STE notes; tests/golden/ste_scale.txt)
and against the forward oracle through the adjoint identity, never against
the backward's own formulas:

  sum(G * Y) = sum(dX * X_hat)            (dX is the adjoint of X_hat -> Y)
  sum(G * Y) = sum(dW * gamma W_q)        (unmasked weights)

with Y the forward oracle's output, X_hat = x_q / s the dequantized input it
multiplies, and G the upstream gradient.  A transposed operand, a dropped
gamma or 1/s, or a wrong sign fails these.
"""
from __future__ import annotations

import os

import numpy as np
import pytest

import oracle
from ternary_quantized_linear_bitlinear_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_scales():
    rows = []
    with open(os.path.join(GOLDEN, "ste_scale.txt")) as f:
        for ln in f:
            ln = ln.split("#")[0].strip()
            if ln:
                ws, beta, exp, tol = (float(v) for v in ln.split())
                rows.append((ws, beta, exp, tol))
    return rows


@pytest.mark.parametrize("ws,beta,expected,tol", _golden_scales())
def test_ste_scale_matches_the_printed_values(ws, beta, expected, tol):
    # gamma = 0.5 and w = ws * gamma are exact floats, so w / gamma == ws
    gamma = np.float32(0.5)
    W = np.array([[ws * 0.5] * 64], dtype=np.float32)
    dY = np.ones((1, 1), dtype=np.float32)
    xq = np.ones((1, 64), dtype=np.int8)
    s = np.ones(1, dtype=np.float32)
    dW = oracle.bwd_dw(dY, xq, s, W, gamma, beta)  # unmasked gradient is exactly 1
    assert abs(dW[0, 0] - expected) <= tol
    if beta > 0:
        assert dW[0, 0] > 0.0  # the soft scale never freezes a weight


def _forward(seed, M, N, K):
    W = workloads.normal((N, K), 0.02, seed).numpy()
    X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, seed + 1), 2, 20.0, seed + 2).numpy()
    ref = oracle.linear(W, X)
    G = workloads.normal((M, N), 1.0, seed + 3).numpy()
    X_hat = ref["xq"].astype(np.float64) / ref["s"].astype(np.float64)[:, None]
    return W, ref, G, X_hat


@pytest.mark.parametrize("M,N,K", [(1, 7, 64), (5, 33, 192), (16, 64, 768)])
def test_dx_is_the_adjoint_of_the_forward(M, N, K):
    W, ref, G, X_hat = _forward(10 + M, M, N, K)
    dX = oracle.bwd_dx(G, ref["wq"], ref["gamma"])
    lhs = float(np.sum(G.astype(np.float64) * ref["Y"]))
    rhs = float(np.sum(dX * X_hat))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, float(np.sum(np.abs(G.astype(np.float64) * ref["Y"]))))
    # and dX's own structure: zero weight columns give zero gradient columns
    wq = ref["wq"].copy()
    wq[:, 0] = 0
    assert np.all(oracle.bwd_dx(G, wq, ref["gamma"])[:, 0] == 0.0)


@pytest.mark.parametrize("M,N,K", [(1, 7, 64), (5, 33, 192), (16, 64, 768)])
def test_dw_is_the_adjoint_of_the_forward(M, N, K):
    W, ref, G, X_hat = _forward(20 + M, M, N, K)
    gamma = np.float32(ref["gamma"])
    Wc = np.clip(W, -gamma, gamma)  # every |w / gamma| <= 1: the hard mask keeps all
    dW = oracle.bwd_dw(G, ref["xq"], ref["s"], Wc, gamma, 0.0)
    lhs = float(np.sum(G.astype(np.float64) * ref["Y"]))
    rhs = float(np.sum(dW * (float(gamma) * ref["wq"].astype(np.float64))))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, float(np.sum(np.abs(G.astype(np.float64) * ref["Y"]))))


def test_hard_mask_freezes_only_weights_outside_the_range():
    rng = np.random.default_rng(5)
    M, N, K = 3, 8, 64
    gamma = np.float32(0.25)
    W = (rng.standard_normal((N, K)) * 0.25).astype(np.float32)
    W[0, 0], W[1, 1], W[2, 2] = gamma, -gamma, np.nextafter(gamma, np.float32(1))  # boundary, boundary, just out
    dY = rng.standard_normal((M, N)).astype(np.float32)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    s = (rng.random(M) + 0.5).astype(np.float32)
    hard = oracle.bwd_dw(dY, xq, s, W, gamma, 0.0)
    soft = oracle.bwd_dw(dY, xq, s, W, gamma, 2.0)
    # without the mask (soft with beta -> 0 tends to 1): the same raw gradient
    raw = oracle.bwd_dw(dY, xq, s, np.zeros_like(W), gamma, 0.0)
    outside = np.abs(W / gamma) > 1  # the float division of the forward
    assert outside[2, 2] and not outside[0, 0] and not outside[1, 1]
    assert np.all(hard[outside] == 0.0)
    assert np.array_equal(hard[~outside], raw[~outside])
    assert np.all(np.abs(soft) <= np.abs(raw) + 0.0) and np.all((soft == 0) == (raw == 0))
