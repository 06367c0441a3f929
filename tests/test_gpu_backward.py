"""Straight-through backward of the activation, dX = dY (gamma W_q), on the
tensor cores (bl_backward_dx: bf16 dY, f32 accumulation) against the
oracle's double-precision bwd_dx on the same bf16 dY.

Tolerance, from the arithmetic: every product dY * W_q is a bf16 value or
its negation (exact in f32), so the only error is the f32 accumulation over
N terms in the hardware's order -- at most N * 2^-23 of sum_n |dY W_q| when
every addition rounds, whatever the rounding direction -- plus the final
rounding of gamma * sum (2^-24 relative).  The test allows twice that."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_weights, np32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [
    (256, 2048, 768),      # one m tile, several n tiles of K
    (300, 768, 2048),      # ragged M (two pair tiles), K = 8 n-tiles of 256
    (1000, 1536, 1536),
    (64, 8, 64),           # N = 8: one partial reduction stage, tails everywhere
    (2048, 4096, 1536),    # a 1.4B-shape gate projection's dX: 6 x 8 tiles over 74 pairs
])
def test_backward_dx_matches_oracle(M, N, K):
    W = workloads.normal((N, K), 0.02, 900 + N)
    dY = workloads.normal((M, N), 1.0, 901 + M, torch.bfloat16)
    dY[0, : N // 2] = 0.0  # a row half of zeros
    packed, gamma = api.bl_quant_weights(W.cuda())
    dX = api.bl_backward_dx(dY.cuda(), packed, gamma, K)
    api.bl_check_device_error()
    wq, g = check_weights(W, packed, gamma)
    ref = oracle.bwd_dx(np32(dY), wq, g)
    bound = oracle.bwd_dx(np.abs(np32(dY)), np.abs(wq), g)   # gamma * sum_n |dY W_q|
    err = np.abs(dX.cpu().numpy().astype(np.float64) - ref)
    lim = 2.0 * (N * 2.0 ** -23 * bound + 2.0 ** -24 * np.abs(ref))
    assert np.all(err <= lim), f"max excess {(err - lim).max():.3e}"
    # a zero dY row gives exactly zero
    dY0 = torch.zeros(4, N, dtype=torch.bfloat16)
    dX0 = api.bl_backward_dx(dY0.cuda(), packed, gamma, K)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dX0).item() == 0


@pytest.mark.parametrize("M,N,K,beta,wdt", [
    (300, 768, 768, 0.0, torch.float32),     # hard mask, ragged M (padded to 320 tokens)
    (64, 256, 2048, 2.0, torch.bfloat16),    # soft scale, beta = 2 (the Soft-STE default)
    (1000, 130, 192, 2.0, torch.float32),    # ragged N and K tiles
    (4096, 1536, 512, 0.0, torch.bfloat16),  # many tokens per output
])
def test_backward_dw_matches_oracle(M, N, K, beta, wdt):
    """dW = (dY^T x_q / s) * scale(W / gamma) against the oracle's double
    computation.  Tolerance from the arithmetic: x_q / s is rounded to bf16
    (2^-9 relative per term), the f32 sum over M terms in the hardware's
    order (at most M * 2^-23 of sum_m |dY x_q / s|), the final product's
    rounding (2^-24), and for the soft scale the float tanh against double
    (a few 2^-24 absolute on the scale, which near tanh = 1 is not small
    relative to it) -- twice their sum."""
    W = workloads.normal((N, K), 0.02, 950 + K, wdt)
    W[0, :8] = torch.tensor([0.0, 1e-6, -0.05, 0.05, 0.2, -0.2, 0.01, -0.012]).to(wdt)  # both sides of |w/g| = 1
    X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, 951 + M, torch.bfloat16), 4, 20.0, 952)
    dY = workloads.normal((M, N), 1.0, 953 + N, torch.bfloat16)
    packed, gamma = api.bl_quant_weights(W.cuda())
    x_q, s = api.bl_quant_act(X.cuda())
    dW = api.bl_backward_dw(dY.cuda(), x_q, s, W.cuda(), gamma, beta)
    api.bl_check_device_error()
    g = gamma.cpu().numpy()[0]
    xq_np, s_np = x_q.cpu().numpy(), s.cpu().numpy()
    ref = oracle.bwd_dw(np32(dY), xq_np, s_np, np32(W), g, beta)
    mag = oracle.bwd_dw(np.abs(np32(dY)), np.abs(xq_np).astype(np.int8), s_np, np.zeros((N, K), np.float32), g, 0.0)
    err = np.abs(dW.cpu().numpy().astype(np.float64) - ref)
    lim = 2.0 * ((2.0 ** -8 + M * 2.0 ** -23) * mag + 2.0 ** -24 * np.abs(ref) + (2.0 ** -21 if beta > 0 else 0) * mag)
    assert np.all(err <= lim), f"max excess {(err - lim).max():.3e}"
    if beta <= 0:
        # the hard mask is decided exactly as the oracle decides it
        r = np32(W) / np.float32(g)
        assert np.all(dW.cpu().numpy()[np.abs(r) > 1] == 0)
