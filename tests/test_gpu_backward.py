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
