"""Full-size workloads on the GPU, checked against the oracle.

Weights, gamma: every byte.  x_q, s: every row for decode, sampled rows for
prefill.  acc and Y: every output for decode, 4096 sampled (m, n) pairs plus
corners for prefill.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_act, check_forward_full, check_forward_sampled, check_weights, np32

pytestmark = pytest.mark.gpu


def run_projection(W, X, gain=None, full=False, sample_rows=256, seed=0):
    Wd, Xd = W.cuda(), X.cuda()
    packed, gamma = api.bl_quant_weights(Wd)
    x_q, s = api.bl_quant_act(Xd, None if gain is None else gain.cuda(), workloads.SUBLN_EPS)
    M, N = X.shape[0], W.shape[0]
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    Y = api.bl_forward(packed, gamma, x_q, s, N, acc_out=acc)
    api.bl_check_device_error()
    wq_ref, g_ref = check_weights(W, packed, gamma)
    if full:
        xq_ref, s_ref = check_act(X, x_q, s, gain)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)
    else:
        rng = np.random.default_rng(seed)
        rows = np.unique(np.concatenate([rng.integers(0, M, sample_rows), [0, M - 1]]))
        xq_ref, s_ref = check_act(X, x_q, s, gain, rows=rows)
        check_forward_sampled(xq_ref, s_ref, wq_ref, g_ref, Y, acc, xq_rows=rows, seed=seed)
    return Y


@pytest.mark.parametrize("which", ["q", "k", "o", "gate", "down"])
def test_prefill1b4_layer(which):
    name, W, X = workloads.prefill1b4(which=(which,))[0]
    run_projection(W, X)


@pytest.mark.parametrize("M", [1, 2048])
def test_layer3b(M):
    for name, W, X in workloads.layer3b(M=M):
        run_projection(W, X, full=(M == 1))


@pytest.mark.parametrize("which", ["o", "gate", "down"])
def test_qat4b_layer(which):
    name, W, X, gain = workloads.qat4b(which=(which,))[0]
    Y = run_projection(W, X, gain)
    # the per-call path (weights re-quantized in the call, act quant overlapping
    # the weight pack, TMA-stored Y) gives the same bits
    Yl = api.bl_linear(W.cuda(), X.cuda(), None if gain is None else gain.cuda(), workloads.SUBLN_EPS)
    torch.cuda.synchronize()
    assert torch.equal(Yl.view(torch.int32), Y.view(torch.int32))


def test_single_workload_full():
    W, X = workloads.single()
    run_projection(W, X, full=True)
