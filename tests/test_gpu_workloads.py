"""Full-size workloads on the GPU, checked against the oracle element by
element: every packed weight byte and gamma, every row of x_q and s, every
int32 accumulator and every Y of each projection run (the accumulators from
the oracle's exact contraction, its BLAS form at these sizes).

Each projection runs twice through the contraction: once with the int32
accumulators requested (plain stores in the prefill epilogue) and once
without (Y by TMA tensor stores); both Y must carry the same bits.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_act, check_weights, check_y

pytestmark = pytest.mark.gpu


def check_acc_full(acc_got: torch.Tensor, acc_ref: np.ndarray):
    got = acc_got.cpu().numpy()
    if not np.array_equal(got, acc_ref):
        bad = np.argwhere(got != acc_ref)
        raise AssertionError(f"acc mismatch at {len(bad)} of {acc_ref.size} entries, first {bad[:5].tolist()}")


def run_projection(W, X, gain=None):
    Wd, Xd = W.cuda(), X.cuda()
    packed, gamma = api.bl_quant_weights(Wd)
    x_q, s = api.bl_quant_act(Xd, None if gain is None else gain.cuda(), workloads.SUBLN_EPS)
    M, N = X.shape[0], W.shape[0]
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    Y = api.bl_forward(packed, gamma, x_q, s, N, acc_out=acc)
    Y2 = api.bl_forward(packed, gamma, x_q, s, N)
    api.bl_check_device_error()
    assert torch.equal(Y.view(torch.int32), Y2.view(torch.int32)), "Y differs between the two store paths"
    del Y2
    wq_ref, g_ref = check_weights(W, packed, gamma)
    xq_ref, s_ref = check_act(X, x_q, s, gain)
    acc_ref = oracle.contract_blas(xq_ref, wq_ref)
    check_acc_full(acc, acc_ref)
    check_y(Y.cpu().numpy(), acc_ref, g_ref, s_ref[:, None])
    return Y


@pytest.mark.parametrize("which", ["q", "k", "v", "o", "gate", "up", "down"])
def test_prefill1b4_layer(which):
    name, W, X = workloads.prefill1b4(which=(which,))[0]
    run_projection(W, X)


@pytest.mark.parametrize("M", [1, 2048])
def test_layer3b(M):
    for name, W, X in workloads.layer3b(M=M):
        run_projection(W, X)


@pytest.mark.parametrize("which", ["o", "gate", "down"])
def test_qat4b_layer(which):
    name, W, X, gain = workloads.qat4b(which=(which,))[0]
    Y = run_projection(W, X, gain)
    # the per-call path (weights re-quantized in the call, act quant overlapping
    # the weight pack, TMA-stored Y) gives the same bits
    Yl = api.bl_linear(W.cuda(), X.cuda(), None if gain is None else gain.cuda(), workloads.SUBLN_EPS)
    torch.cuda.synchronize()
    assert torch.equal(Yl.view(torch.int32), Y.view(torch.int32))


def test_prefill_every_pair_runs_several_tiles():
    """M = 4096, N = 4096, K = 768: 16 x 16 = 256 output tiles of 256 x 256 on
    at most 74 CTA pairs, so every pair runs 3 or 4 tiles: both TMEM
    accumulator buffers and their phase flips are used, every output checked."""
    W = workloads.normal((4096, 768), 0.02, 501)
    X = workloads.with_outlier_channels(workloads.normal((4096, 768), 1.0, 502, torch.bfloat16), 8, 20.0, 503)
    run_projection(W, X)


def test_single_workload_full():
    W, X = workloads.single()
    run_projection(W, X)
