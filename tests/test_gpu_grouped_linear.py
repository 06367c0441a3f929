"""Grouped per-call path against the CPU oracle.

bl_quant_weights_grouped: one reduction grid and one pack grid over several
matrices; every packed byte and every gamma must equal the oracle's (and so
what bl_quant_weights gives one matrix at a time).

bl_linear_grouped: the q, k, v (or gate, up) projections of a layer sharing
one input, every weight re-quantized in the call: each Y must carry the bits
of bl_linear on that projection alone, and be within 1e-6 of the oracle's
double rescale of its exact accumulators.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_weights, check_y, np32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grouped_weight_quant_matches_oracle(dtype):
    shapes = [(1536, 1536), (512, 1536), (37, 192), (4096, 1536), (1, 64), (2560, 9728), (300, 832), (64, 64)]
    Ws = [workloads.normal(sh, 0.02 + 0.001 * i, 1400 + i, dtype) for i, sh in enumerate(shapes)]
    # one matrix with a wide magnitude range (its blocks take the exact bins)
    Ws[2] = (Ws[2].float() * torch.pow(2.0, torch.arange(37 * 192).reshape(37, 192) % 60 - 40.0)).to(dtype)
    packed, gammas = api.bl_quant_weights_grouped([W.cuda() for W in Ws])
    torch.cuda.synchronize()
    for W, p, g in zip(Ws, packed, gammas):
        check_weights(W, p, g)
    # a second call on the same workspace (nothing in it needs clearing)
    packed2, gammas2 = api.bl_quant_weights_grouped([W.cuda() for W in Ws[:3]])
    torch.cuda.synchronize()
    for p, q in zip(packed[:3], packed2):
        assert torch.equal(p, q)


@pytest.mark.parametrize("M,which,subln", [
    (2048, ("q", "k", "v"), False),    # prefill engine, three matrices in one GEMM launch
    (300, ("gate", "up"), True),       # ragged M, SubLN
    (4, ("q", "k", "v"), False),       # decode engine, fused act quant
    (1, ("gate", "up"), True),
])
def test_grouped_linear_matches_single_calls_and_oracle(M, which, subln):
    items = workloads.prefill1b4(which=which, M=M)
    K = items[0][1].shape[1]
    X = items[0][2]  # the projections of a group share their input
    gain = workloads.uniform((K,), 0.9, 1.1, 1500) if subln else None
    Ws = [W for _, W, _ in items]
    Xd = X.cuda()
    gd = None if gain is None else gain.cuda()
    Ys = api.bl_linear_grouped([W.cuda() for W in Ws], Xd, gd, workloads.SUBLN_EPS)
    singles = [api.bl_linear(W.cuda(), Xd, gd, workloads.SUBLN_EPS) for W in Ws]
    api.bl_check_device_error()
    xq_ref, s_ref = oracle.quant_act(np32(X), None if gain is None else np32(gain), workloads.SUBLN_EPS)
    for W, Y, Y1 in zip(Ws, Ys, singles):
        assert torch.equal(Y.view(torch.int32), Y1.view(torch.int32))
        _, g_ref, wq_ref = oracle.quant_weights(np32(W))
        acc_ref = oracle.contract_blas(xq_ref, wq_ref)
        check_y(Y.cpu().numpy(), acc_ref, g_ref, s_ref[:, None])
