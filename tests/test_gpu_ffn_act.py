"""The down projection's input from the gate / up projection outputs
(bl_ffn_act_quant: h = relu(gate)^2 * up, optional SubLN, absmax INT8) vs
the CPU oracle on the same seeded float32 inputs: x_q and s bit for bit;
and the gated forward (bl_forward_glu) that forms h in the GEMM epilogue."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_y, np32

pytestmark = pytest.mark.gpu


def _check(gate, up, gain, x_q, s, eps=1e-6):
    ref_xq, ref_s = oracle.ffn_act_quant(np32(gate), np32(up), None if gain is None else np32(gain), eps)
    got_s = s.cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32)), "s mismatch"
    got = x_q.cpu().numpy()
    if not np.array_equal(got, ref_xq):
        bad = np.argwhere(got != ref_xq)
        raise AssertionError(f"x_q mismatch at {len(bad)} entries, first {bad[:5].tolist()}")


@pytest.mark.parametrize("M,F,subln", [
    (1, 4096, True), (7, 1536, False), (300, 4096, True), (33, 64, False), (5, 9728, True), (2, 32768, False),
    (64, 2048, False), (3, 8640, True), (2, 32768, True),
])
def test_ffn_act_quant_matches_oracle(M, F, subln):
    gate = workloads.normal((M, F), 2.0, 40 + F)
    up = workloads.normal((M, F), 1.0, 41 + M)
    gate[0, : F // 2] = -gate[0, : F // 2].abs()   # a half-negative gate row
    if M > 2:
        gate[2] = -1.0                               # relu kills the whole row: h = 0
    gain = workloads.uniform((F,), 0.9, 1.1, 42) if subln else None
    x_q, s = api.bl_ffn_act_quant(gate.cuda(), up.cuda(), None if gain is None else gain.cuda(), 1e-6)
    torch.cuda.synchronize()
    _check(gate, up, gain, x_q, s)


def test_ffn_act_quant_1b4_shapes_every_row():
    """The 1.4B layer's FFN (M = 8192, F = 4096) in one call, every row."""
    M, F = 8192, 4096
    gate = workloads.normal((M, F), 1.5, 50)
    up = workloads.student_t((M, F), 3, 0.5, 51, torch.float32)
    gain = workloads.uniform((F,), 0.9, 1.1, 52)
    x_q, s = api.bl_ffn_act_quant(gate.cuda(), up.cuda(), gain.cuda(), 1e-6)
    torch.cuda.synchronize()
    _check(gate, up, gain, x_q, s)


@pytest.mark.parametrize("M,F,K", [(300, 4096, 1536), (8192, 4096, 1536), (40, 64, 192), (513, 320, 768)])
def test_forward_glu_matches_the_gate_and_up_outputs(M, F, K):
    """bl_forward_glu (gate and up in one launch, only h stored) against the
    oracle's FFN activation of the plain engine's gate and up outputs (bit
    for bit: the same float operations on the same floats), those outputs
    against the oracle's exact accumulators, and the down projection's
    input quantized from h against the oracle's FFN act quant."""
    Wg = workloads.normal((F, K), 0.02, 60 + F, torch.bfloat16)
    Wu = workloads.normal((F, K), 0.02, 61 + F, torch.bfloat16)
    X = workloads.student_t((M, K), 3, 0.5, 62 + M, torch.bfloat16)
    gain = workloads.uniform((F,), 0.9, 1.1, 63)
    pg, gg = api.bl_quant_weights(Wg.cuda())
    pu, gu = api.bl_quant_weights(Wu.cuda())
    x_q, s = api.bl_quant_act(X.cuda())
    h = api.bl_forward_glu(pg, gg, pu, gu, x_q, s, F)
    Yg = api.bl_forward(pg, gg, x_q, s, F)
    Yu = api.bl_forward(pu, gu, x_q, s, F)
    hq, hs = api.bl_quant_act(h, gain.cuda(), 1e-6)
    api.bl_check_device_error()
    h_ref = oracle.ffn_act(np32(Yg), np32(Yu))
    got = h.cpu().numpy()
    if not np.array_equal(got.view(np.uint32), h_ref.view(np.uint32)):
        bad = np.argwhere(got.view(np.uint32) != h_ref.view(np.uint32))
        raise AssertionError(f"h differs at {len(bad)} entries, first {bad[:5].tolist()}")
    xq_ref, s_ref = oracle.quant_act(np32(X))
    for W, g, Y in ((Wg, gg, Yg), (Wu, gu, Yu)):
        _, g_ref, wq_ref = oracle.quant_weights(np32(W))
        assert g.cpu().numpy()[0] == g_ref
        check_y(Y.cpu().numpy(), oracle.contract_blas(xq_ref, wq_ref), g_ref, s_ref[:, None])
    _check(Yg.cpu(), Yu.cpu(), gain, hq, hs)
