"""The down projection's input from the gate / up projection outputs
(bl_ffn_act_quant: h = relu(gate)^2 * up, optional SubLN, absmax INT8) vs
the CPU oracle on the same seeded float32 inputs: x_q and s bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import np32

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


def test_ffn_act_quant_1b4_shapes_sampled_rows():
    """The 1.4B layer's FFN (M = 8192, F = 4096) in one call, checked on a
    sample of rows (the oracle runs row by row)."""
    M, F = 8192, 4096
    gate = workloads.normal((M, F), 1.5, 50)
    up = workloads.student_t((M, F), 3, 0.5, 51, torch.float32)
    gain = workloads.uniform((F,), 0.9, 1.1, 52)
    x_q, s = api.bl_ffn_act_quant(gate.cuda(), up.cuda(), gain.cuda(), 1e-6)
    torch.cuda.synchronize()
    rows = np.random.default_rng(3).choice(M, 64, replace=False)
    rows.sort()
    ref_xq, ref_s = oracle.ffn_act_quant(np32(gate[rows]), np32(up[rows]), np32(gain), 1e-6)
    assert np.array_equal(s.cpu().numpy()[rows].view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(x_q.cpu().numpy()[rows], ref_xq)
