"""bl_quant_weights_noalloc: weight quantization for callers that cannot
allocate device memory (a plain C host, a runtime that only lends pointers to
tensors it owns, a fixed device-memory budget).  It runs the same kernels as
bl_quant_weights with the library's static device scratch instead of a
caller workspace, so its packed weights and gamma must equal
bl_quant_weights' bit for bit -- on two calls in a row, because the static
scratch keeps the previous call's contents -- and the CPU oracle's.

This file is collected last on purpose: it must pass alone in a fresh process
and after every other test."""
from __future__ import annotations

import pytest
import torch

import numpy as np

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        workloads.normal((2048, 768), 0.02, 41),                    # fp32, many blocks
        workloads.normal((37, 192), 0.015, 42, torch.bfloat16),     # bf16, ragged, few blocks
    ]
    for W_cpu in cases:
        W = W_cpu.cuda()
        ref_packed, ref_gamma = api.bl_quant_weights(W)
        for _ in range(2):  # second call sees the first call's leftover scratch
            packed, gamma = api.bl_quant_weights_noalloc(W)
            torch.cuda.synchronize()
            assert torch.equal(packed, ref_packed)
            assert gamma.view(torch.int32).item() == ref_gamma.view(torch.int32).item()
        # and directly against the CPU oracle, so the check stands on its own
        o_packed, o_gamma, _ = oracle.quant_weights(W_cpu.float().numpy())
        assert np.array_equal(packed.cpu().numpy(), o_packed)
        assert gamma.cpu().numpy().view(np.uint32)[0] == np.float32(o_gamma).view(np.uint32)


def test_noalloc_rejects_oversize_on_host():
    L = api.lib()
    A = 1 << 20
    assert L.bl_quant_weights_noalloc(A, 0, 1 << 17, 1 << 14, A, A, None) == 2  # N*K = 2^31: BL_ERR_SHAPE
    assert L.bl_quant_weights_noalloc(A, 0, 64, 100, A, A, None) == 2
