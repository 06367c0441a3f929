"""The Python binding's argument checks, on CPU: every buffer handed to the
library must be a CUDA tensor, contiguous, of the right dtype and large
enough, so that no kernel touches host memory or runs past a caller's
buffer.  The library is replaced by a recorder (no GPU here); the device
check is relaxed only where a test says so, to drive the valid paths."""
from __future__ import annotations

import pytest
import torch

from ternary_quantized_linear_bitlinear_b200 import api


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes"):
            return lambda *a: 4096
        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(api, "lib", lambda: lib)
    monkeypatch.setattr(api, "_stream", lambda stream: 0)
    monkeypatch.setattr(api, "_is_cuda", lambda t: True)  # CPU tensors stand in for device buffers
    return lib


def test_cpu_tensors_are_rejected_before_the_library():
    W = torch.zeros(64, 128)
    with pytest.raises(ValueError, match="CUDA"):
        api.bl_quant_weights(W)
    with pytest.raises(ValueError, match="CUDA"):
        api.bl_quant_act(torch.zeros(4, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        api.bl_forward(torch.zeros(64, 32, dtype=torch.uint8), torch.zeros(1), torch.zeros(4, 128, dtype=torch.int8),
                       torch.zeros(4), 64)


def test_valid_calls_reach_the_library(fake):
    M, N, K = 4, 64, 128
    W = torch.zeros(N, K)
    packed, gamma = api.bl_quant_weights(W)
    x_q, s = api.bl_quant_act(torch.zeros(M, K, dtype=torch.bfloat16), torch.ones(K), 1e-6)
    acc = torch.zeros(M, N, dtype=torch.int32)
    Y = api.bl_forward(packed, gamma, x_q, s, N, acc_out=acc)
    assert Y.shape == (M, N) and Y.dtype == torch.float32
    api.bl_linear(W, torch.zeros(M, K, dtype=torch.bfloat16))
    api.bl_ffn_act_quant(torch.zeros(M, K), torch.zeros(M, K), torch.ones(K))
    names = [c[0] for c in fake.calls]
    assert names == ["bl_quant_weights", "bl_quant_act", "bl_forward", "bl_linear", "bl_ffn_act_quant"]


@pytest.mark.parametrize("bad", ["packed_dtype", "packed_small", "gamma_dtype", "s_small", "Y_small", "acc_dtype",
                                 "x_q_dtype", "noncontig"])
def test_bad_forward_buffers_are_rejected(fake, bad):
    M, N, K = 4, 64, 128
    packed = torch.zeros(N, K // 4, dtype=torch.uint8)
    gamma = torch.zeros(1)
    x_q = torch.zeros(M, K, dtype=torch.int8)
    s = torch.zeros(M)
    Y = torch.zeros(M, N)
    acc = torch.zeros(M, N, dtype=torch.int32)
    if bad == "packed_dtype":
        packed = packed.to(torch.int8)
    elif bad == "packed_small":
        packed = packed[: N // 2]
    elif bad == "gamma_dtype":
        gamma = gamma.double()
    elif bad == "s_small":
        s = s[: M - 1]
    elif bad == "Y_small":
        Y = Y[: M - 1]
    elif bad == "acc_dtype":
        acc = acc.to(torch.int64)
    elif bad == "x_q_dtype":
        x_q = x_q.to(torch.uint8)
    elif bad == "noncontig":
        Y = torch.zeros(N, M).t()
    with pytest.raises(ValueError):
        api.bl_forward(packed, gamma, x_q, s, N, Y=Y, acc_out=acc)
    assert fake.calls == []


def test_bad_quant_buffers_are_rejected(fake):
    M, N, K = 4, 64, 128
    with pytest.raises(ValueError):
        api.bl_quant_weights(torch.zeros(N, K), packed=torch.zeros(N, K // 8, dtype=torch.uint8))
    with pytest.raises(ValueError):
        api.bl_quant_weights(torch.zeros(N, K), workspace=torch.zeros(4096, dtype=torch.float32))
    with pytest.raises(ValueError):
        api.bl_quant_act(torch.zeros(M, K), x_q=torch.zeros(M, K, dtype=torch.uint8))
    with pytest.raises(ValueError):
        api.bl_quant_act(torch.zeros(M, K), subln_gain=torch.ones(K // 2))
    with pytest.raises(ValueError):
        api.bl_ffn_act_quant(torch.zeros(M, K), torch.zeros(M, K), torch.ones(K, dtype=torch.float64))
    with pytest.raises(ValueError):
        api.bl_quant_act_grouped([(torch.zeros(M, K), None, torch.zeros(M, K, dtype=torch.int8), torch.zeros(M))],
                                 dtype=torch.bfloat16)  # X is f32, the call says bf16
    with pytest.raises(TypeError):
        api.make_problems([(1, 2, 3, 4, 5, None, N, K)])  # raw integers are not device buffers
    assert fake.calls == []
