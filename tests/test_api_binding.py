"""The Python binding's argument checks, on CPU: every buffer handed to the
library must be a CUDA tensor on the current device, contiguous, of the
right dtype and large enough, so that no kernel touches host memory or
another GPU's memory, or runs past a caller's buffer.  The library is
replaced by a recorder (no GPU here); the device check is relaxed only where
a test says so, to drive the valid paths."""
from __future__ import annotations

import pytest
import torch

from ternary_quantized_linear_bitlinear_b200 import api

_REAL_STREAM = api._stream  # the fixture below replaces it with a stub

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
    monkeypatch.setattr(api, "_device_index", lambda t: 0)
    monkeypatch.setattr(api, "_current_device", lambda: 0)
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


def test_mismatched_or_bad_inputs_are_rejected(fake):
    M, N, K = 4, 64, 128
    W = torch.zeros(N, K)
    with pytest.raises(ValueError, match="columns"):
        api.bl_linear(W, torch.zeros(M, K - 64, dtype=torch.bfloat16))  # X narrower than W's K
    with pytest.raises(ValueError, match="2-D"):
        api.bl_linear(W, torch.zeros(M * K, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="float32 or bfloat16"):
        api.bl_linear(W.double(), torch.zeros(M, K))
    with pytest.raises(ValueError, match="float32 or bfloat16"):
        api.bl_quant_act(torch.zeros(M, K, dtype=torch.float16))
    with pytest.raises(ValueError, match="float32 or bfloat16"):
        api.bl_quant_weights(torch.zeros(N, K, dtype=torch.int8))
    with pytest.raises(ValueError, match="2-D"):
        api.bl_forward(torch.zeros(N, K // 4, dtype=torch.uint8), torch.zeros(1),
                       torch.zeros(M * K, dtype=torch.int8), torch.zeros(M), N)
    assert fake.calls == []


def test_buffers_on_another_device_are_rejected(fake, monkeypatch):
    # the library launches on the current device: a buffer (or a stream) of
    # another GPU must not reach it
    monkeypatch.setattr(api, "_current_device", lambda: 1)
    with pytest.raises(ValueError, match="cuda:0"):
        api.bl_quant_weights(torch.zeros(64, 128))

    class _Stream:
        device_index = 0
        cuda_stream = 0

    with pytest.raises(ValueError, match="stream"):
        _REAL_STREAM(_Stream())
    assert fake.calls == []


def _grouped_items(M, N, K, **bad):
    t = dict(packed=torch.zeros(N, K // 4, dtype=torch.uint8), gamma=torch.zeros(1),
             x_q=torch.zeros(M, K, dtype=torch.int8), s=torch.zeros(M), Y=torch.zeros(M, N),
             acc=torch.zeros(M, N, dtype=torch.int32))
    t.update(bad)
    return [(t["packed"], t["gamma"], t["x_q"], t["s"], t["Y"], t["acc"], N, K)]


@pytest.mark.parametrize("bad", ["packed_small", "gamma_dtype", "x_q_small", "s_small", "Y_small", "acc_dtype"])
def test_grouped_forward_buffers_are_checked(fake, bad):
    M, N, K = 4, 64, 128
    repl = {"packed_small": dict(packed=torch.zeros(N // 2, K // 4, dtype=torch.uint8)),
            "gamma_dtype": dict(gamma=torch.zeros(1, dtype=torch.float64)),
            "x_q_small": dict(x_q=torch.zeros(M * K - 16, dtype=torch.int8)),
            "s_small": dict(s=torch.zeros(M - 1)),
            "Y_small": dict(Y=torch.zeros(M * N - 1)),
            "acc_dtype": dict(acc=torch.zeros(M, N))}[bad]
    with pytest.raises(ValueError):
        api.make_problems(_grouped_items(M, N, K, **repl), M=M)
    assert fake.calls == []


def test_grouped_arrays_are_launched_only_as_checked(fake):
    M, N, K = 4, 64, 128
    arr = api.make_problems(_grouped_items(M, N, K))
    api.bl_forward_grouped(arr, 1, M)
    with pytest.raises(ValueError, match="M = 4"):
        api.bl_forward_grouped(arr, 1, 8)  # a larger M would run past x_q, s and Y
    with pytest.raises(ValueError, match="count"):
        api.bl_forward_grouped(arr, 2, M)
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    items = [(torch.zeros(N, K // 4, dtype=torch.uint8), torch.zeros(1), X, None, torch.zeros(M, N), None, None,
              None, N, K)]
    darr = api.make_decode_problems(items)
    api.bl_linear_decode_grouped(darr, 1, M, torch.bfloat16)
    with pytest.raises(ValueError, match="checked for X"):
        api.bl_linear_decode_grouped(darr, 1, M, torch.float32)
    with pytest.raises(ValueError):  # Y too small for M x N
        api.make_decode_problems([items[0][:4] + (torch.zeros(M, N - 1),) + items[0][5:]])
    with pytest.raises(ValueError):  # a second X of another dtype
        api.make_decode_problems(items + [items[0][:2] + (X.float(),) + items[0][3:]])
    assert [c[0] for c in fake.calls] == ["bl_forward_grouped", "bl_linear_decode_grouped"]
