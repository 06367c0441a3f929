"""The C ABI without a GPU: the library loads, exports every function that
include/bitlinear.h declares, and rejects bad arguments on the host before
touching the device (validation pattern: "bitone" README, Security --
ndim / dtype / contiguity / bounds / null checks at the binding boundary)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from ternary_quantized_linear_bitlinear_b200 import api, build

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")

OK, NULL, SHAPE, ALIGN, DTYPE, CUDA, TIMEOUT, WORKSPACE, DEVICE = range(9)
A = 1 << 20  # a fake, 16-byte aligned "device address" (never dereferenced)


@pytest.fixture(scope="module")
def L():
    build.build()
    return api.lib()


def declared_functions():
    names = set()
    for h in sorted(os.listdir(INCLUDE)):
        if h.endswith(".h"):
            text = open(os.path.join(INCLUDE, h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(bl_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(api.EXPORTED)


def test_status_strings_and_version(L):
    for s in range(9):
        assert api.status_string(s).startswith("BL_")
    assert api.status_string(99) == "BL_ERR_UNKNOWN"
    assert L.bl_version() == 100


def test_workspace_queries(L):
    assert L.bl_quant_weights_workspace_bytes(2048, 768) >= 49152
    M, N, K = 16, 2048, 768
    ws = L.bl_linear_workspace_bytes(M, N, K)
    assert ws >= L.bl_quant_weights_workspace_bytes(N, K) + N * K // 4 + M * K + 4 * M
    assert L.bl_linear_workspace_bytes(0, N, K) == 0


def qw(L, W=A, wdt=0, N=64, K=128, packed=A, gamma=A, ws=A, wsb=1 << 20):
    return L.bl_quant_weights(W, wdt, N, K, packed, gamma, ws, wsb, None)


def test_quant_weights_validation(L):
    assert qw(L, W=None) == NULL
    assert qw(L, packed=None) == NULL
    assert qw(L, gamma=None) == NULL
    assert qw(L, wdt=7) == DTYPE
    assert qw(L, K=100) == SHAPE
    assert qw(L, K=0) == SHAPE
    assert qw(L, K=32768 + 64) == SHAPE
    assert qw(L, N=0) == SHAPE
    assert qw(L, N=1 << 17, K=1 << 14) == SHAPE  # N*K = 2^31
    assert qw(L, W=A + 8) == ALIGN
    assert qw(L, packed=A + 4) == ALIGN
    assert qw(L, ws=None) == WORKSPACE
    assert qw(L, wsb=16) == WORKSPACE
    # valid arguments reach the device query, which fails without a GPU
    assert qw(L) in (CUDA, DEVICE)


def test_quant_act_validation(L):
    f = L.bl_quant_act
    assert f(None, 0, 4, 128, None, 1e-6, A, A, None) == NULL
    assert f(A, 0, 4, 128, None, 1e-6, None, A, None) == NULL
    assert f(A, 2, 4, 128, None, 1e-6, A, A, None) == DTYPE
    assert f(A, 0, 0, 128, None, 1e-6, A, A, None) == SHAPE
    assert f(A, 0, 4, 96, None, 1e-6, A, A, None) == SHAPE
    assert f(A, 0, 4, 128, A + 4, 1e-6, A, A, None) == ALIGN
    assert f(A, 1, 4, 128, None, 1e-6, A, A, None) in (CUDA, DEVICE)


def test_forward_validation(L):
    f = L.bl_forward
    assert f(None, A, A, A, 1, 64, 128, A, None, None) == NULL
    assert f(A, A, A, A, 1, 64, 128, None, None, None) == NULL
    assert f(A, A, A, A, 0, 64, 128, A, None, None) == SHAPE
    assert f(A, A, A, A, 1, 0, 128, A, None, None) == SHAPE
    assert f(A, A, A, A, 1, 64, 130, A, None, None) == SHAPE
    assert f(A, A, A, A, 1, 64, 128, A + 1, None, None) == ALIGN
    assert f(A, A, A, A, 1, 64, 128, A, A + 2, None) == ALIGN
    assert f(A, A, A, A, 1, 64, 128, A, None, None) in (CUDA, DEVICE)


def test_linear_validation(L):
    f = L.bl_linear
    wsb = L.bl_linear_workspace_bytes(8, 64, 128)
    assert f(None, 0, A, 0, 8, 64, 128, None, 1e-6, A, wsb, A, None) == NULL
    assert f(A, 3, A, 0, 8, 64, 128, None, 1e-6, A, wsb, A, None) == DTYPE
    assert f(A, 0, A, 3, 8, 64, 128, None, 1e-6, A, wsb, A, None) == DTYPE
    assert f(A, 0, A, 0, 8, 64, 127, None, 1e-6, A, wsb, A, None) == SHAPE
    assert f(A, 0, A, 0, 8, 64, 128, None, 1e-6, A, wsb - 1, A, None) == WORKSPACE
    assert f(A, 0, A, 0, 8, 64, 128, None, 1e-6, A + 8, wsb, A, None) == ALIGN
    assert f(A, 0, A, 0, 8, 64, 128, None, 1e-6, A, wsb, A, None) in (CUDA, DEVICE)


def test_grouped_validation(L):
    P = (api.Problem * 2)()
    for i in range(2):
        P[i] = api.Problem(A, A, A, A, A, None, 64, 128)
    def g(arr, count, M):
        return L.bl_forward_grouped(arr, count, M, 0, None)
    assert g(None, 1, 1) == NULL
    assert g(P, 0, 1) == SHAPE
    assert g(P, api.BL_MAX_GROUP + 1, 1) == SHAPE
    P[1].K = 100
    assert g(P, 2, 1) == SHAPE
    P[1].K = 128
    P[1].Y = None
    assert g(P, 2, 1) == NULL
    P[1].Y = A
    assert g(P, 2, 1) in (CUDA, DEVICE)
    # prefill-sized groups share x_q, s and K, at most BL_MAX_PREFILL_GROUP of them
    R = (api.Problem * 5)()
    for i in range(5):
        R[i] = api.Problem(A, A, A, A, A, None, 64, 128)
    assert g(R, 5, 100) == SHAPE
    assert g(R, 4, 100) in (CUDA, DEVICE)
    R[1].x_q = A + 16
    assert g(R, 2, 100) == SHAPE
    R[1].x_q = A
    R[1].K = 256
    assert g(R, 2, 100) == SHAPE
    Q = (api.ActProblem * 1)()
    Q[0] = api.ActProblem(A, None, A, A, 128)
    assert L.bl_quant_act_grouped(Q, 1, 5, 1, 1e-6, None) == DTYPE
    assert L.bl_quant_act_grouped(Q, 1, 1, 1, 1e-6, None) in (CUDA, DEVICE)


def test_fused_decode_validation(L):
    P = (api.DecodeProblem * 2)()
    for i in range(2):
        P[i] = api.DecodeProblem(A, A, A, None, A, None, None, None, 64, 128)
    def g(arr, count, M, dt=1):
        return L.bl_linear_decode_grouped(arr, count, dt, M, 1e-6, 0, None)
    assert g(None, 1, 1) == NULL
    assert g(P, 0, 1) == SHAPE
    assert g(P, api.BL_MAX_GROUP + 1, 1) == SHAPE
    assert g(P, 2, 17) == SHAPE
    assert g(P, 2, 1, dt=4) == DTYPE
    P[1].X = None
    assert g(P, 2, 1) == NULL
    P[1].X = A
    P[1].K = 96
    assert g(P, 2, 1) == SHAPE
    P[1].K = 32768
    assert g(P, 2, 16) == SHAPE  # x_q staging of 16 rows of 32768 does not fit
    P[1].K = 128
    for field in ("subln_gain", "x_q", "s", "acc_out", "Y"):
        setattr(P[1], field, A + 4)
        assert g(P, 2, 1) == ALIGN, field
        setattr(P[1], field, A if field == "Y" else None)
    assert g(P, 2, 1) in (CUDA, DEVICE)


def test_ffn_act_quant_validation(L):
    f = L.bl_ffn_act_quant
    assert f(None, A, 4, 128, None, 1e-6, A, A, None) == NULL
    assert f(A, None, 4, 128, None, 1e-6, A, A, None) == NULL
    assert f(A, A, 4, 128, None, 1e-6, None, A, None) == NULL
    assert f(A, A, 0, 128, None, 1e-6, A, A, None) == SHAPE
    assert f(A, A, 4, 100, None, 1e-6, A, A, None) == SHAPE
    assert f(A, A + 4, 4, 128, None, 1e-6, A, A, None) == ALIGN
    assert f(A, A, 4, 128, A + 8, 1e-6, A, A, None) == ALIGN
    assert f(A, A, 4, 128, None, 1e-6, A, A, None) in (CUDA, DEVICE)


def test_debug_prefill_validation(L):
    f = L.bl_debug_forward_prefill
    assert f(None, A, A, A, 1, 64, 128, A, None, -1, 1000, None) == NULL
    assert f(A, A, A, A, 1, 64, 100, A, None, -1, 1000, None) == SHAPE
    assert f(A, A, A, A, 1, 64, 128, A, None, -1, 0, None) == SHAPE
    assert f(A, A, A, A, 1, 64, 128, A + 4, None, -1, 1000, None) == ALIGN
    assert f(A, A, A, A, 1, 64, 128, A, None, 0, 1000, None) in (CUDA, DEVICE)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_LIB", None)
    monkeypatch.setattr(build, "LIB", str(tmp_path / "libbitlinear.so"))
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_grouped_weight_quant_validation(L):
    def call(count=1, wdt=0, ws=A, wsb=1 << 20, **kw):
        p = dict(W=A, N=64, K=128, packed=A, gamma=A)
        p.update(kw)
        arr = (api.WeightProblem * 8)()
        for i in range(8):
            arr[i] = api.WeightProblem(p["W"], p["N"], p["K"], p["packed"], p["gamma"])
        return L.bl_quant_weights_grouped(arr, count, wdt, ws, wsb, None)

    assert L.bl_quant_weights_grouped(None, 1, 0, A, 1 << 20, None) == NULL
    assert call(count=0) == SHAPE
    assert call(count=9) == SHAPE
    assert call(wdt=3) == DTYPE
    assert call(W=None) == NULL
    assert call(gamma=None) == NULL
    assert call(K=96) == SHAPE
    assert call(N=1 << 17, K=1 << 14) == SHAPE
    assert call(packed=A + 8) == ALIGN
    assert call(ws=None) == WORKSPACE
    assert call(wsb=100) == WORKSPACE
    assert call(count=8) in (CUDA, DEVICE)


def test_grouped_linear_validation_and_workspace(L):
    M, K = 64, 768
    arr = (api.LinearProblem * 4)()
    for i, N in enumerate((768, 256, 256, 2048)):
        arr[i] = api.LinearProblem(A, A, N)
    ws = L.bl_linear_grouped_workspace_bytes(arr, 3, M, K)
    assert ws >= L.bl_quant_weights_workspace_bytes(1, 64) + (768 + 256 + 256) * K // 4 + M * K + 4 * M
    assert L.bl_linear_grouped_workspace_bytes(arr, 5, M, K) == 0

    def call(count=3, wdt=1, X=A, xdt=1, M=M, K=K, gain=None, wsp=A, wsb=ws):
        return L.bl_linear_grouped(arr, count, wdt, X, xdt, M, K, gain, 1e-6, wsp, wsb, None)

    assert call(X=None) == NULL
    assert call(count=5) == SHAPE
    assert call(wdt=2) == DTYPE
    assert call(xdt=2) == DTYPE
    assert call(K=100) == SHAPE
    assert call(M=0) == SHAPE
    assert call(X=A + 4) == ALIGN
    assert call(gain=A + 4) == ALIGN
    assert call(wsb=ws - 1) == WORKSPACE
    assert call() in (CUDA, DEVICE)


def test_backward_and_gated_validation(L):
    def bdx(dY=A, packed=A, gamma=A, M=64, N=128, K=256, dX=A):
        return L.bl_backward_dx(dY, packed, gamma, M, N, K, dX, None)

    assert bdx(dY=None) == NULL
    assert bdx(dX=None) == NULL
    assert bdx(N=12) == SHAPE       # dY rows must be multiples of 16 bytes
    assert bdx(K=100) == SHAPE
    assert bdx(M=0) == SHAPE
    assert bdx(dY=A + 8) == ALIGN
    assert bdx() in (CUDA, DEVICE)

    def glu(pg=A, gg=A, pu=A, gu=A, xq=A, s=A, M=64, F=256, K=256, h=A):
        return L.bl_forward_glu(pg, gg, pu, gu, xq, s, M, F, K, h, None)

    assert glu(pu=None) == NULL
    assert glu(F=100) == SHAPE      # F is the down projection's K: a multiple of 64
    assert glu(K=96) == SHAPE
    assert glu(h=A + 4) == ALIGN
    assert glu() in (CUDA, DEVICE)


def test_weight_gradient_validation(L):
    M, N, K = 300, 256, 512
    ws = L.bl_backward_dw_workspace_bytes(M, N, K)
    assert ws >= 2 * (N + K) * 320  # dY^T and (x_q / s)^T in bf16 over 320 padded tokens
    assert L.bl_backward_dw_workspace_bytes(0, N, K) == 0

    def dw(dY=A, xq=A, s=A, W=A, wdt=0, g=A, M=M, N=N, K=K, wsp=A, wsb=ws, out=A):
        return L.bl_backward_dw(dY, xq, s, W, wdt, g, 2.0, M, N, K, wsp, wsb, out, None)

    assert dw(dY=None) == NULL
    assert dw(out=None) == NULL
    assert dw(wdt=5) == DTYPE
    assert dw(K=100) == SHAPE
    assert dw(N=0) == SHAPE
    assert dw(xq=A + 2) == ALIGN
    assert dw(wsb=ws - 1) == WORKSPACE
    assert dw() in (CUDA, DEVICE)
