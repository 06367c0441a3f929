"""Shared helpers for the GPU-vs-oracle parity tests.

The oracle side always starts from the seeded CPU inputs; nothing the GPU
produces is ever fed to the oracle.  Integer results (packed bytes, gamma,
x_q, s, acc) must match bit for bit; Y must satisfy
|Y - Y_ref| <= 1e-6 * |Y_ref| elementwise (Y_ref in double from the exact
accumulator).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api

Y_RTOL = 1e-6


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def gpu_quant_weights(W_cpu: torch.Tensor):
    W = W_cpu.cuda()
    packed, gamma = api.bl_quant_weights(W)
    torch.cuda.synchronize()
    return packed, gamma


def check_weights(W_cpu: torch.Tensor, packed, gamma):
    ref_packed, ref_gamma, ref_wq = oracle.quant_weights(np32(W_cpu))
    g = gamma.cpu().numpy()[0]
    assert g.view(np.uint32) == np.float32(ref_gamma).view(np.uint32), (g, ref_gamma)
    got = packed.cpu().numpy()
    if not np.array_equal(got, ref_packed):
        bad = np.argwhere(got != ref_packed)
        raise AssertionError(f"packed mismatch at {len(bad)} bytes, first {bad[:5].tolist()}")
    return ref_wq, ref_gamma


def check_act(X_cpu: torch.Tensor, x_q, s, gain_cpu=None, eps=1e-6, rows=None):
    Xn = np32(X_cpu if rows is None else X_cpu[torch.as_tensor(rows)])
    ref_xq, ref_s = oracle.quant_act(Xn, None if gain_cpu is None else np32(gain_cpu), eps)
    got_s = s.cpu().numpy()
    got_xq = x_q.cpu().numpy()
    if rows is not None:
        got_s, got_xq = got_s[rows], got_xq[rows]
    assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32)), "s mismatch"
    if not np.array_equal(got_xq, ref_xq):
        bad = np.argwhere(got_xq != ref_xq)
        raise AssertionError(f"x_q mismatch at {len(bad)} entries, first {bad[:5].tolist()}")
    return ref_xq, ref_s


def check_y(Y_got: np.ndarray, acc_ref: np.ndarray, gamma, s_rows: np.ndarray):
    Y_ref = oracle.rescale(acc_ref, gamma, s_rows)
    err = np.abs(Y_got.astype(np.float64) - Y_ref)
    lim = Y_RTOL * np.abs(Y_ref)
    assert np.all(err <= lim), f"max rel err {(err / np.maximum(np.abs(Y_ref), 1e-300)).max():.3e}"
    assert np.all(Y_got[acc_ref == 0] == 0.0)


def check_forward_full(xq_ref, s_ref, wq_ref, gamma_ref, Y, acc):
    acc_ref = oracle.contract(xq_ref, wq_ref)
    got = acc.cpu().numpy()
    if not np.array_equal(got, acc_ref):
        bad = np.argwhere(got != acc_ref)
        raise AssertionError(f"acc mismatch at {len(bad)} entries, first {bad[:5].tolist()}")
    check_y(Y.cpu().numpy(), acc_ref, gamma_ref, s_ref[:, None])


def check_forward_sampled(xq_ref, s_ref, wq_ref, gamma_ref, Y, acc, npairs=4096, seed=0, xq_rows=None):
    """Sampled (m, n) outputs; xq_ref may hold only the rows listed in
    xq_rows (then ms index into xq_rows)."""
    rng = np.random.default_rng(seed)
    M, N = Y.shape
    if xq_rows is None:
        ms = rng.integers(0, M, npairs)
        local = ms
    else:
        local = rng.integers(0, len(xq_rows), npairs)
        ms = np.asarray(xq_rows)[local]
    ns = rng.integers(0, N, npairs)
    # always include the corners
    ms = np.concatenate([ms, [0, M - 1, 0, M - 1]]) if xq_rows is None else ms
    local = np.concatenate([local, [0, M - 1, 0, M - 1]]) if xq_rows is None else local
    ns = np.concatenate([ns, [0, N - 1, N - 1, 0]]) if xq_rows is None else ns
    acc_ref = oracle.contract_pairs(xq_ref, wq_ref, local, ns)
    mi = torch.as_tensor(ms, device=Y.device)
    ni = torch.as_tensor(ns, device=Y.device)
    if acc is not None:
        got = acc[mi, ni].cpu().numpy()
        assert np.array_equal(got, acc_ref), f"acc mismatch at {(got != acc_ref).sum()} sampled entries"
    check_y(Y[mi, ni].cpu().numpy(), acc_ref, gamma_ref, s_ref[local])
