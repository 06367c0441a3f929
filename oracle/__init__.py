"""CPU oracle for the BitLinear (BitNet b1.58) forward and its
straight-through backward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never touches the CUDA library and
the CUDA library never touches it; the only thing the two sides share is the
seeded input generator module, which holds none of the method's arithmetic.

The arithmetic lives in ``oracle.c`` (plain C, built by ``build.py``); this
module only marshals numpy arrays.  Each function names the passage of the
source pages it follows; the readings taken where the pages are silent are
spelled out in ``oracle.c``'s header.

Parity status per function (what pins it, see tests/test_oracle_pins.py):
  absmean_gamma   pinned: exact sum vs Python Fraction, constant-magnitude W
  ternarize       pinned: round_clip case form (SLM750-Edge 3.1), brute force
  pack / unpack   pinned: bit layout examples in tests/golden, size N*K/4
  quant_act       pinned: argmax -> +-127, scale invariance, zero row
  rmsnorm         pinned: constant-row closed form, exact sum vs Fraction
  contract        pinned: add/subtract identity (bitone "How 1.58-bit Works"),
                  int64 matmul, brute force over all ternary rows for tiny K
  contract_blas   pinned: equals contract (int64 loop) on ragged shapes and
                  at the extreme |acc| = 128 K; rejects K beyond its bound
  rescale         pinned: closed form on hand values
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_i64 = ctypes.c_int64
_f32 = ctypes.c_float
_ptr = ctypes.c_void_p


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        sig = {
            "oracle_abs_sum_exact": (ctypes.c_int, [_ptr, _i64, _ptr]),
            "oracle_limbs_to_double": (ctypes.c_double, [_ptr, ctypes.c_int, ctypes.c_int]),
            "oracle_absmean_gamma": (ctypes.c_int, [_ptr, _i64, _ptr]),
            "oracle_ternarize": (None, [_ptr, _i64, _f32, _ptr]),
            "oracle_pack": (ctypes.c_int, [_ptr, _i64, _i64, _ptr]),
            "oracle_unpack": (ctypes.c_int, [_ptr, _i64, _i64, _ptr]),
            "oracle_rmsnorm": (ctypes.c_int, [_ptr, _i64, _ptr, _f32, _ptr]),
            "oracle_quant_act": (ctypes.c_int, [_ptr, _i64, _i64, _ptr, _f32, _ptr, _ptr, _ptr]),
            "oracle_ffn_act": (None, [_ptr, _ptr, _i64, _ptr]),
            "oracle_contract": (None, [_ptr, _ptr, _i64, _i64, _i64, _ptr]),
            "oracle_contract_pairs": (None, [_ptr, _ptr, _i64, _ptr, _ptr, _i64, _ptr]),
            "oracle_rescale": (None, [_ptr, _i64, _f32, _ptr, _ptr]),
            "oracle_bwd_dx": (None, [_ptr, _ptr, _f32, _i64, _i64, _i64, _ptr]),
            "oracle_bwd_dw": (ctypes.c_int, [_ptr, _ptr, _ptr, _ptr, _f32, ctypes.c_double, _i64, _i64, _i64, _ptr]),
            "oracle_set_num_threads": (None, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32c(a) -> np.ndarray:
    """Upcast to contiguous float32 (bf16 -> f32 is exact; see workloads)."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc:
        raise OracleError(f"{what}: oracle status {rc}")


# -- step 1 -----------------------------------------------------------------

def abs_sum_exact_limbs(w) -> list[int]:
    """Exact sum|w| as 5 little-endian uint64 limbs, in units of 2**-149."""
    w = _f32c(w).ravel()
    limbs = np.zeros(5, dtype=np.uint64)
    _check(_lib().oracle_abs_sum_exact(_p(w), w.size, _p(limbs)), "abs_sum_exact")
    return [int(x) for x in limbs]


def limbs_to_double(limbs, scale_exp: int) -> float:
    arr = np.asarray(limbs, dtype=np.uint64)
    return float(_lib().oracle_limbs_to_double(_p(arr), arr.size, scale_exp))


def absmean_gamma(w) -> np.float32:
    """gamma = mean|W| + 1e-5 ("Distillix" README, 1. BitNet b1.58 Core;
    "bitone" README, Forward pass: gamma = mean(|W|))."""
    w = _f32c(w).ravel()
    g = np.zeros(1, dtype=np.float32)
    _check(_lib().oracle_absmean_gamma(_p(w), w.size, _p(g)), "absmean_gamma")
    return g[0]


# -- step 2 -----------------------------------------------------------------

def ternarize(w, gamma) -> np.ndarray:
    """W_q = clamp(round(W / gamma), -1, 1) ("SLM750-Edge" 3.1 round_clip)."""
    w = _f32c(w)
    q = np.zeros(w.shape, dtype=np.int8)
    _lib().oracle_ternarize(_p(w), w.size, np.float32(gamma), _p(q))
    return q


def pack(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.zeros((N, K // 4), dtype=np.uint8)
    _check(_lib().oracle_pack(_p(q), N, K, _p(out)), "pack")
    return out


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    q = np.zeros((N, K), dtype=np.int8)
    _check(_lib().oracle_unpack(_p(packed), N, K, _p(q)), "unpack")
    return q


def quant_weights(W):
    """(packed [N, K/4] uint8, gamma float32, W_q [N, K] int8)."""
    W = _f32c(W)
    gamma = absmean_gamma(W)
    q = ternarize(W, gamma)
    return pack(q), gamma, q


# -- step 3 -----------------------------------------------------------------

def rmsnorm(x, g, eps: float) -> np.ndarray:
    x = _f32c(x).ravel()
    g = _f32c(g).ravel()
    y = np.zeros_like(x)
    _check(_lib().oracle_rmsnorm(_p(x), x.size, _p(g), np.float32(eps), _p(y)), "rmsnorm")
    return y


def quant_act(X, gain=None, eps: float = 1e-6):
    """(x_q [M, K] int8, s [M] float32): per-token absmax INT8 ("BitDistill",
    Evaluation and results), after SubLN when ``gain`` is given."""
    X = _f32c(X)
    M, K = X.shape
    xq = np.zeros((M, K), dtype=np.int8)
    s = np.zeros(M, dtype=np.float32)
    if gain is None:
        rc = _lib().oracle_quant_act(_p(X), M, K, None, np.float32(eps), _p(xq), _p(s), None)
    else:
        g = _f32c(gain).ravel()
        y = np.zeros((M, K), dtype=np.float32)
        rc = _lib().oracle_quant_act(_p(X), M, K, _p(g), np.float32(eps), _p(xq), _p(s), _p(y))
    _check(rc, "quant_act")
    return xq, s


def ffn_act(gate, up) -> np.ndarray:
    """h = relu(gate)^2 * up elementwise, float32 ("SLM750-Edge", Key
    Architectural Features: ReLU2; section 2.3: gate / up / down)."""
    g = _f32c(gate)
    u = _f32c(up)
    if g.shape != u.shape:
        raise OracleError("ffn_act: gate and up shapes differ")
    h = np.zeros_like(g)
    _lib().oracle_ffn_act(_p(g), _p(u), g.size, _p(h))
    return h


def ffn_act_quant(gate, up, gain=None, eps: float = 1e-6):
    """(x_q, s) of the down projection's input: quant_act(ffn_act(gate, up))."""
    return quant_act(ffn_act(gate, up), gain, eps)


# -- steps 4, 5 -------------------------------------------------------------

def contract(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc [M, N] int64 = x_q @ W_q^T, exact."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    acc = np.zeros((M, N), dtype=np.int64)
    _lib().oracle_contract(_p(xq), _p(wq), M, N, K, _p(acc))
    return acc


def contract_blas(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc [M, N] int64 = x_q @ W_q^T, exact, through a library float32
    matmul (numpy / BLAS): the same definition as ``contract`` with the
    matmul as its one step, fast enough for the full-size workloads.

    Exact because every product x_q * W_q is an integer in [-128, 128] and
    every partial sum an integer of magnitude <= 128 * K < 2^24, so each
    float32 addition (or fused multiply-add) is exact whatever order the
    library sums in.  Refuses K >= 2^24 / 128."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    K = xq.shape[1]
    if wq.shape[1] != K:
        raise OracleError("contract_blas: x_q and W_q disagree on K")
    if 128 * K >= (1 << 24):
        raise OracleError("contract_blas: K too large for exact float32 sums")
    acc = np.matmul(xq.astype(np.float32), wq.astype(np.float32).T)
    return np.rint(acc).astype(np.int64)


def contract_pairs(xq: np.ndarray, wq: np.ndarray, ms, ns) -> np.ndarray:
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    acc = np.zeros(ms.size, dtype=np.int64)
    _lib().oracle_contract_pairs(_p(xq), _p(wq), xq.shape[1], _p(ms), _p(ns), ms.size, _p(acc))
    return acc


def rescale(acc: np.ndarray, gamma, s_per_item: np.ndarray) -> np.ndarray:
    """Y = acc * gamma / s in double ("bitone" README, Forward pass)."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    s_per_item = np.ascontiguousarray(np.broadcast_to(s_per_item, acc.shape), dtype=np.float32)
    Y = np.zeros(acc.shape, dtype=np.float64)
    _lib().oracle_rescale(_p(acc), acc.size, np.float32(gamma), _p(s_per_item), _p(Y))
    return Y


def linear(W, X, gain=None, eps: float = 1e-6):
    """The whole forward: dict with packed, gamma, wq, xq, s, acc, Y."""
    packed, gamma, wq = quant_weights(W)
    xq, s = quant_act(X, gain, eps)
    acc = contract(xq, wq)
    Y = rescale(acc, gamma, s[:, None])
    return dict(packed=packed, gamma=gamma, wq=wq, xq=xq, s=s, acc=acc, Y=Y)


# -- backward under the straight-through estimator (next step of the path) --

def bwd_dx(dY, wq: np.ndarray, gamma) -> np.ndarray:
    """dX [M, K] float64 = dY @ (gamma W_q): the activation quantizer passed
    straight through ("BitDistill", Evaluation and results)."""
    dY = _f32c(dY)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    M, N = dY.shape
    if wq.shape[0] != N:
        raise OracleError("bwd_dx: dY and W_q disagree on N")
    K = wq.shape[1]
    dX = np.zeros((M, K), dtype=np.float64)
    _lib().oracle_bwd_dx(_p(dY), _p(wq), np.float32(gamma), M, N, K, _p(dX))
    return dX


def bwd_dw(dY, xq: np.ndarray, s, W, gamma, beta: float = 0.0) -> np.ndarray:
    """dW [N, K] float64 = (dY^T @ (x_q / s)) * scale(W / gamma), scale the
    hard STE mask (beta <= 0) or the soft 1 - tanh^2(beta W / gamma) ("bitone"
    README, Soft-STE notes)."""
    dY = _f32c(dY)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    s = _f32c(s).ravel()
    W = _f32c(W)
    M, N = dY.shape
    K = xq.shape[1]
    if xq.shape[0] != M or s.size != M or W.shape != (N, K):
        raise OracleError("bwd_dw: shapes disagree")
    dW = np.zeros((N, K), dtype=np.float64)
    _check(_lib().oracle_bwd_dw(_p(dY), _p(xq), _p(s), _p(W), np.float32(gamma), float(beta), M, N, K, _p(dW)),
           "bwd_dw")
    return dW


def set_num_threads(n: int) -> None:
    """Threads the OpenMP loops use from now on (timing only: every output is
    computed by one thread, in the same order, whatever the count)."""
    _lib().oracle_set_num_threads(int(n))


def num_threads() -> int:
    """Threads the OpenMP loops use (OMP_NUM_THREADS, else the affinity mask)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
