"""Python binding of libbitlinear.so (include/bitlinear.h).

Argument marshalling only: every function here checks that torch tensors are
CUDA tensors on the current device, contiguous, of the right dtype and large
enough for the call, allocates outputs with torch when
the caller passes none, and calls the C entry point of the same name with
raw device pointers and the current torch stream.  All arithmetic runs in
the library's kernels; if the library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

_LIB = None

BL_F32, BL_BF16 = 0, 1
BL_MAX_GROUP = 128
BL_FWD_WEIGHTS_READY = 1
_DTYPES = {torch.float32: BL_F32, torch.bfloat16: BL_BF16}

_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_sz = ctypes.c_size_t
_f32 = ctypes.c_float
_int = ctypes.c_int


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class Problem(ctypes.Structure):
    """bl_problem: one (packed, gamma, x_q, s, Y) problem of a grouped forward."""
    _fields_ = [("packed", _p), ("gamma", _p), ("x_q", _p), ("s", _p), ("Y", _p),
                ("acc_out", _p), ("N", _i64), ("K", _i64)]


class ActProblem(ctypes.Structure):
    """bl_act_problem: one activation input of a grouped act quant."""
    _fields_ = [("X", _p), ("subln_gain", _p), ("x_q", _p), ("s", _p), ("K", _i64)]


class WeightProblem(ctypes.Structure):
    """bl_weight_problem: one weight matrix of a grouped weight quantization."""
    _fields_ = [("W", _p), ("N", _i64), ("K", _i64), ("packed", _p), ("gamma", _p)]


class LinearProblem(ctypes.Structure):
    """bl_linear_problem: one weight matrix (and its output) of a grouped bl_linear."""
    _fields_ = [("W", _p), ("Y", _p), ("N", _i64)]


class DecodeProblem(ctypes.Structure):
    """bl_decode_problem: one problem of the fused grouped decode (X in, Y out)."""
    _fields_ = [("packed", _p), ("gamma", _p), ("X", _p), ("subln_gain", _p), ("Y", _p), ("x_q", _p),
                ("s", _p), ("acc_out", _p), ("N", _i64), ("K", _i64)]


_SIGS = {
    "bl_status_string": (ctypes.c_char_p, [_int]),
    "bl_version": (_int, []),
    "bl_check_device_error": (_int, [_p]),
    "bl_quant_weights_workspace_bytes": (_sz, [_i64, _i64]),
    "bl_quant_weights": (_int, [_p, _int, _i64, _i64, _p, _p, _p, _sz, _p]),
    "bl_quant_weights_noalloc": (_int, [_p, _int, _i64, _i64, _p, _p, _p]),
    "bl_quant_act": (_int, [_p, _int, _i64, _i64, _p, _f32, _p, _p, _p]),
    "bl_ffn_act_quant": (_int, [_p, _p, _i64, _i64, _p, _f32, _p, _p, _p]),
    "bl_forward": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p]),
    "bl_linear_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_linear": (_int, [_p, _int, _p, _int, _i64, _i64, _i64, _p, _f32, _p, _sz, _p, _p]),
    "bl_forward_grouped": (_int, [ctypes.POINTER(Problem), _int, _i64, ctypes.c_uint, _p]),
    "bl_debug_decode_plan": (_int, [_p, _int, _i64, _int, _p, _int, _p]),
    "bl_debug_forward_prefill": (_int, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, ctypes.c_longlong,
                                        ctypes.c_uint32, _p]),
    "bl_quant_act_grouped": (_int, [ctypes.POINTER(ActProblem), _int, _int, _i64, _f32, _p]),
    "bl_linear_decode_grouped": (_int, [ctypes.POINTER(DecodeProblem), _int, _int, _i64, _f32, ctypes.c_uint,
                                        _p]),
    "bl_quant_weights_grouped": (_int, [ctypes.POINTER(WeightProblem), _int, _int, _p, _sz, _p]),
    "bl_forward_glu": (_int, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _p]),
    "bl_backward_dx": (_int, [_p, _p, _p, _i64, _i64, _i64, _p, _p]),
    "bl_backward_dw_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "bl_backward_dw": (_int, [_p, _p, _p, _p, _int, _p, _f32, _i64, _i64, _i64, _p, _sz, _p, _p]),
    "bl_linear_grouped_workspace_bytes": (_sz, [ctypes.POINTER(LinearProblem), _int, _i64, _i64]),
    "bl_linear_grouped": (_int, [ctypes.POINTER(LinearProblem), _int, _int, _p, _int, _i64, _i64, _p, _f32, _p, _sz,
                                 _p]),
}

EXPORTED = tuple(_SIGS)


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libbitlinear.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m ternary_quantized_linear_bitlinear_b200.build`")
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    return lib().bl_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise BitLinearError(status, where)


def _current_device() -> int:
    return torch.cuda.current_device()


def _stream(stream) -> int:
    """Raw handle of `stream` (default: torch's current stream).  The library
    launches on the current device, so an explicit stream must belong to it."""
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if stream.device_index != _current_device():
        raise ValueError(f"stream belongs to cuda:{stream.device_index}, the current device is "
                         f"cuda:{_current_device()}")
    return stream.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _is_cuda(t: torch.Tensor) -> bool:
    return t.is_cuda


def _device_index(t: torch.Tensor) -> int:
    return t.device.index


def _dev(t: torch.Tensor, name: str, dtype=None, min_numel: int = 0):
    """A device buffer the library reads or writes: CUDA, on the current
    device (the library launches there, so every buffer of a call lives on
    one GPU), contiguous, of the given dtype and at least min_numel elements
    (so that no kernel touches host memory, another GPU's memory, or runs
    past the end of a caller's buffer)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not _is_cuda(t):
        raise ValueError(f"{name} must be a CUDA tensor")
    if _device_index(t) != _current_device():
        raise ValueError(f"{name} lives on cuda:{_device_index(t)}, the current device is cuda:{_current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs at least {min_numel}")
    return t


def _opt(t, name: str, dtype=None, min_numel: int = 0):
    return None if t is None else _dev(t, name, dtype, min_numel)


def _mat(t: torch.Tensor, name: str, cols: int | None = None, rows: int | None = None):
    """A 2-D float32 or bfloat16 input matrix ([N, K] weights or [M, K]
    activations) on the current device, optionally with a fixed column
    (and row) count -> (rows, cols)."""
    _dev(t, name)
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    if t.dtype not in _DTYPES:
        raise ValueError(f"{name} must be float32 or bfloat16, got {t.dtype}")
    if cols is not None and t.shape[1] != cols:
        raise ValueError(f"{name} has {t.shape[1]} columns, expected {cols}")
    if rows is not None and t.shape[0] != rows:
        raise ValueError(f"{name} has {t.shape[0]} rows, expected {rows}")
    return t.shape[0], t.shape[1]


# -- workspace queries ---------------------------------------------------------

def quant_weights_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bl_quant_weights_workspace_bytes(N, K))


def linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bl_linear_workspace_bytes(M, N, K))


# -- step 1 --------------------------------------------------------------------

def bl_quant_weights(W: torch.Tensor, packed=None, gamma=None, workspace=None, stream=None):
    """-> (packed uint8 [N, K/4], gamma float32 [1])."""
    N, K = _mat(W, "W")
    if packed is None:
        packed = torch.empty(N, K // 4, dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(4, dtype=torch.float32, device=W.device)[:1]
    if workspace is None:
        workspace = torch.empty(quant_weights_workspace_bytes(N, K), dtype=torch.uint8, device=W.device)
    _dev(packed, "packed", torch.uint8, N * K // 4)
    _dev(gamma, "gamma", torch.float32, 1)
    _dev(workspace, "workspace", torch.uint8)
    rc = lib().bl_quant_weights(W.data_ptr(), _DTYPES.get(W.dtype, -1), N, K, packed.data_ptr(), gamma.data_ptr(),
                                workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(rc, "bl_quant_weights")
    return packed, gamma


def bl_quant_weights_noalloc(W: torch.Tensor, packed=None, gamma=None, stream=None):
    """bl_quant_weights without a workspace argument: the library's static
    device scratch is used instead (for callers that cannot allocate device
    memory; see include/bitlinear.h).  Outputs are allocated here only when
    the caller passes none."""
    N, K = _mat(W, "W")
    if packed is None:
        packed = torch.empty(N, K // 4, dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(4, dtype=torch.float32, device=W.device)[:1]
    _dev(packed, "packed", torch.uint8, N * K // 4)
    _dev(gamma, "gamma", torch.float32, 1)
    rc = lib().bl_quant_weights_noalloc(W.data_ptr(), _DTYPES.get(W.dtype, -1), N, K, packed.data_ptr(),
                                        gamma.data_ptr(), _stream(stream))
    _check(rc, "bl_quant_weights_noalloc")
    return packed, gamma


def bl_quant_weights_grouped(Ws, packed=None, gammas=None, workspace=None, stream=None):
    """Several weight matrices (same dtype) in three launches -> ([packed], [gamma]),
    each as bl_quant_weights(W) would give it."""
    Ws = list(Ws)
    if not 1 <= len(Ws) <= 8:
        raise ValueError("between 1 and 8 weight matrices")
    dtype = Ws[0].dtype
    shapes = [_mat(W, f"Ws[{i}]") for i, W in enumerate(Ws)]
    for i, W in enumerate(Ws):
        _dev(W, f"Ws[{i}]", dtype)
    dev = Ws[0].device
    if packed is None:
        packed = [torch.empty(N, K // 4, dtype=torch.uint8, device=dev) for N, K in shapes]
    if gammas is None:
        gammas = [torch.empty(4, dtype=torch.float32, device=dev)[:1] for _ in Ws]
    if workspace is None:
        workspace = torch.empty(quant_weights_workspace_bytes(1, 64), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8)
    arr = (WeightProblem * len(Ws))()
    for i, ((N, K), W, pk, g) in enumerate(zip(shapes, Ws, packed, gammas)):
        _dev(pk, f"packed[{i}]", torch.uint8, N * K // 4)
        _dev(g, f"gammas[{i}]", torch.float32, 1)
        arr[i] = WeightProblem(W.data_ptr(), N, K, pk.data_ptr(), g.data_ptr())
    rc = lib().bl_quant_weights_grouped(arr, len(Ws), _DTYPES[dtype], workspace.data_ptr(), workspace.numel(),
                                        _stream(stream))
    _check(rc, "bl_quant_weights_grouped")
    return packed, gammas


# -- step 2 --------------------------------------------------------------------

def bl_quant_act(X: torch.Tensor, subln_gain=None, subln_eps: float = 1e-6, x_q=None, s=None, stream=None):
    """-> (x_q int8 [M, K], s float32 [M])."""
    M, K = _mat(X, "X")
    if x_q is None:
        x_q = torch.empty(M, K, dtype=torch.int8, device=X.device)
    if s is None:
        s = torch.empty(M, dtype=torch.float32, device=X.device)
    _dev(x_q, "x_q", torch.int8, M * K)
    _dev(s, "s", torch.float32, M)
    _opt(subln_gain, "subln_gain", torch.float32, K)
    rc = lib().bl_quant_act(X.data_ptr(), _DTYPES.get(X.dtype, -1), M, K, _ptr(subln_gain), subln_eps,
                            x_q.data_ptr(), s.data_ptr(), _stream(stream))
    _check(rc, "bl_quant_act")
    return x_q, s


def bl_quant_act_grouped(items, dtype=torch.bfloat16, subln_eps: float = 1e-6, stream=None):
    """items: list of (X [M, K], gain or None, x_q [M, K], s [M]), same M and dtype."""
    if dtype not in _DTYPES:
        raise ValueError(f"dtype must be float32 or bfloat16, got {dtype}")
    arr = (ActProblem * len(items))()
    M = items[0][0].shape[0]
    for i, (X, gain, xq, s) in enumerate(items):
        _mat(X, f"items[{i}].X", rows=M)
        _dev(X, f"items[{i}].X", dtype)
        _opt(gain, f"items[{i}].gain", torch.float32, X.shape[1])
        _dev(xq, f"items[{i}].x_q", torch.int8, M * X.shape[1])
        _dev(s, f"items[{i}].s", torch.float32, M)
        arr[i] = ActProblem(X.data_ptr(), _ptr(gain), xq.data_ptr(), s.data_ptr(), X.shape[1])
    rc = lib().bl_quant_act_grouped(arr, len(items), _DTYPES.get(dtype, -1), M, subln_eps, _stream(stream))
    _check(rc, "bl_quant_act_grouped")


# -- steps 3 + 4 ---------------------------------------------------------------

def bl_ffn_act_quant(gate: torch.Tensor, up: torch.Tensor, subln_gain=None, subln_eps: float = 1e-6, x_q=None, s=None,
                     stream=None):
    """Down-projection input from the gate / up outputs: (x_q int8 [M, F], s [M])
    of relu(gate)^2 * up, after SubLN when a gain is given."""
    _dev(gate, "gate", torch.float32)
    _dev(up, "up", torch.float32)
    if gate.dim() != 2 or gate.shape != up.shape:
        raise ValueError("gate and up must be 2-D [M, F] of the same shape")
    M, F = gate.shape
    if x_q is None:
        x_q = torch.empty(M, F, dtype=torch.int8, device=gate.device)
    if s is None:
        s = torch.empty(max(M, 4), dtype=torch.float32, device=gate.device)[:M]
    _dev(x_q, "x_q", torch.int8, M * F)
    _dev(s, "s", torch.float32, M)
    _opt(subln_gain, "subln_gain", torch.float32, F)
    rc = lib().bl_ffn_act_quant(gate.data_ptr(), up.data_ptr(), M, F, _ptr(subln_gain), subln_eps, x_q.data_ptr(),
                                s.data_ptr(), _stream(stream))
    _check(rc, "bl_ffn_act_quant")
    return x_q, s


def bl_forward(packed, gamma, x_q, s, N: int, Y=None, acc_out=None, stream=None):
    """-> Y float32 [M, N] (acc_out int32 [M, N] filled when given)."""
    M, K = _xq2d(x_q)
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=x_q.device)
    _check_forward_args(packed, gamma, s, Y, acc_out, M, N, K)
    rc = lib().bl_forward(packed.data_ptr(), gamma.data_ptr(), x_q.data_ptr(), s.data_ptr(), M, N, K, Y.data_ptr(),
                          _ptr(acc_out), _stream(stream))
    _check(rc, "bl_forward")
    return Y


def _xq2d(x_q):
    _dev(x_q, "x_q", torch.int8)
    if x_q.dim() != 2:
        raise ValueError(f"x_q must be 2-D [M, K], got shape {tuple(x_q.shape)}")
    return x_q.shape[0], x_q.shape[1]


def bl_forward_glu(packed_gate, gamma_gate, packed_up, gamma_up, x_q, s, F: int, h=None, stream=None):
    """h float32 [M, F] = relu(Y_gate)^2 * Y_up of the gate and up projections
    on the shared (x_q, s), from one launch that never stores Y_gate or Y_up."""
    M, K = _xq2d(x_q)
    if h is None:
        h = torch.empty(M, F, dtype=torch.float32, device=x_q.device)
    _dev(packed_gate, "packed_gate", torch.uint8, F * K // 4)
    _dev(packed_up, "packed_up", torch.uint8, F * K // 4)
    _dev(gamma_gate, "gamma_gate", torch.float32, 1)
    _dev(gamma_up, "gamma_up", torch.float32, 1)
    _dev(s, "s", torch.float32, M)
    _dev(h, "h", torch.float32, M * F)
    rc = lib().bl_forward_glu(packed_gate.data_ptr(), gamma_gate.data_ptr(), packed_up.data_ptr(), gamma_up.data_ptr(),
                              x_q.data_ptr(), s.data_ptr(), M, F, K, h.data_ptr(), _stream(stream))
    _check(rc, "bl_forward_glu")
    return h


def bl_backward_dx(dY, packed, gamma, K: int, dX=None, stream=None):
    """dX float32 [M, K] = dY @ (gamma W_q) (straight-through backward of the
    activation), dY bfloat16 [M, N]."""
    _dev(dY, "dY", torch.bfloat16)
    if dY.dim() != 2:
        raise ValueError("dY must be 2-D [M, N]")
    M, N = dY.shape
    if dX is None:
        dX = torch.empty(M, K, dtype=torch.float32, device=dY.device)
    _dev(packed, "packed", torch.uint8, N * K // 4)
    _dev(gamma, "gamma", torch.float32, 1)
    _dev(dX, "dX", torch.float32, M * K)
    rc = lib().bl_backward_dx(dY.data_ptr(), packed.data_ptr(), gamma.data_ptr(), M, N, K, dX.data_ptr(),
                              _stream(stream))
    _check(rc, "bl_backward_dx")
    return dX


def bl_backward_dw(dY, x_q, s, W, gamma, beta: float = 0.0, dW=None, workspace=None, stream=None):
    """dW float32 [N, K] = (dY^T @ (x_q / s)) * scale(W / gamma): the weight
    gradient under the hard (beta <= 0) or soft STE scale; dY bfloat16 [M, N],
    x_q, s from the forward's activation quantization, W the latent weights."""
    _dev(dY, "dY", torch.bfloat16)
    if dY.dim() != 2:
        raise ValueError("dY must be 2-D [M, N]")
    M, N = dY.shape
    Mx, K = _xq2d(x_q)
    if Mx != M:
        raise ValueError("x_q and dY disagree on M")
    _mat(W, "W", cols=K, rows=N)
    _dev(s, "s", torch.float32, M)
    _dev(gamma, "gamma", torch.float32, 1)
    if dW is None:
        dW = torch.empty(N, K, dtype=torch.float32, device=dY.device)
    _dev(dW, "dW", torch.float32, N * K)
    need = int(lib().bl_backward_dw_workspace_bytes(M, N, K))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dY.device)
    _dev(workspace, "workspace", torch.uint8, need)
    rc = lib().bl_backward_dw(dY.data_ptr(), x_q.data_ptr(), s.data_ptr(), W.data_ptr(), _DTYPES[W.dtype],
                              gamma.data_ptr(), float(beta), M, N, K, workspace.data_ptr(), workspace.numel(), dW.data_ptr(),
                              _stream(stream))
    _check(rc, "bl_backward_dw")
    return dW


def _check_forward_args(packed, gamma, s, Y, acc_out, M, N, K):
    _dev(packed, "packed", torch.uint8, N * K // 4)
    _dev(gamma, "gamma", torch.float32, 1)
    _dev(s, "s", torch.float32, M)
    _dev(Y, "Y", torch.float32, M * N)
    _opt(acc_out, "acc_out", torch.int32, M * N)


def _rows_of(t, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D [M, K] when M is not given")
    return t.shape[0]


def make_problems(items, M: int | None = None):
    """items: list of (packed, gamma, x_q, s, Y, acc_out or None, N, K) -> ctypes
    array for bl_forward_grouped at token count M (default: the first x_q's
    row count).  Every buffer is checked against N, K and M: packed uint8
    >= N*K/4, gamma float32 >= 1, x_q int8 >= M*K, s float32 >= M, Y float32
    and acc_out int32 >= M*N."""
    if M is None:
        M = _rows_of(items[0][2], "items[0].x_q")
    arr = (Problem * len(items))()
    for i, (packed, gamma, xq, s, Y, acc, N, K) in enumerate(items):
        _dev(packed, f"items[{i}].packed", torch.uint8, N * K // 4)
        _dev(gamma, f"items[{i}].gamma", torch.float32, 1)
        _dev(xq, f"items[{i}].x_q", torch.int8, M * K)
        _dev(s, f"items[{i}].s", torch.float32, M)
        _dev(Y, f"items[{i}].Y", torch.float32, M * N)
        _opt(acc, f"items[{i}].acc_out", torch.int32, M * N)
        arr[i] = Problem(packed.data_ptr(), gamma.data_ptr(), xq.data_ptr(), s.data_ptr(), Y.data_ptr(),
                         _ptr(acc), N, K)
    arr.bl_M = M
    return arr


def _check_array(problems, count: int, M: int, dtype=None):
    """A problem array built by make_problems / make_decode_problems was
    validated for one M (and dtype): launching it with another, or with more
    problems than it holds, would let a kernel run past a buffer."""
    if count < 0 or count > len(problems):
        raise ValueError(f"count {count} outside the {len(problems)} problems of the array")
    checked_M = getattr(problems, "bl_M", None)
    if checked_M is not None and M != checked_M:
        raise ValueError(f"the problem array was checked for M = {checked_M}, called with M = {M}")
    checked_dt = getattr(problems, "bl_dtype", None)
    if dtype is not None and checked_dt is not None and dtype != checked_dt:
        raise ValueError(f"the problem array was checked for X of {checked_dt}, called with {dtype}")


def bl_forward_grouped(problems, count: int, M: int, flags: int = 0, stream=None):
    """problems: ctypes array from make_problems (built once, launched many times)."""
    _check_array(problems, count, M)
    rc = lib().bl_forward_grouped(problems, count, M, flags, _stream(stream))
    _check(rc, "bl_forward_grouped")


def make_decode_problems(items, M: int | None = None):
    """items: list of (packed, gamma, X, subln_gain or None, Y, x_q or None, s or None, acc_out or None, N, K)
    -> ctypes array for bl_linear_decode_grouped at token count M (default:
    the first X's row count).  Every X must have the first one's dtype
    (float32 or bfloat16); every buffer is checked against N, K and M."""
    if M is None:
        M = _rows_of(items[0][2], "items[0].X")
    dtype = items[0][2].dtype if isinstance(items[0][2], torch.Tensor) else None
    if dtype not in _DTYPES:
        raise ValueError(f"X must be float32 or bfloat16, got {dtype}")
    arr = (DecodeProblem * len(items))()
    for i, (packed, gamma, X, gain, Y, xq, s, acc, N, K) in enumerate(items):
        _dev(packed, f"items[{i}].packed", torch.uint8, N * K // 4)
        _dev(gamma, f"items[{i}].gamma", torch.float32, 1)
        _dev(X, f"items[{i}].X", dtype, M * K)
        _opt(gain, f"items[{i}].subln_gain", torch.float32, K)
        _dev(Y, f"items[{i}].Y", torch.float32, M * N)
        _opt(xq, f"items[{i}].x_q", torch.int8, M * K)
        _opt(s, f"items[{i}].s", torch.float32, M)
        _opt(acc, f"items[{i}].acc_out", torch.int32, M * N)
        arr[i] = DecodeProblem(packed.data_ptr(), gamma.data_ptr(), X.data_ptr(), _ptr(gain), Y.data_ptr(), _ptr(xq),
                               _ptr(s), _ptr(acc), N, K)
    arr.bl_M = M
    arr.bl_dtype = dtype
    return arr


def bl_linear_decode_grouped(problems, count: int, M: int, dtype=torch.bfloat16, subln_eps: float = 1e-6,
                             flags: int = 0, stream=None):
    """Steps 2-4 fused: problems from make_decode_problems (X of `dtype`, same M)."""
    if dtype not in _DTYPES:
        raise ValueError(f"dtype must be float32 or bfloat16, got {dtype}")
    _check_array(problems, count, M, dtype)
    rc = lib().bl_linear_decode_grouped(problems, count, _DTYPES[dtype], M, subln_eps, flags, _stream(stream))
    _check(rc, "bl_linear_decode_grouped")


# -- all four steps ------------------------------------------------------------

def bl_linear(W, X, subln_gain=None, subln_eps: float = 1e-6, Y=None, workspace=None, stream=None):
    """-> Y float32 [M, N] = BitLinear(X) with weights W quantized in the call."""
    N, K = _mat(W, "W")
    M, _ = _mat(X, "X", cols=K)
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=X.device)
    _dev(Y, "Y", torch.float32, M * N)
    _dev(workspace, "workspace", torch.uint8)
    _opt(subln_gain, "subln_gain", torch.float32, K)
    rc = lib().bl_linear(W.data_ptr(), _DTYPES.get(W.dtype, -1), X.data_ptr(), _DTYPES.get(X.dtype, -1), M, N, K,
                         _ptr(subln_gain), subln_eps, workspace.data_ptr(), workspace.numel(), Y.data_ptr(),
                         _stream(stream))
    _check(rc, "bl_linear")
    return Y


def bl_linear_grouped(Ws, X, subln_gain=None, subln_eps: float = 1e-6, Ys=None, workspace=None, stream=None):
    """Up to 4 weight matrices sharing the input X (e.g. q, k, v), all steps,
    weights quantized in the call -> [Y_i float32 [M, N_i]]."""
    Ws = list(Ws)
    if not 1 <= len(Ws) <= 4:
        raise ValueError("between 1 and 4 weight matrices")
    wdt = Ws[0].dtype
    shapes = [_mat(W, f"Ws[{i}]") for i, W in enumerate(Ws)]
    K = shapes[0][1]
    for i, W in enumerate(Ws):
        _mat(W, f"Ws[{i}]", cols=K)
        _dev(W, f"Ws[{i}]", wdt)
    M, _ = _mat(X, "X", cols=K)
    if Ys is None:
        Ys = [torch.empty(M, N, dtype=torch.float32, device=X.device) for N, _ in shapes]
    arr = (LinearProblem * len(Ws))()
    for i, ((N, _), W, Y) in enumerate(zip(shapes, Ws, Ys)):
        _dev(Y, f"Ys[{i}]", torch.float32, M * N)
        arr[i] = LinearProblem(W.data_ptr(), Y.data_ptr(), N)
    need = int(lib().bl_linear_grouped_workspace_bytes(arr, len(Ws), M, K))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _dev(workspace, "workspace", torch.uint8, need)
    _opt(subln_gain, "subln_gain", torch.float32, K)
    rc = lib().bl_linear_grouped(arr, len(Ws), _DTYPES[wdt], X.data_ptr(), _DTYPES[X.dtype], M, K, _ptr(subln_gain),
                                 subln_eps, workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(rc, "bl_linear_grouped")
    return Ys


def bl_debug_decode_plan(shapes, M: int, sms: int = 148):
    """Host-side plan of a decode call over problems of the given (N, K)
    shapes at M tokens on a GPU with `sms` SMs (nothing is launched; no GPU
    needed): a list of launches, each {"ctas", "smem", "problems": [{"job",
    "row0", "rows", "glog", "kch", "cta_begin"}]}."""
    shapes = list(shapes)
    arr = (ctypes.c_int64 * (2 * len(shapes)))(*[int(v) for nk in shapes for v in nk])
    cap = 64 + 16 * 6 * max(1, len(shapes)) * 8
    out = (ctypes.c_int * cap)()
    written = ctypes.c_int(0)
    rc = lib().bl_debug_decode_plan(arr, len(shapes), int(M), int(sms), out, cap, ctypes.byref(written))
    _check(rc, "bl_debug_decode_plan")
    vals, launches, i = list(out[:written.value]), [], 0
    while i < len(vals):
        ctas, smem, n = vals[i:i + 3]
        i += 3
        probs = []
        for _ in range(n):
            job, row0, rows, glog, kch, cta0 = vals[i:i + 6]
            i += 6
            probs.append(dict(job=job, row0=row0, rows=rows, glog=glog, kch=kch, cta_begin=cta0))
        launches.append(dict(ctas=ctas, smem=smem, problems=probs))
    return launches


def bl_debug_forward_prefill(packed, gamma, x_q, s, N: int, Y=None, acc_out=None, skip_iter: int = -1,
                             timeout_us: int = 2_000_000, stream=None):
    """Test hook (include/bitlinear_debug.h): bl_forward forced through the
    tcgen05 prefill engine, with bounded waits of timeout_us and an optional
    stalled k-iteration."""
    M, K = _xq2d(x_q)
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=x_q.device)
    _check_forward_args(packed, gamma, s, Y, acc_out, M, N, K)
    rc = lib().bl_debug_forward_prefill(packed.data_ptr(), gamma.data_ptr(), x_q.data_ptr(), s.data_ptr(), M, N, K,
                                        Y.data_ptr(), _ptr(acc_out), skip_iter, timeout_us, _stream(stream))
    _check(rc, "bl_debug_forward_prefill")
    return Y


def bl_check_device_error(stream=None):
    _check(lib().bl_check_device_error(_stream(stream)), "bl_check_device_error")
