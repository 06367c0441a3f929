"""Seeded synthetic inputs for the BitLinear forward.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests; it holds none of the method's arithmetic (no scale, no
rounding, no packing) -- only random tensors with the shapes and value
distributions of the five workloads.  Everything is drawn on the CPU from a
``torch.Generator`` so both sides see identical bits.

Workloads (projection shapes are (N, K) = (out_features, in_features)):
  single    one BitLinear 768 -> 2048, M = 16; W fp32 ~ N(0, 0.02^2);
            X fp32 ~ N(0, 1) with 4 outlier channels scaled x20.
  decode125m 12 layers of a 125M student (hidden 768, 12 Q / 4 KV heads of
            dim 64, MLP 2048): q,o 768x768; k,v 256x768; gate,up 2048x768;
            down 768x2048.  Weights already ternary with a 29/42/29 split of
            -1/0/+1 (the "Distillix 125M" model card, Model Stats), stored
            as +-c / 0 floats; X bf16 ~ N(0, 1); M in {1, 4, 8}.
  prefill1b4 one layer of a 1.4B-shape model (hidden 1536, FFN 4096,
            12 Q / 4 KV heads of dim 128 -- "SLM750-Edge" section 2.2):
            q,o 1536^2; k,v 512x1536; gate,up 4096x1536; down 1536x4096;
            M = 8192; W bf16 ~ N(0, 0.02^2); X bf16 = 0.5 * Student-t(3).
  layer3b   one layer of a 3B-shape model (hidden 3200, FFN 8640):
            q,k,v,o 3200^2; gate,up 8640x3200; down 3200x8640; M = 1 and
            M = 2048; W ~ N(0, 0.015^2); X bf16 ~ N(0, 1) with 1 % of the
            channels scaled x30.
  qat4b     one layer of a 4B-shape model (hidden 2560, FFN 9728; q,k,v,o
            taken as 2560^2), M = 16 x 2048 = 32768; bf16 master W
            ~ N(0, 0.02^2) re-quantized every call; SubLN gain ~ U(0.9, 1.1),
            eps 1e-6, before o_proj and down_proj.
"""
from __future__ import annotations

import torch

SUBLN_EPS = 1e-6

# (name, N, K, subln_before)
DECODE125M = dict(hidden=768, kv=256, ffn=2048, layers=12, tokens=(1, 4, 8))
PREFILL1B4 = dict(hidden=1536, kv=512, ffn=4096, tokens=8192)
LAYER3B = dict(hidden=3200, kv=3200, ffn=8640, tokens=(1, 2048))
QAT4B = dict(hidden=2560, kv=2560, ffn=9728, tokens=16 * 2048)


def projections(hidden: int, kv: int, ffn: int):
    """[(name, N, K, subln_before)] for one transformer layer.  SubLN sits
    before the attention output projection and the FFN down projection
    ("BitDistill", Stage 1)."""
    return [
        ("q", hidden, hidden, False),
        ("k", kv, hidden, False),
        ("v", kv, hidden, False),
        ("o", hidden, hidden, True),
        ("gate", ffn, hidden, False),
        ("up", ffn, hidden, False),
        ("down", hidden, ffn, True),
    ]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, dtype=torch.float32) -> torch.Tensor:
    g = _gen(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)


def with_outlier_channels(x: torch.Tensor, count: int, mult: float, seed: int) -> torch.Tensor:
    """Scale ``count`` seeded columns of x (computed in fp32, then cast back)."""
    g = _gen(seed)
    idx = torch.randperm(x.shape[-1], generator=g)[:count]
    y = x.float().clone()
    y[..., idx] *= mult
    return y.to(x.dtype)


def student_t(shape, nu: int, scale: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """scale * Z / sqrt(chi2_nu / nu), chi2 drawn as a sum of nu squared normals."""
    g = _gen(seed)
    z = torch.randn(*shape, generator=g, dtype=torch.float64)
    chi2 = torch.zeros(shape, dtype=torch.float64)
    for _ in range(nu):
        chi2 += torch.randn(*shape, generator=g, dtype=torch.float64) ** 2
    t = z / torch.sqrt(chi2 / nu)
    return (t * scale).to(dtype)


def ternary_weights(N: int, K: int, seed: int, probs=(0.29, 0.42, 0.29), magnitude: float = 0.02,
                    dtype=torch.float32) -> torch.Tensor:
    """Already-ternary weights: -magnitude / 0 / +magnitude with the given
    probabilities, i.i.d."""
    g = _gen(seed)
    u = torch.rand(N, K, generator=g, dtype=torch.float64)
    w = torch.zeros(N, K, dtype=torch.float32)
    w[u < probs[0]] = -magnitude
    w[u >= probs[0] + probs[1]] = magnitude
    return w.to(dtype)


def uniform(shape, lo: float, hi: float, seed: int, dtype=torch.float32) -> torch.Tensor:
    g = _gen(seed)
    return (torch.rand(*shape, generator=g, dtype=torch.float32) * (hi - lo) + lo).to(dtype)


# -- the five workloads -------------------------------------------------------

def single(seed: int = 0):
    """W fp32 [2048, 768], X fp32 [16, 768] with 4 outlier channels x20."""
    W = normal((2048, 768), 0.02, seed)
    X = normal((16, 768), 1.0, seed + 1)
    X = with_outlier_channels(X, 4, 20.0, seed + 2)
    return W, X


def decode125m_layer_shapes():
    c = DECODE125M
    return projections(c["hidden"], c["kv"], c["ffn"])


def decode125m(seed: int = 1, M: int = 1, layers: int | None = None):
    """List of (name, W float32 ternary*0.02 [N, K], X bf16 [M, K]) for every
    projection of every layer, layer-major."""
    c = DECODE125M
    L = c["layers"] if layers is None else layers
    out = []
    for layer in range(L):
        for p, (name, N, K, _) in enumerate(decode125m_layer_shapes()):
            s = seed * 100003 + layer * 101 + p * 7
            W = ternary_weights(N, K, s)
            X = normal((M, K), 1.0, s + 1, torch.bfloat16)
            out.append((f"L{layer}.{name}", W, X))
    return out


def prefill1b4_shapes():
    c = PREFILL1B4
    return projections(c["hidden"], c["kv"], c["ffn"])


def prefill1b4(seed: int = 2, M: int | None = None, which=None):
    """List of (name, W bf16 [N, K], X bf16 [M, K])."""
    M = PREFILL1B4["tokens"] if M is None else M
    out = []
    for p, (name, N, K, _) in enumerate(prefill1b4_shapes()):
        if which is not None and name not in which:
            continue
        s = seed * 100003 + p * 7
        W = normal((N, K), 0.02, s, torch.bfloat16)
        X = student_t((M, K), 3, 0.5, s + 1, torch.bfloat16)
        out.append((name, W, X))
    return out


def layer3b_shapes():
    c = LAYER3B
    return projections(c["hidden"], c["kv"], c["ffn"])


def layer3b(seed: int = 3, M: int = 1, which=None):
    """List of (name, W float32 [N, K], X bf16 [M, K]); 1 % of channels x30."""
    out = []
    for p, (name, N, K, _) in enumerate(layer3b_shapes()):
        if which is not None and name not in which:
            continue
        s = seed * 100003 + p * 7
        W = normal((N, K), 0.015, s)
        X = normal((M, K), 1.0, s + 1, torch.bfloat16)
        X = with_outlier_channels(X, max(1, K // 100), 30.0, s + 2)
        out.append((name, W, X))
    return out


def qat4b_shapes():
    c = QAT4B
    return projections(c["hidden"], c["kv"], c["ffn"])


def qat4b(seed: int = 4, M: int | None = None, which=None):
    """List of (name, W bf16 [N, K], X bf16 [M, K], gain fp32 [K] or None)."""
    M = QAT4B["tokens"] if M is None else M
    out = []
    for p, (name, N, K, subln) in enumerate(qat4b_shapes()):
        if which is not None and name not in which:
            continue
        s = seed * 100003 + p * 7
        W = normal((N, K), 0.02, s, torch.bfloat16)
        X = normal((M, K), 1.0, s + 1, torch.bfloat16)
        gain = uniform((K,), 0.9, 1.1, s + 2) if subln else None
        out.append((name, W, X, gain))
    return out
