"""The rounding bounds behind the double-estimate fast paths (CPU).

Both fast paths take a sum of non-negative terms in double and use a value
only when both ends of a rounding bound agree: the weight absmean (terms
|w|, the bound 2 D 2^-53 relative with D the roundings on a term's path,
plus n 2^-126 for zero / subnormal w entering as values below 2^-126) and
SubLN's sum of squares (terms x^2, 2 (K + 256) 2^-53 relative, plus
K 2^-250).  These tests replay the kernels' summation order in float64 --
per-thread chains, warp butterflies, block and final trees -- on seeded
matrices and rows, and check that the exact sum lies inside the bound each
time, so a miscounted D or a missing term in the bound would show.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

WQ_THREADS = 512
WQ_PACK_THREADS = 256


def _abs_double(bits: np.ndarray) -> np.ndarray:
    """|w| as the kernels build it: exact for normal floats, in [2^-127, 2^-126) for zero / subnormal."""
    a = bits & np.uint32(0x7FFFFFFF)
    normal = a.view(np.float32).astype(np.float64)
    tiny = (1.0 + (a & np.uint32(0x7FFFFF)).astype(np.float64) / 2.0 ** 23) * 2.0 ** -127
    return np.where(a < 0x00800000, tiny, normal)


def _butterfly(v):
    v = list(v)
    off = 16
    while off:
        v = [v[i] + v[i ^ off] for i in range(32)]
        off //= 2
    return v[0]


def _absmean_estimate(bits: np.ndarray, epv: int, nblk: int):
    """S_hat in the kernels' order and the host's D for one matrix."""
    nvec = bits.size // epv
    vecs = bits.reshape(nvec, epv)
    stride = nblk * WQ_THREADS
    blocks = []
    for b in range(nblk):
        thread_sums = []
        for t in range(WQ_THREADS):
            d0 = d1 = 0.0
            for i in range(b * WQ_THREADS + t, nvec, stride):
                x = _abs_double(vecs[i])
                for j in range(0, epv, 2):
                    d0 = d0 + x[j]
                    d1 = d1 + x[j + 1]
            thread_sums.append(d0 + d1)
        warps = [_butterfly(thread_sums[w * 32:(w + 1) * 32]) for w in range(WQ_THREADS // 32)]
        s = warps[0]
        for w in warps[1:]:
            s = s + w
        blocks.append(s)
    per = [0.0] * WQ_PACK_THREADS
    for i, v in enumerate(blocks):
        per[i % WQ_PACK_THREADS] = per[i % WQ_PACK_THREADS] + v
    warps = [_butterfly(per[w * 32:(w + 1) * 32]) for w in range(WQ_PACK_THREADS // 32)]
    s_hat = warps[0]
    for w in warps[1:]:
        s_hat = s_hat + w
    vpt = -(-nvec // stride)
    depth = vpt * epv // 2 + 64 + -(-nblk // WQ_PACK_THREADS)
    return s_hat, depth


def _exact_abs_sum(bits: np.ndarray) -> Fraction:
    s = Fraction(0)
    for v in np.abs(bits.view(np.float32)).astype(np.float64):
        s += Fraction(float(v))
    return s


@pytest.mark.parametrize("n,bf16,kind,nblk", [
    (8 * 512 * 3, True, "normal", 2),
    (4 * 512 * 5 + 64, False, "normal", 3),
    (8 * 512 * 2, True, "wide", 1),
    (4 * 512 * 2, False, "zeros_subnormal", 2),
])
def test_absmean_bound_holds(n, bf16, kind, nblk):
    rng = np.random.default_rng(n + nblk)
    w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    if kind == "wide":
        w = (w * np.float32(10.0) ** rng.integers(-30, 30, n)).astype(np.float32)
    if kind == "zeros_subnormal":
        w[::3] = 0.0
        w[1::7] = np.float32(1e-40)
    bits = w.view(np.uint32)
    if bf16:
        bits = bits & np.uint32(0xFFFF0000)
    s_hat, depth = _absmean_estimate(bits, 8 if bf16 else 4, nblk)
    beta = 2.0 * depth * 2.0 ** -53
    exact = _exact_abs_sum(bits)
    lo = Fraction(s_hat) * (1 - Fraction(beta)) - Fraction(n) * Fraction(1, 2 ** 126)
    hi = Fraction(s_hat) * (1 + Fraction(beta))
    assert lo <= exact <= hi


def _subln_estimate(x: np.ndarray, threads: int = 128):
    """S_hat of the CTA-per-row SubLN kernel: per-thread FMA chains, warp butterflies, four warps."""
    xd = _abs_double(x.view(np.uint32))
    chains = []
    for t in range(threads):
        acc = 0.0
        for k in range(t, x.size, threads):
            # the kernel's fma: xd^2 has at most 48 significant bits, so it is
            # exact in double and the fma rounds once, as this addition does
            acc = acc + float(xd[k]) * float(xd[k])
        chains.append(acc)
    warps = [_butterfly(chains[w * 32:(w + 1) * 32]) for w in range(threads // 32)]
    s = warps[0]
    for w in warps[1:]:
        s = s + w
    return s


@pytest.mark.parametrize("K,kind", [(2560, "normal"), (9728, "wide"), (4096, "zeros_subnormal")])
def test_subln_sum_of_squares_bound_holds(K, kind):
    rng = np.random.default_rng(K)
    x = rng.standard_normal(K).astype(np.float32)
    if kind == "wide":
        x = (x * np.float32(10.0) ** rng.integers(-15, 15, K)).astype(np.float32)
    if kind == "zeros_subnormal":
        x[::5] = 0.0
        x[2::11] = np.float32(3e-39)
    s_hat = _subln_estimate(x)
    exact = sum(Fraction(float(v)) ** 2 for v in x.astype(np.float64))
    beta = 2.0 * (K + 256) * 2.0 ** -53
    lo = Fraction(s_hat) * (1 - Fraction(beta)) - Fraction(K) * Fraction(1, 2 ** 250)
    hi = Fraction(s_hat) * (1 + Fraction(beta))
    assert lo <= exact <= hi


def test_the_bound_is_tight_enough_to_decide_almost_always():
    """For the layer shapes the relative bound is far below a float's half-ulp
    (2^-25): the exact fallback is a rare event, not the common path."""
    for n, epv, nblk in ((9728 * 2560, 8, 296), (2048 * 768, 4, 296), (1536 * 1536, 8, 296)):
        vpt = -(-(n // epv) // (nblk * WQ_THREADS))
        depth = vpt * epv // 2 + 64 + -(-nblk // WQ_PACK_THREADS)
        assert 2.0 * depth * 2.0 ** -53 < 2.0 ** -40
    assert 2.0 * (24576 + 256) * 2.0 ** -53 < 2.0 ** -37
