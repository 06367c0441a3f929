"""Property pins for the CPU oracle (hypothesis, CPU only): symmetries that
the definitions fix exactly, whatever the data.

- step 2 (per-token absmax INT8, "BitDistill" Evaluation and results, with
  the SubLN RMSNorm of "SLM750-Edge" section 2.1): negating a row negates
  x_q and keeps s; permuting the k axis (with the SubLN gain) permutes x_q
  and keeps s; scaling a row by 2^j leaves x_q unchanged and divides s by
  2^j, and with SubLN (eps = 0) leaves both unchanged, because every
  rounding step commutes with exact power-of-two scaling;
- step 1 (absmean, "Distillix" README 1. BitNet b1.58 Core): negating W
  negates W_q and keeps gamma; permuting rows and columns permutes W_q and
  keeps gamma (the sum of |w| is exact, so its order cannot matter);
- steps 4-5 ("bitone" README, Forward pass): the exact contraction is
  linear in x_q, and the rescale is odd in acc.

Each property catches a class of plausible oracle mistakes: a sign
dropped or a |.| missing, an index transposed or a gain applied to the
wrong k, a sum rounded in the wrong precision or order, an eps applied
in the wrong place.
"""
from __future__ import annotations

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _rows(seed: int, M: int, K: int, spread: int) -> np.ndarray:
    """float32 rows with magnitudes over 2^-spread .. 2^spread, some exact zeros."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)) * np.exp2(rng.integers(-spread, spread + 1, (M, K)))
    x[rng.random((M, K)) < 0.05] = 0.0
    return x.astype(np.float32)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 4), k64=st.integers(1, 6), spread=st.integers(0, 40),
       subln=st.booleans())
def test_act_quant_sign_symmetry(seed, M, k64, spread, subln):
    K = 64 * k64
    X = _rows(seed, M, K, spread)
    gain = (np.random.default_rng(seed + 1).random(K) * 0.2 + 0.9).astype(np.float32) if subln else None
    xq, s = oracle.quant_act(X, gain, 1e-6)
    xq_n, s_n = oracle.quant_act(-X, gain, 1e-6)
    assert np.array_equal(xq_n, -xq)
    assert np.array_equal(s_n.view(np.uint32), s.view(np.uint32))
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 4), k64=st.integers(1, 6), spread=st.integers(0, 40),
       subln=st.booleans())
def test_act_quant_permutation_equivariance(seed, M, k64, spread, subln):
    K = 64 * k64
    X = _rows(seed, M, K, spread)
    rng = np.random.default_rng(seed + 2)
    gain = (rng.random(K) * 0.2 + 0.9).astype(np.float32) if subln else None
    perm = rng.permutation(K)
    xq, s = oracle.quant_act(X, gain, 1e-6)
    xq_p, s_p = oracle.quant_act(X[:, perm], None if gain is None else gain[perm], 1e-6)
    assert np.array_equal(xq_p, xq[:, perm])
    assert np.array_equal(s_p.view(np.uint32), s.view(np.uint32))


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 3), k64=st.integers(1, 4), j=st.integers(-16, 30))
def test_act_quant_power_of_two_scaling(seed, M, k64, j):
    K = 64 * k64
    X = _rows(seed, M, K, 8)
    X[:, 0] = 1.5  # max|x| >= 1.5: above the 1e-5 floor of s also after scaling down by 2^16
    Xs = (X.astype(np.float64) * 2.0 ** j).astype(np.float32)
    assert np.array_equal(Xs.astype(np.float64), X.astype(np.float64) * 2.0 ** j)  # exact, no subnormals
    xq, s = oracle.quant_act(X)
    xq_s, s_s = oracle.quant_act(Xs)
    assert np.array_equal(xq_s, xq)
    assert np.array_equal(s_s.astype(np.float64) * 2.0 ** j, s.astype(np.float64))
    # with SubLN and eps = 0 the normalised row itself is scale free
    gain = (np.random.default_rng(seed + 3).random(K) * 0.2 + 0.9).astype(np.float32)
    yq, t = oracle.quant_act(X, gain, 0.0)
    yq_s, t_s = oracle.quant_act(Xs, gain, 0.0)
    assert np.array_equal(yq_s, yq)
    assert np.array_equal(t_s.view(np.uint32), t.view(np.uint32))


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), N=st.integers(1, 40), k64=st.integers(1, 4), spread=st.integers(0, 30))
def test_weight_quant_sign_and_permutation(seed, N, k64, spread):
    K = 64 * k64
    W = _rows(seed, N, K, spread)
    packed, gamma, wq = oracle.quant_weights(W)
    _, gamma_n, wq_n = oracle.quant_weights(-W)
    assert np.float32(gamma_n).view(np.uint32) == np.float32(gamma).view(np.uint32)
    assert np.array_equal(wq_n, -wq)
    rng = np.random.default_rng(seed + 4)
    pr, pc = rng.permutation(N), rng.permutation(K)
    _, gamma_p, wq_p = oracle.quant_weights(W[pr][:, pc])
    assert np.float32(gamma_p).view(np.uint32) == np.float32(gamma).view(np.uint32)
    assert np.array_equal(wq_p, wq[pr][:, pc])
    assert set(np.unique(wq).tolist()) <= {-1, 0, 1}
    assert packed.shape == (N, K // 4)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 5), N=st.integers(1, 30), k64=st.integers(1, 4))
def test_contraction_linear_and_rescale_odd(seed, M, N, k64):
    K = 64 * k64
    rng = np.random.default_rng(seed)
    x1 = rng.integers(-63, 64, (M, K)).astype(np.int8)
    x2 = rng.integers(-64, 64, (M, K)).astype(np.int8)
    wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
    a1, a2 = oracle.contract(x1, wq), oracle.contract(x2, wq)
    a12 = oracle.contract((x1.astype(np.int16) + x2).astype(np.int8), wq)
    assert np.array_equal(a12, a1 + a2)
    s = (rng.random(M) + 0.5).astype(np.float32)
    gamma = np.float32(rng.random() * 0.05 + 1e-5)
    Y = oracle.rescale(a1, gamma, s[:, None])
    Yn = oracle.rescale(-a1, gamma, s[:, None])
    assert np.array_equal(Yn, -Y)
