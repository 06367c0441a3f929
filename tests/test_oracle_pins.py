"""Pins for the CPU oracle: checks against what the source pages and the
mathematics fix, never against the oracle's own formulas.

Each test says which plausible oracle mistake it would catch.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# -- independent exact helpers (Fractions, integer rounding) ------------------

def f32_rne(fr: Fraction) -> float:
    """Float32 nearest to the rational ``fr`` (ties to even), by integer
    arithmetic; an implementation independent of the oracle's C code."""
    if fr == 0:
        return 0.0
    sign = -1.0 if fr < 0 else 1.0
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = max(e - 23, -149)
    scaled = a / (Fraction(2) ** q)
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * 2.0 ** q


def rne_int(fr: Fraction) -> int:
    n = math.floor(fr)
    rem = fr - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def exact_abs_sum(w: np.ndarray) -> Fraction:
    return sum((Fraction(float(abs(x))) for x in w.ravel()), Fraction(0))


def read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split("#")[0].strip() for ln in f if ln.split("#")[0].strip()]


# -- gamma ---------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["normal", "wide", "subnormal", "huge"])
def test_abs_sum_is_exact(kind):
    """Exact sum|W| vs Fraction arithmetic.  Catches a dropped limb carry, a
    wrong exponent bias, mishandled subnormals."""
    rng = np.random.default_rng(7)
    if kind == "normal":
        w = rng.standard_normal(3000).astype(np.float32) * 0.02
    elif kind == "wide":
        w = (rng.standard_normal(3000) * 2.0 ** rng.integers(-60, 60, 3000)).astype(np.float32)
    elif kind == "subnormal":
        w = (rng.standard_normal(500) * 1e-40).astype(np.float32)
        w = np.concatenate([w, np.array([1.0, -2.0 ** -149], dtype=np.float32)])
    else:
        w = (rng.standard_normal(500) * 1e37).astype(np.float32)
        w = np.concatenate([w, np.array([3.4e38, -3.4e38], dtype=np.float32)])
    S = exact_abs_sum(w)
    limbs = oracle.abs_sum_exact_limbs(w)
    as_int = sum(v << (64 * i) for i, v in enumerate(limbs))
    assert Fraction(as_int, 2 ** 149) == S
    # one RNE rounding to double == Python's correctly rounded float(Fraction)
    assert oracle.limbs_to_double(limbs, -149) == float(S)


def test_limbs_to_double_ties_to_even():
    """Integer-to-double rounding: halfway cases go to the even mantissa."""
    two53 = 1 << 53
    for v in [two53 + 1, two53 + 3, (two53 + 1) << 70, (1 << 120) + (1 << 67), (1 << 120) + (1 << 67) + 1]:
        limbs = [(v >> (64 * i)) & (2 ** 64 - 1) for i in range(5)]
        assert oracle.limbs_to_double(limbs, 0) == float(v)  # Python int->float is RNE


def test_gamma_constant_magnitude():
    """Constant-magnitude W = +-c gives gamma = |c| (+1e-5) and W_q = sign(W)
    ("Distillix" 1. BitNet b1.58 Core).  Catches a missing +1e-5, a sum over
    signed instead of absolute values, a wrong divisor n."""
    rng = np.random.default_rng(3)
    for c in [0.02, 0.015, 1.0, 3.0e-3, 7.5]:
        signs = rng.choice([-1.0, 1.0], size=(37, 64))
        W = (signs * c).astype(np.float32)
        g = oracle.absmean_gamma(W)
        assert g == np.float32(np.float32(c) + np.float32(1e-5))
        q = oracle.ternarize(W, g)
        assert np.array_equal(q, signs.astype(np.int8))


def test_gamma_random_vs_fraction():
    """gamma = float32(double(S)/n) + 1e-5f, S from Fractions."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((48, 80)) * 0.02).astype(np.float32)
    S = exact_abs_sum(W)
    mean_f = np.float32(float(S) / W.size)
    assert oracle.absmean_gamma(W) == np.float32(mean_f + np.float32(1e-5))


# -- ternarize -----------------------------------------------------------------

def test_round_clip_golden():
    for ln in read_golden("round_clip_cases.txt"):
        w, g, want = ln.split()
        q = oracle.ternarize(np.array([float(w)], dtype=np.float32), np.float32(float(g)))
        assert int(q[0]) == int(want), ln


def test_round_clip_case_form_near_threshold():
    """Against the case form of the SLM750-Edge card (+1 if x > 0.5, 0 if
    |x| <= 0.5, else -1) on x = RNE32(w / gamma) computed with Fractions, for
    w straddling 0.5*gamma.  Catches round-half-up, a <= / < swap, double
    instead of float division."""
    rng = np.random.default_rng(5)
    gammas = np.array([0.0123456, 0.02, 1.0 / 3.0, 0.75, 7.0], dtype=np.float32)
    for g in gammas:
        t = np.float32(g * np.float32(0.5))
        ws = [t]
        a = t
        b = t
        for _ in range(6):
            a = np.nextafter(a, np.float32(np.inf))
            b = np.nextafter(b, np.float32(0))
            ws += [a, b]
        ws += list((rng.standard_normal(50) * g).astype(np.float32))
        w = np.array(ws + [-x for x in ws], dtype=np.float32)
        q = oracle.ternarize(w, g)
        for wi, qi in zip(w, q):
            x = f32_rne(Fraction(float(wi)) / Fraction(float(g)))
            want = 1 if x > 0.5 else (0 if abs(x) <= 0.5 else -1)
            assert int(qi) == want, (wi, g, x)


def test_ternary_distribution_gaussian():
    """Gaussian W: P(W_q = 0) = P(|z| <= sqrt(2/pi)/2) = erf(1/(2 sqrt(pi)))
    ~ 0.3101 (gamma ~ sigma sqrt(2/pi)); +-1 split the rest evenly."""
    W = workloads.normal((1000, 1000), 0.02, seed=123).numpy()
    g = oracle.absmean_gamma(W)
    q = oracle.ternarize(W, g)
    n = q.size
    p0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    tol = 6 * math.sqrt(p0 * (1 - p0) / n)
    assert abs((q == 0).mean() - p0) < tol
    assert abs((q == 1).mean() - (1 - p0) / 2) < tol
    assert abs((q == -1).mean() - (1 - p0) / 2) < tol


def test_ternary_distribution_trained_split():
    """The 125M decode workload's weights reproduce the 29/42/29 split of the
    "Distillix 125M" Model Stats after quantization (W_q = sign(W) for
    constant magnitude)."""
    want = {int(v): float(f) for v, f in (ln.split() for ln in read_golden("weight_distribution.txt"))}
    W = workloads.ternary_weights(768, 2048, seed=9).numpy()
    q = oracle.quant_weights(W)[2]
    n = q.size
    for v, f in want.items():
        tol = 6 * math.sqrt(f * (1 - f) / n)
        assert abs((q == v).mean() - f) < tol


# -- packing -------------------------------------------------------------------

def test_pack_golden_and_size():
    rows = dict(ln.split(":", 1) for ln in read_golden("linear_small.txt"))
    wq = np.array([[int(v) for v in rows["Wq0"].split()], [int(v) for v in rows["Wq1"].split()]],
                  dtype=np.int8)
    packed = oracle.pack(wq)
    want = np.array([[int(b, 16) for b in rows["P0"].split()], [int(b, 16) for b in rows["P1"].split()]],
                    dtype=np.uint8)
    assert np.array_equal(packed, want)
    assert packed.nbytes == wq.size // 4


def test_pack_roundtrip_and_bits_per_weight():
    """pack o unpack = identity; 2 bits per weight, inside the 1.58..2 bits
    the pages state, and 8x smaller than FP16 ("bitone" memory table gives
    ~10x at 1.6 bits)."""
    rng = np.random.default_rng(1)
    q = rng.integers(-1, 2, size=(33, 256)).astype(np.int8)
    p = oracle.pack(q)
    assert np.array_equal(oracle.unpack(p, 256), q)
    bits = 8 * p.nbytes / q.size
    assert bits == 2.0
    assert math.log2(3) <= bits <= 2.0
    for ln in read_golden("model_sizes.txt"):
        params, fp16_gb, bitone_gb = (float(v) for v in ln.split())
        page_bits = 8 * bitone_gb * 1e9 / params
        assert 1.5 < page_bits <= bits  # the pages' 1.6 bits < our 2 bits
        ours_gb = params * bits / 8 / 1e9
        assert abs(fp16_gb / ours_gb - 8.0) < 1e-9


def test_unpack_rejects_reserved_code():
    p = np.full((1, 4), 0x55, dtype=np.uint8)  # sixteen zero weights
    assert np.array_equal(oracle.unpack(p, 16), np.zeros((1, 16), np.int8))
    p[0, 2] = 0x57  # k = 2 gets code 11
    with pytest.raises(oracle.OracleError):
        oracle.unpack(p, 16)


# -- activation quant --------------------------------------------------------

def test_act_quant_golden():
    lines = read_golden("act_quant_cases.txt")
    for i in range(0, len(lines), 3):
        x = np.array([[float(v) for v in lines[i].split(":")[1].split()]], dtype=np.float32)
        want = [int(v) for v in lines[i + 1].split(":")[1].split()]
        s_want = float(lines[i + 2].split(":")[1])
        xq, s = oracle.quant_act(x)
        assert xq[0].tolist() == want
        assert float(s[0]) == s_want


def test_act_quant_properties():
    """argmax -> +-127 exactly; x -> 2^j x leaves x_q unchanged; all-zero row
    gives s = float32(127 / float32(1e-5)) and x_q = 0.  Catches max over
    signed values, truncation instead of rounding, a wrong clamp."""
    X = workloads.with_outlier_channels(workloads.normal((9, 256), 1.0, 5), 3, 20.0, 6).numpy()
    X[8] = 0.0
    xq, s = oracle.quant_act(X)
    for m in range(8):
        k = int(np.argmax(np.abs(X[m])))
        assert xq[m, k] == (127 if X[m, k] > 0 else -127)
        assert np.abs(xq[m]).max() == 127
    assert np.all(xq[8] == 0)
    assert s[8] == np.float32(f32_rne(Fraction(127) / Fraction(float(np.float32(1e-5)))))
    for j in (-3, 5):
        xq2, s2 = oracle.quant_act((X[:8] * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(xq2, xq[:8])
        assert np.array_equal(s2, (s[:8] * np.float32(2.0 ** -j)).astype(np.float32))


def test_act_quant_vs_fraction():
    """x_q = RNE(RNE32(x * s)), s = RNE32(127 / a), all with Fractions."""
    X = workloads.normal((4, 64), 1.0, 8).numpy()
    xq, s = oracle.quant_act(X)
    for m in range(4):
        a = max(abs(Fraction(float(v))) for v in X[m])
        s_ref = f32_rne(Fraction(127) / max(a, Fraction(float(np.float32(1e-5)))))
        assert float(s[m]) == s_ref
        for k in range(64):
            t = f32_rne(Fraction(float(X[m, k])) * Fraction(s_ref))
            assert int(xq[m, k]) == max(-128, min(127, rne_int(Fraction(t))))


# -- SubLN ---------------------------------------------------------------------

def test_rmsnorm_constant_row_closed_form():
    """x = c, g = 1: y = c / sqrt(c^2 + eps) (closed form)."""
    for c in [0.5, 3.0, 1e-3]:
        K = 512
        y = oracle.rmsnorm(np.full(K, c, np.float32), np.ones(K, np.float32), 1e-6)
        ref = c / math.sqrt(c * c + 1e-6)
        assert np.all(np.abs(y.astype(np.float64) - ref) <= 4 * np.spacing(np.float32(ref)))
        xq, _ = oracle.quant_act(np.full((1, K), c, np.float32), np.ones(K, np.float32), 1e-6)
        assert np.all(xq == 127)


def test_rmsnorm_vs_fraction():
    """ms = float32(double(exact sum x^2) / K); r = sqrtf(ms + eps);
    y = float32(float32(x / r) * g), with Fractions and an exact
    integer square root for the correctly rounded sqrt."""
    x = workloads.student_t((96,), 3, 0.5, 4, torch.bfloat16).float().numpy()
    g = workloads.uniform((96,), 0.9, 1.1, 5).numpy()
    eps = np.float32(1e-6)
    S2 = sum((Fraction(float(v)) ** 2 for v in x), Fraction(0))
    ms = f32_rne(Fraction(float(S2)) / 96)
    arg = f32_rne(Fraction(ms) + Fraction(float(eps)))
    # correctly rounded float32 sqrt: compare candidates by exact squares
    r0 = np.float32(math.sqrt(arg))
    cands = [np.nextafter(r0, np.float32(0)), r0, np.nextafter(r0, np.float32(np.inf))]
    r = min(cands, key=lambda c: abs(Fraction(float(c)) ** 2 - Fraction(arg)))
    y = oracle.rmsnorm(x, g, 1e-6)
    for k in range(96):
        t = f32_rne(Fraction(float(x[k])) / Fraction(float(r)))
        want = f32_rne(Fraction(t) * Fraction(float(g[k])))
        assert float(y[k]) == want


# -- contraction and rescale -------------------------------------------------

def test_contraction_add_subtract_identity():
    """Y_int = sum of x_q over +1 weights - sum over -1 weights ("bitone",
    How 1.58-bit Works), via masked numpy sums; and int64 torch matmul.
    Non-square shapes catch a transposed operand."""
    rng = np.random.default_rng(2)
    M, N, K = 5, 7, 96
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    acc = oracle.contract(xq, wq)
    x64 = xq.astype(np.int64)
    ident = np.stack([np.stack([x64[m][wq[n] == 1].sum() - x64[m][wq[n] == -1].sum() for n in range(N)])
                      for m in range(M)])
    assert np.array_equal(acc, ident)
    tm = torch.from_numpy(x64) @ torch.from_numpy(wq.astype(np.int64)).T
    assert np.array_equal(acc, tm.numpy())
    pairs = oracle.contract_pairs(xq, wq, [0, 4, 2], [6, 0, 3])
    assert pairs.tolist() == [acc[0, 6], acc[4, 0], acc[2, 3]]


def test_contraction_brute_force_tiny():
    """Every ternary row of length 4 against a few x_q rows, by a literal
    nested sum."""
    import itertools
    wq = np.array(list(itertools.product([-1, 0, 1], repeat=4)), dtype=np.int8)
    xq = np.array([[1, 2, 3, 4], [-128, 127, 0, -1], [5, -5, 5, -5]], dtype=np.int8)
    acc = oracle.contract(xq, wq)
    for m in range(3):
        for n in range(81):
            s = 0
            for k in range(4):
                s += int(xq[m, k]) * int(wq[n, k])
            assert acc[m, n] == s


def test_contract_blas_equals_the_integer_loop():
    """The BLAS form of the contraction (float32 matmul, exact below 2^24)
    against the int64 loop and the add/subtract identity, on ragged
    non-square shapes (a transposed operand or a dropped column fails)."""
    rng = np.random.default_rng(7)
    for M, N, K in ((37, 53, 448), (1, 5, 64), (9, 300, 2048)):
        xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
        wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        got = oracle.contract_blas(xq, wq)
        assert got.shape == (M, N) and got.dtype == np.int64
        assert np.array_equal(got, oracle.contract(xq, wq))
    x64 = xq.astype(np.int64)
    ident = np.stack([(x64 * (wq[n] == 1)).sum(1) - (x64 * (wq[n] == -1)).sum(1) for n in range(N)], axis=1)
    assert np.array_equal(got, ident)


def test_contract_blas_extreme_sums_and_bound():
    """|acc| = 128 K at the largest K the library takes (closed form), and
    refusal where float32 partial sums could round."""
    K = 32768
    xq = np.full((2, K), -128, dtype=np.int8)
    xq[1] = 127
    wq = np.full((3, K), -1, dtype=np.int8)
    wq[1] = 1
    wq[2, ::2] = 0
    got = oracle.contract_blas(xq, wq)
    want = np.array([[128 * K, -128 * K, 64 * K], [-127 * K, 127 * K, -127 * K // 2]], dtype=np.int64)
    assert np.array_equal(got, want)
    with pytest.raises(oracle.OracleError):
        oracle.contract_blas(np.zeros((1, 1 << 17), np.int8), np.zeros((1, 1 << 17), np.int8))


def test_rescale_hand_values():
    acc = np.array([254, 0, -6], dtype=np.int64)
    Y = oracle.rescale(acc, np.float32(0.5), np.array([127.0, 3.0, 1.0], dtype=np.float32))
    assert Y.tolist() == [1.0, 0.0, -3.0]


def test_linear_small_golden():
    rows = dict(ln.split(":", 1) for ln in read_golden("linear_small.txt"))
    W = np.array([[float(v) for v in rows["W0"].split()], [float(v) for v in rows["W1"].split()]],
                 dtype=np.float32)
    X = np.array([[float(v) for v in rows["X"].split()]], dtype=np.float32)
    out = oracle.linear(W, X)
    mean = np.float32(float(rows["mean"]))
    assert out["gamma"] == np.float32(mean + np.float32(1e-5))
    assert 0.22461 < float(out["gamma"]) < 0.22462
    assert out["packed"].tolist() == [[int(b, 16) for b in rows["P0"].split()],
                                      [int(b, 16) for b in rows["P1"].split()]]
    assert out["xq"][0].tolist() == [int(v) for v in rows["Xq"].split()]
    assert float(out["s"][0]) == float(rows["s"])
    assert out["acc"][0].tolist() == [int(v) for v in rows["acc"].split()]
    assert out["Y"][0].tolist() == [a * float(out["gamma"]) for a in (-6.0, -183.0)]


# -- FFN activation (ReLU^2-gated) feeding the down projection ---------------

def test_ffn_act_relu_closed_forms():
    """relu(g)^2 * u: g <= 0 gives 0; g = 1 gives u; g = 2^k gives u * 4^k
    exactly (SLM750-Edge, Key Architectural Features: ReLU2)."""
    rng = np.random.default_rng(7)
    u = rng.standard_normal(64).astype(np.float32)
    for g0 in (-3.5, -1e-30, -0.0, 0.0):
        h = oracle.ffn_act(np.full(64, g0, np.float32), u)
        assert np.all(h == 0.0)
    assert np.array_equal(oracle.ffn_act(np.ones(64, np.float32), u), u)
    for k in range(-10, 11):
        g = np.full(64, 2.0 ** k, np.float32)
        assert np.array_equal(oracle.ffn_act(g, u), (u.astype(np.float64) * 4.0 ** k).astype(np.float32))


def test_ffn_act_two_roundings_exact():
    """Each product of two floats is exact in double (48-bit mantissa), so
    float(float(r * r) * u) is two correctly rounded conversions of exact
    products."""
    rng = np.random.default_rng(8)
    g = (rng.standard_normal(4096) * 3).astype(np.float32)
    u = (rng.standard_normal(4096) * 2).astype(np.float32)
    h = oracle.ffn_act(g, u)
    for gi, ui, hi in zip(g.tolist(), u.tolist(), h.tolist()):
        r = gi if gi > 0 else 0.0
        sq = float(np.float32(r * r))          # r * r exact in double, one rounding to float
        want = float(np.float32(sq * ui))      # sq * u exact in double, one rounding
        assert hi == want or (hi == 0.0 and want == 0.0)


def test_ffn_act_quant_constant_row():
    """gate = 2, up = c on every element: h = 4c, so every x_q is +-127 and
    s = 127 / (4|c|); with SubLN (gain 1) y = h / sqrt(h^2 + eps) per element."""
    c = np.float32(0.375)
    g = np.full((2, 256), 2.0, np.float32)
    u = np.full((2, 256), c, np.float32)
    u[1] = -c
    xq, s = oracle.ffn_act_quant(g, u)
    assert xq[0].tolist() == [127] * 256 and xq[1].tolist() == [-127] * 256
    assert s.tolist() == [float(np.float32(127.0) / np.float32(1.5))] * 2
    xq2, s2 = oracle.ffn_act_quant(g, u, np.ones(256, np.float32), 1e-6)
    assert xq2[0].tolist() == [127] * 256 and xq2[1].tolist() == [-127] * 256


# -- exact ties that the GPU parity cases build ---------------------------------

def _midpoint_weights(n: int) -> np.ndarray:
    # n/2 - 1 entries of 2, one of 1, one of -1, one of -2^-24 n, the rest 0:
    # sum |W| = n (1 + 2^-24), so sum |W| / n lies exactly halfway between
    # 1 and the next float 1 + 2^-23
    w = np.zeros(n, dtype=np.float32)
    w[: n // 2 - 1] = 2.0
    w[n // 2 - 1] = 1.0
    w[n // 2] = -1.0
    w[n // 2 + 1] = -(2.0 ** -24) * n
    return w


@pytest.mark.parametrize("n", [64, 256, 64 * 4096])
def test_gamma_at_an_exact_midpoint_ties_to_even(n):
    """mean|W| exactly halfway between two floats rounds to the even one
    (1.0), so gamma = 1 + 1e-5 in float: an oracle that summed |W| in float
    or double with rounding (landing on either side) or rounded the mean
    away from zero would give the odd neighbour's gamma."""
    w = _midpoint_weights(n)
    assert exact_abs_sum(w) == n * (1 + Fraction(1, 2 ** 24))
    assert oracle.absmean_gamma(w) == np.float32(np.float32(1.0) + np.float32(1e-5))
    assert oracle.absmean_gamma(w) != np.float32(np.float32(1.0 + 2.0 ** -23) + np.float32(1e-5))


@pytest.mark.parametrize("K", [1024, 2048, 4096])
def test_subln_at_an_exact_midpoint_ties_to_even(K):
    """Row [8, 2^-9, 0, ...]: sum x^2 / K = (64 + 2^-18) / K, exactly halfway
    between two floats for K a power of two; ms rounds to the even one
    (64 / K), then r = sqrtf(ms + eps) and y follow (checked by Fractions)."""
    x = np.zeros(K, dtype=np.float32)
    x[0], x[1] = 8.0, 2.0 ** -9
    g = np.ones(K, dtype=np.float32)
    eps = np.float32(1e-6)
    mid = (Fraction(64) + Fraction(1, 2 ** 18)) / K
    assert f32_rne(mid) == 64.0 / K  # the tie goes to the even float
    arg = f32_rne(Fraction(64, K) + Fraction(float(eps)))
    r0 = np.float32(math.sqrt(arg))
    cands = [np.nextafter(r0, np.float32(0)), r0, np.nextafter(r0, np.float32(np.inf))]
    r = min(cands, key=lambda c: abs(Fraction(float(c)) ** 2 - Fraction(arg)))
    y = oracle.rmsnorm(x, g, 1e-6)
    assert float(y[0]) == f32_rne(Fraction(8) / Fraction(float(r)))
    assert float(y[1]) == f32_rne(Fraction(1, 2 ** 9) / Fraction(float(r)))
    xq, s = oracle.quant_act(x.reshape(1, K), g, 1e-6)
    assert xq[0, 0] == 127 and s[0] == np.float32(np.float32(127.0) / y[0])
