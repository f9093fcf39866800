"""Pins of the reference oracle to facts outside itself.

Each ``pin_*`` function checks the oracle against something the pages or the
mathematics fix: hand-worked cases (``tests/golden``), closed forms, exact
rational arithmetic, invariants, a textbook routine (numpy integer matmul,
Python's half-even ``round``) or a statistical law.  They raise
AssertionError on a mismatch.  ``test_oracle_pins.py`` runs them against the
oracle; ``test_oracle_mutants.py`` runs them against deliberately broken
copies of the oracle source to show that each plausible mistake is caught.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction as F

import numpy as np

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _exact_mean(W):
    return sum(F(float(v)) for v in np.abs(W).ravel()) / W.size


def _half_even(fr: F) -> int:
    return round(fr)  # Fraction.__round__ rounds half to even, exactly


# ---------------------------------------------------------------- hand cases
def pin_hand_4x8():
    """Hand-worked N=4, K=8 case; every 0.5 is a tie (pins half-even)."""
    g = _golden("hand_4x8.json")
    W = np.array(g["W"], np.float32)
    codes, mean = orc.ternarize(W)
    assert mean == g["mean_abs"], mean
    assert codes.tolist() == g["codes"], codes
    out = orc.ternary_linear(np.array(g["x"], np.float32), codes, mean)
    assert out["amax"].tolist() == g["amax"]
    assert out["q"].tolist() == g["q"], out["q"]
    assert out["acc"].tolist() == g["acc"], out["acc"]
    assert out["y"].tolist() == g["y"], out["y"]
    assert codes.tolist() != g["half_away"]["codes"]
    assert out["q"].tolist() != g["half_away"]["q"]


def pin_hand_2x8_scaled():
    """Hand-worked case with mean = 0.25, amax = 64 and an all-zero token."""
    g = _golden("hand_2x8_scaled.json")
    W = np.array(g["W"], np.float32)
    codes, mean = orc.ternarize(W)
    assert mean == g["mean_abs"], mean
    assert codes.tolist() == g["codes"], codes
    out = orc.ternary_linear(np.array(g["x"], np.float32), codes, mean)
    assert out["amax"].tolist() == g["amax"]
    assert out["q"].tolist() == g["q"], out["q"]
    assert out["acc"].tolist() == g["acc"], out["acc"]
    den = g["y_den"]
    for m, row in enumerate(g["y_num"]):
        for n, num in enumerate(row):
            want = num / den
            got = out["y"][m, n]
            assert abs(got - want) <= 1e-14 * max(1.0, abs(want)), (m, n, got, want)


# ---------------------------------------------------------------- closed forms
def pin_zero_weights():
    """W = 0: mean floors at 1e-5, all codes 0, y = 0 for any x."""
    W = np.zeros((5, 12), np.float32)
    codes, mean = orc.ternarize(W)
    assert mean == 1e-5
    assert not codes.any()
    x = np.linspace(-3, 4, 3 * 12, dtype=np.float32).reshape(3, 12)
    out = orc.ternary_linear(x, codes, mean)
    assert not out["acc"].any() and not out["y"].any()


def pin_zero_codes_any_x():
    """All-zero codes give acc = 0 and y = 0."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 40)).astype(np.float32)
    out = orc.ternary_linear(x, np.zeros((7, 40), np.int8), 0.37)
    assert not out["acc"].any() and not out["y"].any()


def pin_identity_like():
    """W = diag(+-c) (K x K): mean = c/K, diagonal codes +-1, acc = +-q."""
    K, c = 16, 0.75
    signs = np.array([1, -1] * (K // 2), np.float32)
    W = np.diag(signs * c).astype(np.float32)
    codes, mean = orc.ternarize(W)
    assert mean == c / K
    assert (codes == np.diag(signs).astype(np.int8)).all()
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, K)) * 5).astype(np.float32)
    out = orc.ternary_linear(x, codes, mean)
    assert (out["acc"] == out["q"].astype(np.int32) * signs.astype(np.int32)).all()
    want = out["q"] * signs[None, :] * (out["amax"][:, None].astype(np.float64) / 127.0) * (c / K)
    assert np.allclose(out["y"], want, rtol=1e-14, atol=0)


def pin_mean_bruteforce():
    """mean|W| equals the exact rational mean, correctly rounded to fp64, on
    tiny dyadic matrices (the sums are exact; only the division rounds)."""
    cases = [
        np.array([[-0.625]], np.float32),
        np.array([[1.5, -0.25, 3.0], [0.125, -2.0, 0.0]], np.float32),
        np.array(_golden("hand_4x8.json")["W"], np.float32) * np.float32(0.375),
    ]
    for W in cases:
        got = orc.mean_abs(W)
        assert got == float(_exact_mean(W)), (W, got)


def pin_mean_random_bound():
    """On random fp32 data the fp64 mean is within 1e-13 of the exact mean."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((37, 53)) * 0.02).astype(np.float32)
    exact = _exact_mean(W)
    got = F(orc.mean_abs(W))
    assert abs(got - exact) <= exact * F(1, 10**13)


def pin_codes_match_exact_rounding():
    """Codes equal clip(round_half_even(W / mean_exact)) away from ties."""
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((23, 41)) * 0.02).astype(np.float32)
    codes, mean = orc.ternarize(W)
    m = _exact_mean(W)
    for (n, k), v in np.ndenumerate(W):
        r = F(float(v)) / m
        frac = abs(r) - math.floor(abs(r))
        if abs(frac - F(1, 2)) < F(1, 10**9):
            continue
        want = max(-1, min(1, _half_even(r)))
        assert codes[n, k] == want, (n, k, v)


def pin_clip():
    """A dominating weight is clipped to +-1; small ones round to 0."""
    W = np.array([[10.0, 0.1, -0.1, 0.1], [0.1, -10.0, 0.1, 0.1]], np.float32)
    codes, mean = orc.ternarize(W)
    assert codes.tolist() == [[1, 0, 0, 0], [0, -1, 0, 0]], codes


def pin_quant_exact_rounding():
    """q is the half-even rounding of the exact x*127/amax (fp32 scale
    error < 1e-5 away from ties), and |q| reaches 127 at the absmax entry."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((6, 97)) * rng.uniform(0.01, 50, (6, 1))).astype(np.float32)
    q, amax = orc.quantize_act(x)
    assert (amax == np.abs(x).max(axis=1)).all()
    for (m, k), v in np.ndenumerate(x):
        r = F(float(v)) * 127 / F(float(amax[m]))
        frac = abs(r) - math.floor(abs(r))
        if abs(frac - F(1, 2)) < F(1, 10**5):
            continue
        assert q[m, k] == _half_even(r), (m, k, v, q[m, k], float(r))
    assert (np.abs(q).max(axis=1) == 127).all()


def pin_quant_unit_scale_is_round():
    """amax = 127 makes the scale exactly 1: q = Python round(x) (half-even)."""
    x = np.array([[127.0, -0.5, 0.5, 1.5, 2.5, -3.5, 4.49, -126.5]], np.float32)
    q, amax = orc.quantize_act(x)
    assert amax[0] == 127.0
    assert q[0].tolist() == [round(float(v)) for v in x[0]], q


def pin_zero_token():
    """amax = 0 gives q = 0 and y = 0 (no NaN)."""
    x = np.zeros((2, 16), np.float32)
    x[1, 3] = -2.0
    codes = np.ones((3, 16), np.int8)
    out = orc.ternary_linear(x, codes, 0.5)
    assert out["amax"][0] == 0.0 and not out["q"][0].any()
    assert np.isfinite(out["y"]).all() and not out["y"][0].any()


def pin_rescale_exact():
    """y equals acc * amax/127 * mean in exact arithmetic to 1e-15."""
    rng = np.random.default_rng(6)
    acc = rng.integers(-2_000_000, 2_000_000, (4, 9)).astype(np.int32)
    amax = rng.uniform(0.1, 300, 4).astype(np.float32)
    mean = 0.0160957
    y = orc.rescale(acc, amax, mean)
    for (m, n), a in np.ndenumerate(acc):
        want = F(int(a)) * F(float(amax[m])) / 127 * F(mean)
        if want == 0:
            assert y[m, n] == 0
        else:
            assert abs(F(float(y[m, n])) - want) <= abs(want) * F(1, 10**15)


# ---------------------------------------------------------------- library / invariants
def pin_acc_numpy_matmul():
    """acc equals an int64 numpy matmul on non-square shapes (catches a
    transposed operand, a dropped term or a wrong sign)."""
    rng = np.random.default_rng(7)
    for (M, N, K) in [(1, 5, 7), (3, 11, 64), (5, 2, 130)]:
        codes = rng.integers(-1, 2, (N, K)).astype(np.int8)
        q = rng.integers(-128, 128, (M, K)).astype(np.int8)
        acc = orc.ternary_acc(codes, q)
        want = q.astype(np.int64) @ codes.astype(np.int64).T
        assert (acc == want).all(), (M, N, K)


def pin_scale_invariance():
    """W*2^j keeps the codes and scales mean by 2^j exactly; x*2^j keeps q."""
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((13, 29)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, 29)).astype(np.float32)
    c0, m0 = orc.ternarize(W)
    q0, a0 = orc.quantize_act(x)
    for j in (-3, 1, 5):
        c1, m1 = orc.ternarize(W * np.float32(2.0 ** j))
        assert (c1 == c0).all() and m1 == m0 * 2.0 ** j
        q1, a1 = orc.quantize_act(x * np.float32(2.0 ** j))
        assert (q1 == q0).all() and (a1 == a0 * np.float32(2.0 ** j)).all()


def pin_permutation_and_negation():
    """A joint permutation of K leaves acc unchanged, negated codes negate
    acc, and a code-only permutation (a 64-vs-128 block mis-read) changes it."""
    rng = np.random.default_rng(9)
    K = 256
    codes = rng.integers(-1, 2, (6, K)).astype(np.int8)
    q = rng.integers(-127, 128, (2, K)).astype(np.int8)
    acc = orc.ternary_acc(codes, q)
    perm = rng.permutation(K)
    assert (orc.ternary_acc(codes[:, perm], q[:, perm]) == acc).all()
    assert (orc.ternary_acc(-codes, q) == -acc).all()
    blk = np.arange(K).reshape(-1, 2, 64)[:, ::-1, :].ravel()
    assert (orc.ternary_acc(codes[:, blk], q) != acc).any()


def pin_acc_bound():
    """|acc| <= 127 * nnz(row) (|q| <= 127 after absmax quantisation)."""
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((9, 300)) * 0.02).astype(np.float32)
    x = rng.standard_normal((4, 300)).astype(np.float32)
    codes, mean = orc.ternarize(W)
    out = orc.ternary_linear(x, codes, mean)
    nnz = (codes != 0).sum(axis=1)
    assert (np.abs(out["acc"]) <= 127 * nnz[None, :]).all()
    assert np.abs(out["q"]).max() <= 127


def pin_gaussian_code_statistics():
    """For W ~ N(0, s^2): P(code = 0) = erf(0.5*sqrt(2/pi)/sqrt(2)) ~ 0.3101,
    P(+1) = P(-1) ~ 0.3449, within 5 standard errors."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((512, 1024)) * 0.02).astype(np.float32)
    codes, mean = orc.ternarize(W)
    n = codes.size
    p0 = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    for val, p in ((0, p0), (1, (1 - p0) / 2), (-1, (1 - p0) / 2)):
        frac = float((codes == val).mean())
        se = math.sqrt(p * (1 - p) / n)
        assert abs(frac - p) < 5 * se, (val, frac, p)


def pin_end_to_end_bruteforce():
    """Tiny layer computed with exact rationals reproduces codes, q and acc
    (entries within 1e-6 of a rounding tie are not expected on random data)."""
    rng = np.random.default_rng(12)
    N, K, M = 3, 9, 2
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    codes, mean = orc.ternarize(W)
    out = orc.ternary_linear(x, codes, mean)
    me = _exact_mean(W)
    ce = [[max(-1, min(1, _half_even(F(float(v)) / me))) for v in row] for row in W]
    qe = []
    for row in x:
        a = max(abs(F(float(v))) for v in row)
        qe.append([_half_even(F(float(v)) * 127 / a) for v in row])
    acce = [[sum(c * qq for c, qq in zip(cr, qr)) for cr in ce] for qr in qe]
    assert codes.tolist() == ce
    assert out["q"].tolist() == qe
    assert out["acc"].tolist() == acce
    for m in range(M):
        for n in range(N):
            want = F(acce[m][n]) * max(abs(F(float(v))) for v in x[m]) / 127 * me
            got = F(float(out["y"][m, n]))
            assert abs(got - want) <= abs(want) * F(1, 10**12) + F(1, 10**30)


def pin_nonfinite_weight_rejected():
    W = np.ones((2, 4), np.float32)
    W[1, 2] = np.inf
    try:
        orc.ternarize(W)
    except ValueError:
        return
    raise AssertionError("non-finite W accepted")


# ---------------------------------------------- decoder-layer chain stand-ins
def pin_gqa_expand_hand():
    """Hand-worked identity attention: 4 query heads of 2 channels over 2 KV
    heads (groups of 2), then one KV head shared by all, then groups of 1."""
    v = np.array([[10, 11, 20, 21], [30, 31, 40, 41]], np.float32)
    assert orc.gqa_expand(v, 8, 2).tolist() == [
        [10, 11, 10, 11, 20, 21, 20, 21],
        [30, 31, 30, 31, 40, 41, 40, 41]]
    assert orc.gqa_expand(v[:, :2], 8, 2).tolist() == [
        [10, 11] * 4, [30, 31] * 4]
    assert orc.gqa_expand(v, 4, 2).tolist() == v.tolist()


def pin_add_f32_ieee():
    """Single-precision addition: numpy's float32 add, and the half-even
    ties 1 + 2^-24 = 1 and 1 + 3*2^-24 = 1 + 2^-22."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal(1000).astype(np.float32)
    y = (rng.standard_normal(1000) * 1e-3).astype(np.float32)
    assert np.array_equal(orc.add_f32(x, y), x + y)
    one = np.ones(2, np.float32)
    t = np.array([2.0 ** -24, 3 * 2.0 ** -24], np.float32)
    assert orc.add_f32(one, t).tolist() == [1.0, 1.0 + 2.0 ** -22]


def pin_silu_closed_forms():
    """SiLU(0) = 0; SiLU(z) - SiLU(-z) = z; the logistic form z * expit(z)
    (scipy); large |z| gives z and -0."""
    from scipy.special import expit
    one = np.ones(1, np.float32)
    assert orc.silu_mul(np.zeros(1, np.float32), one)[0] == 0.0
    z = np.random.default_rng(12).uniform(-20, 20, 500).astype(np.float32)
    ones = np.ones_like(z)
    sp, sm = orc.silu_mul(z, ones), orc.silu_mul(-z, ones)
    assert np.allclose(sp - sm, z.astype(np.float64), rtol=1e-14, atol=1e-14)
    ref = z.astype(np.float64) * expit(z.astype(np.float64))
    assert np.allclose(sp, ref, rtol=1e-14, atol=1e-300)
    big = np.array([1000.0, -1000.0], np.float32)
    assert orc.silu_mul(big, np.ones(2, np.float32)).tolist() == [1000.0, 0.0]


def pin_silu_mul_linear_in_u():
    """SiLU(g) * u scales with u: u = 0 gives 0, u = c gives c * SiLU(g)."""
    rng = np.random.default_rng(13)
    g = rng.standard_normal(200).astype(np.float32)
    u = rng.standard_normal(200).astype(np.float32)
    base = orc.silu_mul(g, np.ones_like(g))
    assert np.array_equal(orc.silu_mul(g, u), base * u.astype(np.float64))
    assert not orc.silu_mul(g, np.zeros_like(u)).any()


def _chain_layer(rng, hidden, kv, inter, zero=()):
    shapes = {"q": (hidden, hidden), "k": (kv, hidden), "v": (kv, hidden),
              "o": (hidden, hidden), "gate": (inter, hidden), "up": (inter, hidden),
              "down": (hidden, inter)}
    layer = {}
    for name, (N, K) in shapes.items():
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        if name in zero:
            W[:] = 0
        layer[name] = orc.ternarize(W)
    return layer


def pin_decoder_layer_zero_weights():
    """All seven projections zero: every intermediate is zero and the layer
    returns its input exactly (the residuals add +0)."""
    rng = np.random.default_rng(14)
    layer = _chain_layer(rng, 256, 128, 512, zero=("q", "k", "v", "o", "gate", "up", "down"))
    h = rng.standard_normal((3, 256)).astype(np.float32)
    out = orc.decoder_layer(h, layer)
    for name in ("q", "k", "v", "a", "o", "g", "u", "act", "d"):
        assert not out[name].any(), name
    assert np.array_equal(out["h1"], h) and np.array_equal(out["h_next"], h)


def pin_decoder_layer_attention_reads_v():
    """Identity attention passes v only: with v zero (q, k random) the
    attention block adds nothing, h1 == h; with v random it does."""
    rng = np.random.default_rng(15)
    h = rng.standard_normal((2, 256)).astype(np.float32)
    zero_v = orc.decoder_layer(h, _chain_layer(rng, 256, 128, 512, zero=("v",)))
    assert np.array_equal(zero_v["h1"], h)
    with_v = orc.decoder_layer(h, _chain_layer(rng, 256, 128, 512))
    assert not np.array_equal(with_v["h1"], h)


# ------------------------------------------------ I8_S linear (R17-R19)
def pin_i8_hand_3x8():
    """Hand-worked I8_S case: ties pin half-even for weights and tokens, the
    dyadic scales pin both /127 factors, the bias signs pin ReLU."""
    g = _golden("hand_i8_3x8.json")
    W = (np.array(g["W128"], np.float64) / 128.0).astype(np.float32)
    wq, amax_w = orc.i8_quantize_weights(W)
    assert float(amax_w) == g["amax_w"], amax_w
    assert wq.tolist() == g["wq"], wq
    assert wq.tolist() != g["wq_half_away"]
    x = np.array(g["x"], np.float32)
    bias = np.array(g["bias"], np.float32)
    out = orc.i8_linear(x, wq, amax_w, bias, relu=True)
    assert out["amax"].tolist() == g["amax_x"]
    assert out["q"].tolist() == g["q"], out["q"]
    assert out["acc"].tolist() == g["acc"], out["acc"]
    assert out["y"].tolist() == g["y_relu"], out["y"]
    lin = orc.i8_linear(x, wq, amax_w, bias, relu=False)
    assert lin["y"].tolist() == g["y_linear"], lin["y"]


def pin_i8_weight_quant_is_the_fp32_rule():
    """wq = half-even(fl(W * fl(127 / max|W|))) with IEEE fp32 operations
    (numpy's float32 arithmetic and rint), amax_w = max|W| exactly; |wq| <= 127."""
    rng = np.random.default_rng(17)
    for shape in [(7, 40), (1, 128), (33, 96)]:
        W = (rng.standard_normal(shape) * 0.05).astype(np.float32)
        W[rng.integers(shape[0]), rng.integers(shape[1])] = -0.25   # the extreme is negative
        wq, amax_w = orc.i8_quantize_weights(W)
        a = np.float32(np.abs(W).max())
        assert amax_w == a
        scale = np.float32(127.0) / a
        want = np.clip(np.rint(W * scale), -128, 127).astype(np.int8)
        assert (wq == want).all()
        assert np.abs(wq.astype(np.int32)).max() == 127


def pin_i8_acc_numpy_matmul():
    """acc of full-range int8 weights and tokens equals numpy's int64 matmul."""
    rng = np.random.default_rng(18)
    wq = rng.integers(-127, 128, (9, 200)).astype(np.int8)
    q = rng.integers(-128, 128, (5, 200)).astype(np.int8)
    acc = orc.ternary_acc(wq, q)
    assert (acc == q.astype(np.int64) @ wq.astype(np.int64).T).all()


def pin_i8_epilogue_closed_forms():
    """Zero weights give relu(bias); no bias equals a zero bias; ReLU is
    max(0, linear); a bias far below the products zeroes every output."""
    rng = np.random.default_rng(19)
    M, N, K = 4, 6, 64
    x = rng.standard_normal((M, K)).astype(np.float32)
    bias = np.array([-2.0, -0.5, 0.0, 0.25, 1.0, 3.0], np.float32)
    z = orc.i8_linear(x, np.zeros((N, K), np.int8), np.float32(0.5), bias, relu=True)
    assert (z["y"] == np.maximum(0.0, bias.astype(np.float64))[None, :]).all()
    zl = orc.i8_linear(x, np.zeros((N, K), np.int8), np.float32(0.5), bias, relu=False)
    assert (zl["y"] == bias.astype(np.float64)[None, :]).all()
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    a = orc.i8_linear(x, wq, np.float32(0.3), None, relu=False)["y"]
    b = orc.i8_linear(x, wq, np.float32(0.3), np.zeros(N, np.float32), relu=False)["y"]
    assert (a == b).all()
    r = orc.i8_linear(x, wq, np.float32(0.3), bias, relu=True)["y"]
    l = orc.i8_linear(x, wq, np.float32(0.3), bias, relu=False)["y"]
    assert (r == np.maximum(0.0, l)).all() and (l < 0).any() and (l > 0).any()
    low = orc.i8_linear(x, wq, np.float32(0.3), np.full(N, -1e6, np.float32), relu=True)["y"]
    assert not low.any()


def pin_i8_linear_exact_fraction():
    """y against exact rational arithmetic on a tiny case: within 1e-15 of
    the magnitudes summed (|product| + |bias|; the bias may cancel)."""
    rng = np.random.default_rng(20)
    W = (rng.standard_normal((3, 16)) * 0.03).astype(np.float32)
    x = rng.standard_normal((2, 16)).astype(np.float32)
    bias = np.array([0.125, -0.03, 0.0], np.float32)
    wq, aw = orc.i8_quantize_weights(W)
    out = orc.i8_linear(x, wq, aw, bias, relu=False)
    for m in range(2):
        for n in range(3):
            acc = sum(int(out["q"][m, k]) * int(wq[n, k]) for k in range(16))
            assert acc == out["acc"][m, n]
            prod = F(acc) * F(float(out["amax"][m])) / 127 * F(float(aw)) / 127
            exact = prod + F(float(bias[n]))
            got = out["y"][m, n]
            bound = F(1, 10**15) * (abs(prod) + abs(F(float(bias[n]))))
            assert abs(F(got) - exact) <= bound, (m, n, got, float(exact))


def pin_i8_scale_invariance():
    """Scaling W by 2^j leaves wq unchanged and scales amax_w, and the
    bias-free outputs, by exactly 2^j."""
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((5, 48)) * 0.02).astype(np.float32)
    x = rng.standard_normal((3, 48)).astype(np.float32)
    wq, aw = orc.i8_quantize_weights(W)
    y = orc.i8_linear(x, wq, aw, None, relu=False)["y"]
    for j in (-3, 5):
        wq2, aw2 = orc.i8_quantize_weights((W * np.float32(2.0 ** j)).astype(np.float32))
        assert (wq2 == wq).all() and aw2 == np.float32(aw * 2.0 ** j)
        y2 = orc.i8_linear(x, wq2, aw2, None, relu=False)["y"]
        assert (y2 == y * 2.0 ** j).all()


# ------------------------------------------------ tensor-parallel split (R20)
def pin_quantize_given_own_amax_is_r4():
    """With each row's own absmax the given-scale rule is the R4 quantiser;
    a larger given amax follows the fp32 rule (numpy float32 division,
    product and rint) and never clips."""
    rng = np.random.default_rng(30)
    x = rng.standard_normal((5, 96)).astype(np.float32)
    x[2] = 0.0
    q, amax = orc.quantize_act(x)
    assert (orc.quantize_act_given(x, amax) == q).all()
    big = (amax * np.float32(3.0)).astype(np.float32)
    got = orc.quantize_act_given(x, big)
    for m in range(5):
        if big[m] == 0:
            assert not got[m].any()
            continue
        scale = np.float32(127.0) / big[m]
        assert (got[m] == np.rint(x[m] * scale).astype(np.int8)).all()
    assert np.abs(got.astype(np.int32)).max() <= 43   # 127 / 3, rounded


def pin_row_parallel_slices_sum_to_the_row():
    """Slices of a token row quantised with the whole row's absmax, summed
    over their partial accumulators, give the unsplit layer exactly."""
    rng = np.random.default_rng(31)
    N, K, M = 24, 512, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    codes, mean = orc.ternarize(W)
    full = orc.ternary_linear(x, codes, mean)
    bounds = [0, 128, 384, 512]
    amax = np.max([np.abs(x[:, a:b]).max(axis=1) for a, b in zip(bounds, bounds[1:])], axis=0)
    assert (amax == full["amax"]).all()
    acc = sum(orc.ternary_acc(codes[:, a:b], orc.quantize_act_given(x[:, a:b], amax))
              for a, b in zip(bounds, bounds[1:]))
    assert (acc == full["acc"]).all()
    assert (orc.rescale(acc, amax, mean) == full["y"]).all()


ALL_PINS = {name: fn for name, fn in sorted(globals().items())
            if name.startswith("pin_") and callable(fn)}
