"""Pins of the oracle's Jensen-bias terms against closed forms, quadrature and Monte Carlo (no GPU).

b_i = log E[exp(delta_i)] with delta_i the score error of cached key i (agents-report.net,
'KV-Cache 量化導致的 Jensen 偏差', section 方法); its Taylor form is (1/(24 d)) sum_c q_c^2 Delta^2.
"""
import json
import math
from fractions import Fraction
import os

import mpmath
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bias_cases():
    with open(os.path.join(GOLDEN, "bias_worked_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _bias_cases(), ids=lambda c: c["name"])
def test_taylor_worked_examples(case):
    q = np.array([case["q"]])
    step = np.array([case["step"]])
    b = oracle.jensen_bias_taylor(q, step, case["group"], 1.0 / math.sqrt(case["d"]))
    assert b.shape == (1, 1)
    assert b[0, 0] == pytest.approx(case["taylor"], rel=1e-14, abs=1e-300)


def test_log_sinhc_against_mpmath():
    mpmath.mp.dps = 50
    a = np.concatenate([np.geomspace(1e-9, 0.0999, 40), np.geomspace(0.1, 40.0, 60), [0.0, -0.3, -7.0]])
    got = oracle.log_sinhc(a)
    for ai, gi in zip(a, got):
        if ai == 0:
            assert gi == 0.0
            continue
        x = mpmath.mpf(abs(float(ai)))
        want = float(mpmath.log(mpmath.sinh(x) / x))
        assert gi == pytest.approx(want, rel=2e-14), ai


def test_taylor_is_upper_bound_with_quartic_gap():
    """log(sinh a/a) = a^2/6 - a^4/180 + ...: Taylor >= exact, gap <= sum a^4/180, excess -> a^2/30."""
    rng = np.random.default_rng(11)
    d, group = 16, 4
    q = rng.standard_normal((30, d)) * 2
    step = rng.uniform(0.0, 2.0, (20, d // group))
    scale = 1.0 / math.sqrt(d)
    bt = oracle.jensen_bias_taylor(q, step, group, scale)
    be = oracle.jensen_bias_exact(q, step, group, scale)
    dc = np.repeat(step, group, axis=-1)
    a4 = ((0.5 * scale * q[:, None, :] * dc[None]) ** 4).sum(-1) / 180.0
    assert np.all(bt - be >= -1e-15)
    assert np.all(bt - be <= a4 * (1 + 1e-9) + 1e-15)
    # single channel: relative excess of the Taylor term tends to a^2/30
    for a in (1e-2, 3e-2, 1e-1):
        qq = np.zeros((1, 4)); qq[0, 0] = 2 * a / 0.5   # scale 1/2 at d = 4, step 1
        t = oracle.jensen_bias_taylor(qq, np.ones((1, 1)), 4, 0.5)[0, 0]
        e = oracle.jensen_bias_exact(qq, np.ones((1, 1)), 4, 0.5)[0, 0]
        assert t == pytest.approx(a * a / 6, rel=1e-13)
        assert (t - e) / e == pytest.approx(a * a / 30, rel=0.01)


def test_exact_bias_against_monte_carlo():
    """b_exact = log E[exp(scale q.e)] for e_c ~ U(-Delta_c/2, Delta_c/2), by sampling."""
    rng = np.random.default_rng(5)
    d, group = 64, 32
    scale = 1.0 / math.sqrt(d)
    q = rng.standard_normal(d) * np.repeat([1.0, 3.0], 32)
    step = np.array([[0.8, 2.5]])
    n = 400_000
    e = (rng.random((n, d)) - 0.5) * np.repeat(step[0], group)
    delta = scale * e @ q
    w = np.exp(delta)
    est = math.log(w.mean())
    se = w.std() / w.mean() / math.sqrt(n)
    be = oracle.jensen_bias_exact(q[None], step, group, scale)[0, 0]
    bt = oracle.jensen_bias_taylor(q[None], step, group, scale)[0, 0]
    assert abs(est - be) < 4 * se
    assert be > 0.05                          # the test has signal
    assert abs(bt - be) < 0.02 * be           # and Taylor is close at this size


@pytest.mark.parametrize("d", [2, 3])
def test_exact_bias_against_quadrature(d):
    """E[exp(delta)] as a d-dimensional tensor-product Gauss-Legendre integral over the noise cube."""
    x, wts = np.polynomial.legendre.leggauss(40)
    q = np.array([1.7, -2.2, 0.9])[:d]
    step = np.array([[1.3] * d])            # group = 1: one step per channel
    step[0, -1] = 0.4
    scale = 0.8
    half = 0.5 * step[0]
    grids = np.meshgrid(*[x * h for h in half], indexing="ij")
    W = np.ones_like(grids[0])
    for k, wk in enumerate(np.meshgrid(*[wts] * d, indexing="ij")):
        W = W * wk
    delta = scale * sum(q[c] * grids[c] for c in range(d))
    mean = (W * np.exp(delta)).sum() / (2.0 ** d)     # density 1/Delta per channel, dx = half dt
    be = oracle.jensen_bias_exact(q[None], step, 1, scale)[0, 0]
    assert math.log(mean) == pytest.approx(be, rel=1e-12)


def test_exact_bias_through_the_quantiser():
    """Quantise random keys whose group extremes are fixed; the empirical log E[exp(delta)] over keys
    equals the exact bias computed from the quantiser's stored steps (group-to-channel mapping included)."""
    rng = np.random.default_rng(21)
    d, group, bits = 8, 4, 2
    lo = np.array([-1.0, 2.0]); hi = np.array([2.0, 2.6])     # steps 1.0 and 0.2
    n = 300_000
    K = np.empty((n, d), dtype=np.float32)
    for g in range(2):
        sl = slice(g * group, (g + 1) * group)
        block = rng.uniform(lo[g], hi[g], (n, group))
        block[:, 0] = lo[g]; block[:, 1] = hi[g]              # extremes have zero error
        K[:, sl] = block
    codes, step, zp = oracle.quantize(K, bits, group, "f32")
    assert np.allclose(step, step[0]) and np.allclose(zp, zp[0])
    kh = oracle.dequantize(codes, step, zp, group)
    q = np.array([0.0, 0.0, 2.5, -1.5, 0.0, 0.0, 6.0, 4.0])   # zero on the extreme positions
    scale = 1.0 / math.sqrt(d)
    delta = scale * (kh - K.astype(np.float64)) @ q
    w = np.exp(delta)
    est = math.log(w.mean())
    se = w.std() / w.mean() / math.sqrt(n)
    be = oracle.jensen_bias_exact(q[None], step[:1].astype(np.float64), group, scale)[0, 0]
    assert abs(est - be) < 4 * se
    # a swapped group-to-channel mapping would be far outside the error bar
    swapped = oracle.jensen_bias_exact(q[None], step[:1, ::-1].astype(np.float64), group, scale)[0, 0]
    assert abs(swapped - be) > 20 * se


def test_bias_scaling_and_zero():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((5, 32))
    step = rng.uniform(0, 1, (7, 2))
    b1 = oracle.jensen_bias_taylor(q, step, 16, 0.3)
    b3 = oracle.jensen_bias_taylor(3.0 * q, step, 16, 0.3)
    np.testing.assert_allclose(b3, 9.0 * b1, rtol=1e-13)
    assert np.all(oracle.jensen_bias_taylor(q, np.zeros((7, 2)), 16, 0.3) == 0)
    assert np.all(oracle.jensen_bias_exact(q, np.zeros((7, 2)), 16, 0.3) == 0)


# --------------------------------------------------------------------------------------------
# Fourth-order correction (the a^4 term of the series of log(sinh a / a)).
# --------------------------------------------------------------------------------------------
def test_taylor4_worked_example():
    """One channel, q = 2, Delta = 1, scale = 0.5: a = scale q Delta / 2 = 0.5, so
    b = a^2/6 - a^4/180 = 1/24 - 1/2880 = 119/2880 (by hand)."""
    b = oracle.jensen_bias_taylor4(np.array([[2.0]]), np.array([[1.0]]), 1, 0.5)
    assert b.shape == (1, 1)
    assert abs(b[0, 0] - 119.0 / 2880.0) < 1e-15


def test_taylor4_sums_the_channels_of_each_group():
    """Channels of one group share the key's step: b = sum_c (a_c^2/6 - a_c^4/180), checked with
    exact rationals channel by channel."""
    q = np.array([[1.0, 2.0, 3.0, -1.5]])
    step = np.array([[0.75, 1.25]])              # groups of 2 channels
    scale = 0.5
    want = Fraction(0)
    for c, qc in enumerate(q[0]):
        a = Fraction(scale) * Fraction(qc) * Fraction(step[0, c // 2]) / 2
        want += a * a / 6 - a ** 4 / 180
    got = oracle.jensen_bias_taylor4(q, step, 2, scale)[0, 0]
    assert abs(got - float(want)) < 1e-15


@pytest.mark.parametrize("a", [0.02, 0.05, 0.1, 0.2])
def test_taylor4_error_against_mpmath_is_the_sixth_order_term(a):
    """log(sinh a / a) = a^2/6 - a^4/180 + a^6/2835 - ...: the fourth-order form misses the exact
    value by a^6/2835 to leading order (exact value from mpmath at 50 digits)."""
    import mpmath
    mpmath.mp.dps = 50
    exact = float(mpmath.log(mpmath.sinh(a) / a))
    b4 = oracle.jensen_bias_taylor4(np.array([[2.0 * a]]), np.array([[1.0]]), 1, 1.0)[0, 0]
    b2 = oracle.jensen_bias_taylor(np.array([[2.0 * a]]), np.array([[1.0]]), 1, 1.0)[0, 0]
    assert abs((exact - b4) / (a ** 6 / 2835.0) - 1.0) < 0.01 + 2 * a * a
    assert abs(exact - b4) < abs(exact - b2)     # the extra term brings the form closer


def test_taylor4_modes_in_attention():
    """correct = 2 subtracts the fourth-order form, correct = 3 the exact one (oracle only)."""
    rng = np.random.default_rng(3)
    d, group, Lc, Lcur, Lq = 8, 4, 20, 5, 5
    q = rng.normal(size=(Lq, d))
    k_hat = rng.normal(size=(Lc, d))
    v_hat = rng.normal(size=(Lc, d))
    step = rng.uniform(0.2, 1.5, (Lc, d // group))
    kc, vc = rng.normal(size=(Lcur, d)), rng.normal(size=(Lcur, d))
    scale = 1 / math.sqrt(d)
    outs = {}
    for correct in (1, 2, 3):
        outs[correct] = oracle.attention_rows(q, np.arange(Lq), k_hat, v_hat, step, group, kc, vc,
                                              correct, False, scale, Lq)[1]
    b2 = oracle.jensen_bias_taylor(q, step, group, scale)
    b4 = oracle.jensen_bias_taylor4(q, step, group, scale)
    s = scale * q @ k_hat.T
    for correct, b in ((1, b2), (2, b4)):
        s_all = np.concatenate([s - b, scale * q @ kc.T], axis=1)
        lse = np.log(np.exp(s_all).sum(1))
        np.testing.assert_allclose(outs[correct], lse, rtol=0, atol=1e-12)
    # the fourth-order LSE lies between the second-order and the exact one (b2 >= b_exact, b4 <= b_exact
    # for these small a, so LSE(b2) <= LSE(exact) <= LSE(b4))
    assert np.all(outs[1] <= outs[3] + 1e-15) and np.all(outs[3] <= outs[2] + 1e-15)
