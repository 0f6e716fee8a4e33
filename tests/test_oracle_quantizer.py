"""Pins of the oracle's quantiser against hand-derived values and exact arithmetic (no GPU)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases("quantizer_worked_examples.json"), ids=lambda c: c["name"])
def test_worked_examples(case):
    x = np.array([case["x"]], dtype=np.float32)
    codes, step, zp = oracle.quantize(x, case["bits"], case["group"], case["meta"])
    assert codes[0].tolist() == case["codes"]
    np.testing.assert_array_equal(step[0].astype(np.float64), np.array(case["step"]))
    np.testing.assert_array_equal(zp[0].astype(np.float64), np.array(case["zp"]))
    assert oracle.pack_codes(codes, case["bits"])[0].tolist() == case["packed"]
    if "step_f16_bits" in case:
        assert step.dtype == np.float16
        assert step[0].view(np.uint16).tolist() == case["step_f16_bits"]


def _exact_nearest(x, zp, step, bits):
    """Nearest code in exact rational arithmetic, ties to even, clamped; None near a tie."""
    if step == 0:
        return 0
    t = (Fraction(float(x)) - Fraction(float(zp))) / Fraction(float(step))
    fl = t.numerator // t.denominator
    frac = t - fl
    if abs(frac - Fraction(1, 2)) < Fraction(1, 10**5) * max(1, abs(t)):
        return None
    k = fl + (1 if frac > Fraction(1, 2) else 0)
    return int(min(max(k, 0), oracle.levels(bits)))


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("group", [2, 4])
@pytest.mark.parametrize("meta", ["f32", "f16"])
def test_codes_are_nearest_grid_points(bits, group, meta):
    """Each code is the grid point zp + step*c nearest to x (exact arithmetic against the stored meta)."""
    rng = np.random.default_rng(100 + bits * 10 + group + (meta == "f16"))
    x = (rng.standard_normal((400, 4 * group)) * rng.uniform(0.01, 30, (400, 1))).astype(np.float32)
    codes, step, zp = oracle.quantize(x, bits, group, meta)
    n_g = x.shape[1] // group
    checked = 0
    for r in range(x.shape[0]):
        for c in range(x.shape[1]):
            g = c // group
            want = _exact_nearest(x[r, c], np.float32(zp[r, g]), np.float32(step[r, g]), bits)
            if want is None:
                continue
            assert codes[r, c] == want, (r, c, x[r, c], step[r, g], zp[r, g])
            checked += 1
    assert checked > 0.99 * x.size
    assert step.shape == (400, n_g)


@pytest.mark.parametrize("bits", [2, 4])
def test_invariants_fp32_meta(bits):
    rng = np.random.default_rng(7 + bits)
    x = (rng.standard_normal((64, 3, 50, 128)) * 3).astype(np.float32)
    group = 64
    codes, step, zp = oracle.quantize(x, bits, group, "f32")
    xg = x.reshape(64, 3, 50, 2, 64)
    cg = codes.reshape(xg.shape)
    # the group minimum maps to code 0 and the maximum to the top code
    imin = xg.argmin(-1)[..., None]
    imax = xg.argmax(-1)[..., None]
    assert np.all(np.take_along_axis(cg, imin, -1) == 0)
    assert np.all(np.take_along_axis(cg, imax, -1) == oracle.levels(bits))
    # the dequantisation error is at most half a step (fp32 rounding slack)
    xh = oracle.dequantize(codes, step, zp, group)
    err = np.abs(xh - x.astype(np.float64)).reshape(xg.shape)
    bound = 0.5 * step.astype(np.float64)[..., None] * (1 + 1e-5) + 1e-6 * np.abs(xg)
    assert np.all(err <= bound)
    # step is (max-min)/(2^bits-1) to fp32 rounding
    rel = np.abs(step * oracle.levels(bits) - (xg.max(-1) - xg.min(-1))) / (xg.max(-1) - xg.min(-1))
    assert rel.max() < 1e-6


def test_pack_roundtrip_and_bit_order():
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        codes = rng.integers(0, 1 << bits, size=(5, 7, 128), dtype=np.uint8)
        packed = oracle.pack_codes(codes, bits)
        assert packed.shape == (5, 7, 128 * bits // 8)
        np.testing.assert_array_equal(oracle.unpack_codes(packed, bits), codes)
        # channel c sits at bit c*bits of the little-endian row bit string
        bitstr = np.unpackbits(packed, axis=-1, bitorder="little")
        for c in (0, 1, 5, 77, 127):
            val = sum(int(bitstr[2, 3, c * bits + k]) << k for k in range(bits))
            assert val == codes[2, 3, c]


def test_zero_step_group_codes_zero():
    x = np.zeros((2, 64), dtype=np.float32)
    x[1, 32:] = np.linspace(-1, 1, 32, dtype=np.float32)
    codes, step, zp = oracle.quantize(x, 2, 32, "f32")
    assert np.all(codes[0] == 0) and np.all(step[0] == 0)
    assert np.all(codes[1, :32] == 0) and step[1, 0] == 0 and step[1, 1] > 0
