"""Pins for the oracle's INT8 quantiser (CPU only).

Checks against exact cases (a row whose amax is 127 has scale exactly 1, so
the codes are round-half-even of the values), the zero row, the error bound,
and an independent evaluation of every fp32 division in exact rational
arithmetic (Python fractions) followed by round-to-nearest-even.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import quantize_row, dequantize_rows
from oracle.quant import quantize_rows


def _f32_nearest(fr: Fraction) -> float:
    """Round an exact rational to the nearest fp32 (ties to even)."""
    lo = np.float32(float(fr))                       # double rounding is fixed below
    cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - fr),
                                     int(np.float32(c).view(np.uint32)) & 1))
    return float(best)


def _rhe(fr: float) -> int:
    """Round half to even of a float, by exact comparison."""
    f = Fraction(fr)
    fl = f.numerator // f.denominator
    rem = f - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def pin_exact_scale_one(q=quantize_row):
    x = np.array([127, 2.5, 3.5, -2.5, -127, 0, 1.5, 0.5, -0.5, 126.5], np.float16)
    codes, scale = q(x)
    assert scale == np.float32(1.0)
    assert codes.tolist() == [127, 2, 4, -2, -127, 0, 2, 0, 0, 126]


def pin_zero_row(q=quantize_row):
    codes, scale = q(np.zeros(64, np.float16))
    assert scale == 0.0 and not codes.any()


def pin_exact_rational(q=quantize_row):
    rng = np.random.default_rng(5)
    for trial in range(40):
        D = 64 if trial % 2 else 128
        x = (rng.standard_normal(D) * (4.0 if trial % 3 == 0 else 1.0)).astype(np.float16)
        codes, scale = q(x)
        amax = max(abs(float(v)) for v in x)
        exp_scale = _f32_nearest(Fraction(amax) / 127)
        assert float(scale) == exp_scale, trial
        for d in range(D):
            ratio = _f32_nearest(Fraction(float(x[d])) / Fraction(exp_scale))
            exp_code = max(-127, min(127, _rhe(ratio)))
            assert int(codes[d]) == exp_code, (trial, d)


def pin_error_bound(q=quantize_row):
    rng = np.random.default_rng(6)
    for _ in range(50):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 30)).astype(np.float16)
        codes, scale = q(x)
        xh = dequantize_rows(codes[None], np.array([scale]))[0]
        err = np.abs(x.astype(np.float64) - xh.astype(np.float64))
        # half a step, plus fp32 rounding of x/scale and of code*scale (127 * 2^-24 each)
        assert err.max() <= float(scale) * (0.5 + 2 * 127 * 2.0 ** -24)
        assert np.abs(codes.astype(int)).max() == 127
        assert codes.min() >= -127


def pin_division_not_reciprocal(q=quantize_row):
    # Find seeded rows where x/scale and x*(1/scale) round to different codes,
    # then check those codes against the exactly rounded quotient.
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((4000, 128)) * 3).astype(np.float16).astype(np.float32)
    amax = np.abs(x).max(1)
    scale = (amax / np.float32(127)).astype(np.float32)
    div = (x / scale[:, None]).astype(np.float32)
    rec = (x * (np.float32(1) / scale)[:, None]).astype(np.float32)
    rows, cols = np.nonzero(np.rint(div) != np.rint(rec))
    assert rows.size >= 3          # the seed is chosen so that such elements exist
    for r, c in list(zip(rows, cols))[:8]:
        codes, sc = q(x[r].astype(np.float16))
        exact = _f32_nearest(Fraction(float(x[r, c])) / Fraction(float(sc)))
        assert int(codes[c]) == max(-127, min(127, _rhe(exact))), (r, c)


ALL_PINS = [pin_exact_scale_one, pin_zero_row, pin_exact_rational, pin_error_bound,
            pin_division_not_reciprocal]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_quant_pins(pin):
    pin()


def _mutant(kind):
    def q(x16):
        x = np.asarray(x16, np.float16).astype(np.float32)
        amax = np.float32(np.max(np.abs(x)))
        scale = np.float32(amax / np.float32(128.0 if kind == "div128" else 127.0))
        if scale == 0:
            return np.zeros(x.shape, np.int8), np.float32(0)
        if kind == "reciprocal":
            r = (x * np.float32(np.float32(1.0) / scale)).astype(np.float32)
        else:
            r = (x / scale).astype(np.float32)
        if kind == "half_away":
            c = np.sign(r) * np.floor(np.abs(r) + 0.5)
        elif kind == "trunc":
            c = np.trunc(r)
        else:
            c = np.rint(r)
        return np.clip(c, -127, 127).astype(np.int8), scale
    return q


@pytest.mark.parametrize("kind", ["div128", "reciprocal", "half_away", "trunc"])
def test_pins_catch_planted_mistakes(kind):
    bad = _mutant(kind)
    caught = 0
    for pin in ALL_PINS:
        try:
            pin(bad)
        except AssertionError:
            caught += 1
    assert caught >= 1, kind


def test_unmutated_copy_passes():
    for pin in ALL_PINS:
        pin(_mutant("none"))


def test_rows_equal_row_by_row():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((300, 128)) * rng.uniform(0.01, 20, size=(300, 1))).astype(np.float16)
    x[17] = 0
    x[40, :5] = [127, 2.5, 3.5, -2.5, -127]
    codes, scales = quantize_rows(x)
    for i in range(300):
        c1, s1 = quantize_row(x[i])
        assert np.array_equal(codes[i], c1) and scales[i] == s1, i
