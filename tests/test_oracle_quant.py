"""Pins of the oracle's KIVI-style group quantizer.

Checked against facts that do not depend on the oracle's own code: values built as
zero + scale*k come back as codes k; a constant group has scale 0; the directed roundings
bracket the group (zero <= min, zero + L*scale >= max); every code is the nearest level
under exact rational arithmetic (ties to even), except where the exact quotient lies within
fp32 rounding of a tie; and the reconstruction error is at most half a scale step.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O

F16 = O.f16_bits_to_f64


def _exact_f32(v):
    return float(np.float32(v)) == v


@pytest.mark.parametrize("bits", [4, 2])
def test_construction_recovers_codes(bits):
    L = (1 << bits) - 1
    rng = np.random.default_rng(10 + bits)
    done = 0
    while done < 300:
        z = float(np.float16(rng.normal() * 4))
        s = float(np.float16(abs(rng.normal()) * 0.5 + 1e-3))
        k = rng.integers(0, L + 1, 32)
        k[rng.integers(32)] = 0
        k[rng.integers(32)] = L
        vals = [z + s * int(c) for c in k]
        if not all(_exact_f32(v) for v in vals) or k.min() != 0 or k.max() != L:
            continue
        zb, sb, codes, st = O.quantize_group(np.array(vals, np.float32), bits)
        assert st == O.OK
        assert F16(zb) == z and F16(sb) == s
        assert np.array_equal(codes, k.astype(np.uint8))
        done += 1


def test_constant_group_has_zero_scale():
    # an fp16-representable constant is its own zero point, so (max - zero) / L = 0
    for c in [0.0, 1.0, -3.25, 2.0 ** -24, 123.5]:
        zb, sb, codes, st = O.quantize_group(np.full(32, c, np.float32), 4)
        assert st == O.OK and F16(sb) == 0.0 and not codes.any() and F16(zb) == c
    # otherwise the zero point lies below it and the scale is the smallest step above the gap
    for c in [1e-7, 123.456, -0.3]:
        zb, sb, codes, st = O.quantize_group(np.full(32, c, np.float32), 4)
        z, s = F16(zb), F16(sb)
        assert st == O.OK and z < np.float32(c) and s > 0
        assert abs(np.float32(c) - (z + s * codes.astype(np.float64))).max() <= s / 2


def test_ties_round_to_even():
    # zero = 0 and scale = 1 (max 15, min 0): x = k + 0.5 is an exact tie
    x = np.zeros(32, np.float32)
    x[1] = 15.0
    ties = [0.5, 1.5, 2.5, 3.5, 4.5, 13.5, 14.5]
    x[2:2 + len(ties)] = ties
    zb, sb, codes, st = O.quantize_group(x, 4)
    assert st == O.OK and F16(zb) == 0.0 and F16(sb) == 1.0
    assert list(codes[2:2 + len(ties)]) == [0, 2, 2, 4, 4, 14, 14]


def _nearest_even(fr: Fraction) -> int:
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


@pytest.mark.parametrize("bits", [4, 2])
def test_bracketing_error_bound_and_exact_nearest(bits):
    L = (1 << bits) - 1
    rng = np.random.default_rng(20 + bits)
    near_tie = 0
    for trial in range(400):
        scale = np.exp(rng.normal() * 2)
        x = (rng.standard_normal(32) * scale + rng.normal() * scale).astype(np.float32)
        zb, sb, codes, st = O.quantize_group(x, bits)
        assert st == O.OK
        z, s = F16(zb), F16(sb)
        assert z <= x.min()
        assert z + L * s >= x.max()
        deq = z + s * codes.astype(np.float64)
        assert np.all(np.abs(x - deq) <= s / 2 * (1 + 2.0 ** -20) + 1e-300)
        for xi, ci in zip(x, codes):
            q = (Fraction(float(xi)) - Fraction(float(z))) / Fraction(float(s))
            ref = min(max(_nearest_even(q), 0), L)
            frac = q - (q.numerator // q.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 6) * max(1, abs(q)):
                near_tie += 1
                assert abs(int(ci) - ref) <= 1
            else:
                assert int(ci) == ref, (float(q), ci, ref)


def test_nonfinite_and_range_errors():
    x = np.linspace(-1, 1, 32).astype(np.float32)
    for bad in (np.nan, np.inf, -np.inf):
        y = x.copy()
        y[5] = bad
        zb, sb, codes, st = O.quantize_group(y, 4)
        assert st == O.NONFINITE and zb == 0 and sb == 0 and not codes.any()
    y = x.copy()
    y[0] = -70000.0  # zero point rounds down past the fp16 range
    assert O.quantize_group(y, 4)[3] == O.RANGE
    y = x.copy()
    y[0] = -60000.0
    y[1] = 60000.0 * 16  # (max - min)/15 > 65504
    assert O.quantize_group(y, 4)[3] == O.RANGE
    y = np.full(32, 70000.0, np.float32)  # zero = 65504 is still a valid lower bound
    assert O.quantize_group(y, 4)[3] == O.OK


@pytest.mark.parametrize("bits", [4, 2])
def test_grouping_axes(bits):
    """Keys are grouped per channel over 32 tokens, values per token over 32 channels."""
    rng = np.random.default_rng(3)
    T, D = 64, 64
    k = rng.standard_normal((T, D)).astype(np.float32)
    base = O.quantize_k(k, bits)
    k2 = k.copy()
    k2[37, 5] = 50.0  # token 37 -> group 1, channel 5
    mod = O.quantize_k(k2, bits)
    ds = np.argwhere(base[1] != mod[1])
    assert {tuple(p) for p in ds} <= {(1, 5)} and len(ds) == 1
    v = rng.standard_normal((T, D)).astype(np.float32)
    vb = O.quantize_v(v, bits)
    v2 = v.copy()
    v2[9, 40] = 50.0  # token 9, channel group 1
    vm = O.quantize_v(v2, bits)
    ds = np.argwhere(vb[1] != vm[1])
    assert [tuple(p) for p in ds] == [(9, 1)]
    # per-group quantization equals the single-group routine
    for t in (0, 31, 63):
        zb, sb, codes, _ = O.quantize_group(v[t, 32:64], bits)
        assert vb[2][t, 1] == zb and vb[1][t, 1] == sb and np.array_equal(vb[0][t, 32:64], codes)
