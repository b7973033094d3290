"""Pins of the oracle's binary16 conversions against NumPy's float16 and a brute-force search.

The directed roundings (toward -inf for the zero point, toward +inf for the scale) are the
reading of the quantizer's rounding rule; they are checked here against an exhaustive table
of every finite binary16 value, and the nearest-even rounding against NumPy's conversion.
"""
import numpy as np
import pytest

from oracle import oracle as O

ALL = np.arange(65536, dtype=np.uint32).astype(np.uint16)
VALS = ALL.view(np.float16).astype(np.float64)
FINITE = np.unique(VALS[np.isfinite(VALS)])  # sorted, -0 and +0 merged


def test_decode_every_pattern_matches_numpy():
    for h in range(0, 65536, 1):
        got = O.f16_to_f64(h)
        ref = VALS[h]
        if np.isnan(ref):
            assert np.isnan(got)
        else:
            assert got == ref and np.signbit(got) == np.signbit(ref), hex(h)


def _probe_values(rng):
    xs = [0.0, -0.0, 1.0, -1.0, 65504.0, -65504.0, 65519.9, 65520.0, 65536.0, 1e6, -1e6,
          2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, -(2.0 ** -25), 2.0 ** -14, 2.0 ** -14 - 2.0 ** -30]
    fin = FINITE[(FINITE != 0)]
    pick = rng.choice(fin.size - 1, 3000)
    a, b = fin[pick], fin[pick + 1]
    xs += list(a) + list((a + b) / 2) + list(a + (b - a) * 1e-3) + list(b - (b - a) * 1e-3)
    xs += list(rng.standard_normal(2000) * np.exp(rng.uniform(-20, 12, 2000)))
    return np.array(xs, dtype=np.float64)


@pytest.mark.parametrize("direction", [-1, 1])
def test_directed_rounding_brute_force(direction):
    rng = np.random.default_rng(1)
    for x in _probe_values(rng):
        got = O.f16_to_f64(O.f64_to_f16(x, direction))
        if direction < 0:
            cand = FINITE[FINITE <= x]
            ref = cand[-1] if cand.size else -np.inf
            if x > 65504:
                ref = 65504.0
        else:
            cand = FINITE[FINITE >= x]
            ref = cand[0] if cand.size else np.inf
            if x < -65504:
                ref = -65504.0
        assert got == ref, (x, got, ref)


def test_nearest_even_matches_numpy():
    rng = np.random.default_rng(2)
    for x in _probe_values(rng):
        got = O.f16_to_f64(O.f64_to_f16(x, 0))
        with np.errstate(over="ignore"):
            ref = float(np.float64(x).astype(np.float16))
        assert got == ref or (np.isinf(got) and np.isinf(ref) and np.sign(got) == np.sign(ref)), (x, got, ref)
