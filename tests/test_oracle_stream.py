"""Pins of the oracle's streaming refine rule (seeded maximum), the reading of LoopKV §3.3
"Read-time V precision" and §3.4 (seed from the sink maximum, fallback that marks every
token hot) that the streaming reader will be checked against: S_stream contains S_exact.

The exact rule it must reduce to is the oracle's decode_row refine set, pinned in
test_oracle_decode.py."""
import numpy as np
import pytest

from oracle import oracle as O

TAU = 0.1  # ln(0.1) = -2.302585...


def _hand_scores():
    # group 0: tokens 0, 1, 2 at 0, -2.0, -2.5; group 1: tokens 32, 33, 34 at 1.0, -1.0, -1.5;
    # every other token far below (-10).  Exact maximum 1.0: hot iff s >= 1 - 2.3026.
    s = np.full(64, -10.0)
    s[[0, 1, 2, 32, 33, 34]] = [0.0, -2.0, -2.5, 1.0, -1.0, -1.5]
    return s


def test_hand_worked_running_maximum():
    s = _hand_scores()
    # group 0 read first with no seed: its own maximum 0 makes token 1 (-2.0 >= -2.30) hot as
    # well; group 1 then sees the row maximum 1.0 -> tokens 32, 33
    assert list(O.stream_refine(s, [0, 1], -np.inf, TAU)) == [0b011, 0b011]
    # group 1 first: the running maximum is already the row's -> the exact set {0} | {32, 33}
    assert list(O.stream_refine(s, [1, 0], -np.inf, TAU)) == [0b001, 0b011]
    # a seed of 0.5 (a sink maximum below the row's): group 0 tested against 0.5 -> {0}
    assert list(O.stream_refine(s, [0, 1], 0.5, TAU)) == [0b001, 0b011]


def test_hand_worked_seed_only():
    s = _hand_scores()
    # the fallback seed -inf marks every token hot
    assert list(O.stream_refine(s, [0, 1], -np.inf, TAU, running=False)) == [0xFFFFFFFF, 0xFFFFFFFF]
    # seed 0.5 alone: hot iff s >= 0.5 - 2.3026 = -1.80 -> {0}, {32, 33, 34}
    assert list(O.stream_refine(s, [0, 1], 0.5, TAU, running=False)) == [0b001, 0b111]
    # the exact maximum as the seed gives the exact set
    assert list(O.stream_refine(s, [1, 0], 1.0, TAU, running=False)) == [0b001, 0b011]


def _row(seed, T=256, D=64):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((T, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    v = rng.standard_normal((T, D)).astype(np.float32)
    q = rng.standard_normal(D)
    hist = O.HeadHistory(k, v, 4)
    tail_k = rng.standard_normal((5, D))
    tail_v = rng.standard_normal((5, D))
    return q, hist, tail_k, tail_v


def _bits(words, n):
    return np.array([(int(words[t // 32]) >> (t % 32)) & 1 for t in range(n)], bool)


@pytest.mark.parametrize("seed", range(6))
def test_superset_of_the_exact_set(seed):
    q, hist, tk, tv = _row(seed)
    tau = [0.01, 0.05, 0.3][seed % 3]
    res = O.decode_row(q, hist, tk, tv, tau)
    T = hist.T
    with np.errstate(divide="ignore"):
        s = res["m"] + np.log(res["r"][:T])  # scores of the history, natural-log units
    exact = _bits(res["s_bits"], T)
    rng = np.random.default_rng(100 + seed)
    for _ in range(8):
        order = rng.permutation(T // 32)
        m0 = res["m"] - rng.uniform(0.0, 6.0) if rng.random() < 0.8 else -np.inf
        for running in (True, False):
            got = _bits(O.stream_refine(s, order, m0, tau, running), T)
            assert np.all(got[exact]), "a token of the exact set is missing from the streamed set"


@pytest.mark.parametrize("seed", range(4))
def test_exact_maximum_as_seed_reduces_to_the_exact_rule(seed):
    q, hist, tk, tv = _row(seed + 10)
    tau = 0.02
    res = O.decode_row(q, hist, tk, tv, tau)
    T = hist.T
    with np.errstate(divide="ignore"):
        s = res["m"] + np.log(res["r"][:T])
    exact = _bits(res["s_bits"], T)
    away = np.abs(res["r"][:T] - tau) > 1e-9 * tau  # rounding of s = m + ln r stays off ties
    for running in (True, False):
        got = _bits(O.stream_refine(s, np.arange(T // 32)[::-1], res["m"], tau, running), T)
        assert np.array_equal(got[away], exact[away])


def test_higher_seed_gives_a_subset():
    q, hist, tk, tv = _row(42)
    res = O.decode_row(q, hist, tk, tv, 0.05)
    T = hist.T
    with np.errstate(divide="ignore"):
        s = res["m"] + np.log(res["r"][:T])
    order = np.arange(T // 32)
    for running in (True, False):
        prev = None
        for m0 in (-np.inf, res["m"] - 8, res["m"] - 4, res["m"] - 1, res["m"]):
            cur = _bits(O.stream_refine(s, order, m0, 0.05, running), T)
            if prev is not None:
                assert np.all(prev[cur]), "a higher seed added a token"
            prev = cur


def test_malformed_order_is_rejected():
    s = np.zeros(64)
    for order in ([0, 0], [0], [0, 2], [-1, 0]):
        with pytest.raises(ValueError):
            O.stream_refine(s, order, 0.0, 0.1)
