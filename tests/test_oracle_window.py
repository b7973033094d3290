"""Pins of the oracle's sliding-window decode (decode_row with hist_first): history tokens
before the window are not attended; the row maximum, the refine set and the output run over
the attended tokens only (the sliding-window layers of the Dory model, LoopKV §2.1).

Checked against scaled_dot_product_attention on the dequantized tensors sliced to the window
(tau = 0: every attended 4-bit token full; tau > 1: every one mid-bin), against a refine set
rebuilt in NumPy from independently computed scores, and for the degenerate windows.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _keys(h):
    g = np.arange(h.T) // 32
    return _f16(h.kz)[g] + _f16(h.ks)[g] * h.kc.astype(np.float64)


def _values(h, hot):
    j = np.arange(h.D) // 32
    z, s = _f16(h.vz)[:, j], _f16(h.vs)[:, j]
    full = z + s * h.vc.astype(np.float64)
    if h.bits == 2:
        return full
    return np.where(hot[:, None], full, z + s * (4.0 * (h.vc >> 2).astype(np.float64) + 1.5))


def _sdpa(q, K, V):
    t = lambda a: torch.tensor(a, dtype=torch.float64).view(1, 1, -1, a.shape[-1])  # noqa: E731
    return torch.nn.functional.scaled_dot_product_attention(t(q[None]), t(K), t(V)).view(-1).numpy()


def _row(seed, T=320, D=64, n_tail=11, bits=4):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((T, D)) * np.exp(rng.standard_normal(D))[None, :]).astype(np.float32)
    v = rng.standard_normal((T, D)).astype(np.float32)
    h = O.HeadHistory(k, v, bits)
    tk = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    tv = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal(D).astype(np.float32).astype(np.float64)
    return q, h, tk, tv


@pytest.mark.parametrize("first", [0, 1, 31, 32, 45, 200, 319])
@pytest.mark.parametrize("bits,tau", [(4, 0.0), (4, 2.0), (2, 0.0)])
def test_window_matches_library_attention(first, bits, tau):
    q, h, tk, tv = _row(first * 3 + bits, bits=bits)
    res = O.decode_row(q, h, tk, tv, tau, hist_first=first)
    hot = np.full(h.T, tau <= 0.0)
    K = np.concatenate([_keys(h)[first:], tk])
    V = np.concatenate([_values(h, hot)[first:], tv])
    assert np.allclose(res["o"], _sdpa(q, K, V), rtol=0, atol=1e-12)
    assert np.all(res["r"][:first] == 0.0)
    bits_set = np.array([(int(res["s_bits"][t // 32]) >> (t % 32)) & 1 for t in range(h.T)], bool)
    assert not bits_set[:first].any()


def test_window_zero_is_the_full_decode():
    q, h, tk, tv = _row(5)
    a = O.decode_row(q, h, tk, tv, 0.02)
    b = O.decode_row(q, h, tk, tv, 0.02, hist_first=0)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["s_bits"], b["s_bits"])


@pytest.mark.parametrize("tau", [0.01, 0.05, 0.3])
@pytest.mark.parametrize("first", [17, 64, 250])
def test_window_refine_set_from_independent_scores(tau, first):
    q, h, tk, tv = _row(int(tau * 1000) + first, D=128)
    s = np.concatenate([_keys(h) @ q, tk @ q]) / math.sqrt(128)
    att = np.arange(s.size) >= first
    m = s[att].max()  # the maximum over the attended tokens only
    w = np.where(att, np.exp(s - m), 0.0)
    ref_hot = (w[: h.T] >= tau) & att[: h.T]
    res = O.decode_row(q, h, tk, tv, tau, hist_first=first)
    got = np.array([(int(res["s_bits"][t // 32]) >> (t % 32)) & 1 for t in range(h.T)], bool)
    clear = np.abs(w[: h.T] - tau) > 1e-9
    assert np.array_equal(got[clear], ref_hot[clear])
    ref = _sdpa(q, np.concatenate([_keys(h)[first:], tk]), np.concatenate([_values(h, ref_hot)[first:], tv]))
    assert np.allclose(res["o"], ref, rtol=0, atol=1e-12)


def test_window_degenerate_cases():
    q, h, tk, tv = _row(9, n_tail=0)
    with pytest.raises(ValueError):  # a window that leaves no token
        O.decode_row(q, h, tk, tv, 0.0, hist_first=h.T)
    with pytest.raises(ValueError):
        O.decode_row(q, h, tk, tv, 0.0, hist_first=h.T + 1)
    # only the tail attended
    q, h, tk, tv = _row(10, n_tail=5)
    res = O.decode_row(q, h, tk, tv, 0.0, hist_first=h.T)
    assert np.allclose(res["o"], _sdpa(q, tk, tv), rtol=0, atol=1e-13)
