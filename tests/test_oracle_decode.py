"""Pins of the oracle's decode attention.

* tau = 0 marks every history token hot, so the output is plain softmax attention over the
  fully dequantized INT4 cache; tau > 1 marks none, so it is attention over the mid-bin
  (hi-plane) values; a 2-bit cell reads its own codes.  Each case is compared with
  torch.nn.functional.scaled_dot_product_attention in fp64 on the same dequantized tensors
  (a library routine, independent of the oracle's loops).
* Identical keys give uniform weights, so the output is the mean of the values.
* Proposition 1 of the LoopKV paper (Appendix "Proof of Proposition 1"): scores come from the
  full 4-bit keys, so the weights do not depend on tau; a cold token's value moves by at most
  1.5 scale steps, which bounds |o_tau - o_0| by sum over cold tokens of p_t * 1.5 * s_t.
* The refine set shrinks as tau grows, and the normalised-weight test at tau equals the
  row-max test at tau * l.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O


def _case(rng, T, D, n_tail, bits, key_scale=True):
    k = rng.standard_normal((T, D))
    if key_scale:
        k = k * np.exp(rng.standard_normal(D))[None, :]
    v = rng.standard_normal((T, D))
    h = O.HeadHistory(k.astype(np.float32), v.astype(np.float32), bits) if T else None
    tk = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    tv = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal(D).astype(np.float32).astype(np.float64)
    return q, h, tk, tv


def _sdpa(q, K, V):
    qt = torch.tensor(q, dtype=torch.float64).view(1, 1, 1, -1)
    Kt = torch.tensor(K, dtype=torch.float64).view(1, 1, K.shape[0], -1)
    Vt = torch.tensor(V, dtype=torch.float64).view(1, 1, V.shape[0], -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt).view(-1).numpy()


@pytest.mark.parametrize("bits,tau", [(4, 0.0), (4, 2.0), (2, 0.0), (2, 0.3)])
@pytest.mark.parametrize("T,D,n_tail", [(64, 64, 0), (96, 128, 7), (32, 32, 32)])
def test_matches_library_attention(bits, tau, T, D, n_tail):
    rng = np.random.default_rng(T * 7 + D + n_tail + bits)
    q, h, tk, tv = _case(rng, T, D, n_tail, bits)
    res = O.decode_row(q, h, tk, tv, tau)
    hot = np.full(T, tau <= 0.0)
    K = np.concatenate([O.dequant_k(h), tk])
    V = np.concatenate([O.dequant_v(h, hot), tv])
    ref = _sdpa(q, K, V)
    assert np.allclose(res["o"], ref, rtol=0, atol=1e-12)
    n_hot = sum(bin(int(w)).count("1") for w in res["s_bits"])
    assert n_hot == (T if (bits == 4 and tau <= 0) else 0)


def test_tail_only_row():
    rng = np.random.default_rng(4)
    q, _, tk, tv = _case(rng, 0, 64, 5, 4)
    res = O.decode_row(q, None, tk, tv, 0.01)
    assert np.allclose(res["o"], _sdpa(q, tk, tv), atol=1e-13)


def test_identical_keys_give_the_mean():
    rng = np.random.default_rng(6)
    D, T = 64, 64
    k = np.tile(rng.standard_normal(D), (T, 1)).astype(np.float32)
    v = rng.standard_normal((T, D)).astype(np.float32)
    h = O.HeadHistory(k, v, 4)
    q = rng.standard_normal(D)
    res = O.decode_row(q, h, np.zeros((0, D)), np.zeros((0, D)), 0.0)
    assert np.allclose(res["o"], O.dequant_v(h, np.ones(T, bool)).mean(axis=0), atol=1e-13)
    assert np.allclose(res["r"], 1.0) and res["l"] == pytest.approx(T)


@pytest.mark.parametrize("tau", [0.005, 0.01, 0.05, 0.3])
def test_proposition1_bound(tau):
    rng = np.random.default_rng(int(tau * 1000))
    D, T = 128, 256
    q, h, tk, tv = _case(rng, T, D, 9, 4)
    full = O.decode_row(q, h, tk, tv, 0.0)
    res = O.decode_row(q, h, tk, tv, tau)
    assert res["m"] == full["m"] and res["l"] == full["l"]  # weights independent of tau
    hot = np.array([(res["s_bits"][t // 32] >> (t % 32)) & 1 for t in range(T)], bool)
    p = res["r"][:T] / res["l"]
    assert np.all(p[~hot] < tau * p.max() * (1 + 1e-12))
    s = O.f16_bits_to_f64(h.vs)[:, np.arange(D) // 32]  # [T, D] value scale per channel
    bound = (p[~hot, None] * 1.5 * s[~hot]).sum(axis=0)
    assert np.all(np.abs(res["o"] - full["o"]) <= bound * (1 + 1e-9) + 1e-15)


def test_refine_set_monotone_and_abs_rel_equivalence():
    rng = np.random.default_rng(8)
    q, h, tk, tv = _case(rng, 320, 128, 12, 4)
    prev = None
    for tau in [0.0, 1e-4, 1e-3, 0.01, 0.1, 0.5, 1.0, 1.5]:
        res = O.decode_row(q, h, tk, tv, tau)
        bits = np.array([(res["s_bits"][t // 32] >> (t % 32)) & 1 for t in range(320)], bool)
        if prev is not None:
            assert not (bits & ~prev).any()
        prev = bits
        ab = O.decode_row(q, h, tk, tv, tau / res["l"], O.TAU_ABS_PROB)
        assert np.array_equal(ab["s_bits"], res["s_bits"])
    assert not prev.any()  # tau > 1: nothing is hot


def test_forced_refine_set_reproduces_output():
    rng = np.random.default_rng(9)
    q, h, tk, tv = _case(rng, 128, 64, 3, 4)
    res = O.decode_row(q, h, tk, tv, 0.02)
    again = O.decode_row(q, h, tk, tv, 0.9, s_force=res["s_bits"])
    assert np.array_equal(again["o"], res["o"])
