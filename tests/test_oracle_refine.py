"""Independent pins of the oracle's refine set S and of the mixed-precision output it selects,
at thresholds strictly between 0 and 1 (LoopKV §3.3 "Read-time V precision": a history token
is cold when its weight falls below tau times the largest weight of its row; a cold 4-bit
value decodes to the middle of its 4-code bucket, a hot one to its full code).

Nothing here reads the oracle's scores, weights or row statistics.  The scores are rebuilt in
NumPy from the stored codes and fp16 metadata (dequantized key = zero + scale * code, score =
q . k / sqrt(D)), the set is formed from them, and the output is taken from the library routine
torch.nn.functional.scaled_dot_product_attention on values dequantized in this file.  A wrong
factor in the threshold (tau / 2), a strict comparison, or a wrong cold reconstruction fails
one of the cases below.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O

TAUS = [0.005, 0.01, 0.05, 0.3]


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
    mid = z + s * (4.0 * (h.vc >> 2).astype(np.float64) + 1.5)
    return np.where(hot[:, None], full, mid)


def _bits(words, n):
    return np.array([(int(words[t // 32]) >> (t % 32)) & 1 for t in range(n)], bool)


def _words(hot):
    out = np.zeros(max((hot.size + 31) // 32, 1), np.uint32)
    for t in np.flatnonzero(hot):
        out[t // 32] |= np.uint32(1 << (t % 32))
    return out


def _sdpa(q, K, V):
    t = lambda a: torch.tensor(a, dtype=torch.float64).view(1, 1, -1, a.shape[-1])  # noqa: E731
    return torch.nn.functional.scaled_dot_product_attention(t(q[None]), t(K), t(V)).view(-1).numpy()


def _row(seed, T, D, n_tail, spread=1.0):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((T, D)) * np.exp(spread * rng.standard_normal(D))[None, :]).astype(np.float32)
    v = rng.standard_normal((T, D)).astype(np.float32)
    h = O.HeadHistory(k, v, 4)
    tk = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    tv = rng.standard_normal((n_tail, D)).astype(np.float32).astype(np.float64)
    q = rng.standard_normal(D).astype(np.float32).astype(np.float64)
    return q, h, tk, tv


@pytest.mark.parametrize("tau", TAUS)
@pytest.mark.parametrize("mode", [O.TAU_REL_MAX, O.TAU_ABS_PROB])
@pytest.mark.parametrize("seed,T,D,n_tail,spread", [(1, 256, 128, 9, 1.0), (2, 512, 64, 0, 1.5), (3, 96, 128, 31, 0.5)])
def test_refine_set_and_output_from_independent_scores(tau, mode, seed, T, D, n_tail, spread):
    q, h, tk, tv = _row(seed, T, D, n_tail, spread)
    s = np.concatenate([_keys(h) @ q, tk @ q]) / math.sqrt(D)
    w = np.exp(s - s.max())
    qty = w[:T] / w.sum() if mode == O.TAU_ABS_PROB else w[:T]
    if mode == O.TAU_ABS_PROB:  # normalised weights are small: place tau inside their range
        tau = tau * float(qty.max())
    ref_hot = qty >= tau
    res = O.decode_row(q, h, tk, tv, tau, mode)
    got = _bits(res["s_bits"], T)
    clear = np.abs(qty - tau) > 1e-9 * max(tau, 1e-300)
    assert np.array_equal(got[clear], ref_hot[clear])
    # the cases are chosen so that both sides of the threshold are populated
    assert ref_hot.any() and (~ref_hot).any()
    ref = _sdpa(q, np.concatenate([_keys(h), tk]), np.concatenate([_values(h, ref_hot), tv]))
    assert np.allclose(res["o"], ref, rtol=0, atol=1e-12)


def _integer_row():
    """A row whose scores are exact in binary: D = 64 (1/sqrt(D) = 1/8), keys quantized without
    loss (every channel of the group holds 0 and 15, so zero 0 and scale 1), small integer q."""
    D, T = 64, 32
    codes = np.zeros((T, D), np.float32)
    codes[1, :] = 15.0  # token 1 spans the group in every channel
    codes[2:9, 0] = [8, 7, 6, 5, 4, 3, 2]
    codes[0, 0] = 9  # token 0 has the largest score (q = e_0)
    v = np.random.default_rng(5).standard_normal((T, D)).astype(np.float32)
    h = O.HeadHistory(codes, v, 4)
    assert np.array_equal(_keys(h), codes.astype(np.float64))
    q = np.zeros(D)
    q[0] = 1.0
    q[1] = -1.0  # token 1: 15 - 15 = 0
    return q, h


def test_tie_at_tau_is_hot():
    """A token whose weight equals tau exactly is hot (>=, not >)."""
    q, h = _integer_row()
    s = (_keys(h) @ q) / 8.0  # exact: token 0 at 9/8, token j = 2..8 at (10 - j)/8
    assert s[0] == 9 / 8 and s.max() == 9 / 8
    # tau = the weight of token 4 computed with the same exp on the same exact difference
    tau = math.exp(s[4] - s[0])
    res = O.decode_row(q, h, np.zeros((0, 64)), np.zeros((0, 64)), tau)
    hot = _bits(res["s_bits"], 32)
    assert res["r"][4] == tau
    assert list(np.flatnonzero(hot)) == [0, 2, 3, 4]
    # just above the tie the token turns cold
    res2 = O.decode_row(q, h, np.zeros((0, 64)), np.zeros((0, 64)), math.nextafter(tau, 1.0))
    assert list(np.flatnonzero(_bits(res2["s_bits"], 32))) == [0, 2, 3]
    # tau = 1: exactly the tokens at the row maximum
    res3 = O.decode_row(q, h, np.zeros((0, 64)), np.zeros((0, 64)), 1.0)
    assert list(np.flatnonzero(_bits(res3["s_bits"], 32))) == [0]


def test_tie_at_tau_normalised_weight():
    """The normalised-weight rule at a tie: tau = r_4 / l with l summed in token order."""
    q, h = _integer_row()
    s = (_keys(h) @ q) / 8.0
    r = [math.exp(x - s[0]) for x in s]
    l = 0.0
    for x in r:
        l += x
    tau = r[4] / l
    res = O.decode_row(q, h, np.zeros((0, 64)), np.zeros((0, 64)), tau, O.TAU_ABS_PROB)
    assert list(np.flatnonzero(_bits(res["s_bits"], 32))) == [0, 2, 3, 4]


def test_hand_worked_mixed_output():
    """Output of the integer row at tau = exp(-2/8): tokens 0, 2, 3 hot, the rest cold, checked
    against a sum written out token by token."""
    q, h = _integer_row()
    s = (_keys(h) @ q) / 8.0
    tau = math.exp(-2 / 8)
    res = O.decode_row(q, h, np.zeros((0, 64)), np.zeros((0, 64)), tau)
    hot = np.zeros(32, bool)
    hot[[0, 2, 3]] = True
    assert np.array_equal(_bits(res["s_bits"], 32), hot)
    vs, vz = _f16(h.vs), _f16(h.vz)
    num = np.zeros(64)
    den = 0.0
    for t in range(32):
        wt = math.exp(s[t] - s[0])
        den += wt
        for c in range(64):
            code = int(h.vc[t, c])
            level = code if hot[t] else 4 * (code >> 2) + 1.5
            num[c] += wt * (vz[t, c // 32] + vs[t, c // 32] * level)
    assert np.allclose(res["o"], num / den, rtol=0, atol=1e-13)
