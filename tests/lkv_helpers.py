"""Shared helpers for the parity tests: run the CPU oracle on exactly the inputs given to
the CUDA path and compare element by element.

Tolerances (from the target stated for this path): codes, scales and packed bytes
bit-exact; the refine set S bit-exact except for tokens whose oracle weight lies within
1e-6 of tau (in the quantity the tau mode compares); attention outputs within 2e-3 absolute
after the oracle is re-evaluated with the GPU's S (so that a tie flip is not counted twice).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O

OUT_ATOL = 2e-3
TIE_BAND = 1e-6


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def bits_of(words: np.ndarray, n: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint32)
    return np.array([(int(w[t // 32]) >> (t % 32)) & 1 for t in range(n)], dtype=bool)


def oracle_packed(hist: O.HeadHistory):
    """Oracle-packed blocks of one head: (main [nb][bytes], lo [nb][bytes])."""
    return hist.packed_blocks()


def check_row(gpu_out: np.ndarray, gpu_bits: np.ndarray, gpu_m: float | None, gpu_l: float | None,
              q: np.ndarray, hist: O.HeadHistory | None, tail_k: np.ndarray, tail_v: np.ndarray,
              tau: float, tau_mode: int, where: str = "", hist_first: int = 0):
    """Compare one (request, head) row; history tokens before hist_first are outside a sliding
    attention window.  Returns (max abs error, n S mismatches inside the tie band)."""
    res = O.decode_row(q, hist, tail_k, tail_v, tau, tau_mode, hist_first=hist_first)
    n_hist = 0 if hist is None else hist.T
    ref_bits = bits_of(res["s_bits"], n_hist)
    got_bits = bits_of(gpu_bits, n_hist) if n_hist else np.zeros(0, bool)
    diff = np.flatnonzero(ref_bits != got_bits)
    if diff.size:
        r = res["r"][:n_hist]
        qty = r / res["l"] if tau_mode == O.TAU_ABS_PROB else r
        far = diff[np.abs(qty[diff] - tau) > TIE_BAND]
        assert far.size == 0, (
            f"{where}: refine set differs outside the tie band at tokens {far[:8]} "
            f"(oracle weight {qty[far[:8]]}, tau {tau})")
        res = O.decode_row(q, hist, tail_k, tail_v, tau, tau_mode, s_force=words_from_bits(got_bits),
                           hist_first=hist_first)
    err = float(np.max(np.abs(gpu_out.astype(np.float64) - res["o"])))
    assert err <= OUT_ATOL, f"{where}: max abs output error {err}"
    if gpu_m is not None:
        assert abs(gpu_m - res["m"]) <= 1e-4 * max(1.0, abs(res["m"])), f"{where}: row max {gpu_m} vs {res['m']}"
    if gpu_l is not None:
        assert abs(gpu_l - res["l"]) <= 1e-4 * res["l"], f"{where}: row sum {gpu_l} vs {res['l']}"
    return err, int(diff.size)


def words_from_bits(bits: np.ndarray) -> np.ndarray:
    out = np.zeros((bits.size + 31) // 32, np.uint32)
    for t in np.flatnonzero(bits):
        out[t // 32] |= np.uint32(1 << (t % 32))
    return out
