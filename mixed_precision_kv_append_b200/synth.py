"""Seeded synthetic workloads shaped like the LoopKV pages' models (inputs only).

This module holds no arithmetic of the method: it draws queries, keys and values, the
per-request context lengths and the per-cell storage plan.  Both the CUDA path and the
CPU oracle are fed from it, so that they see the same bytes.

Recipe (stated once, used by the tests and the benchmark):
  * Ouro-1.4B shape: 24 layers x 4 loops, 16 KV heads x 128 (MHA); Ouro-2.6B: 48 layers
    (LoopKV paper §2.1 and Appendix on Ouro-2.6B).  The tiny case: 1 layer x 2 loops,
    2 heads x 64.
  * Q, K, V ~ N(0, 1).  Keys are multiplied per (layer, head, channel) by a lognormal(0, 1)
    channel scale shared by all loops of the layer.  Loop l+1's keys are
    0.85 * loop l's keys + 0.53 * (channel scale * N(0, 1)), so adjacent loops correlate
    with coefficient 0.85 and the variance is kept (0.85^2 + 0.53^2 ~ 1).  Values and
    queries are independent per loop.
  * Plans: the loops named by the workload get round(p2 * N) 2-bit cells and
    round(psh * N) share cells, chosen by a seeded shuffle, the rest 4-bit; other loops
    4-bit; the final loop always stores its own pages.
  * Every draw uses torch's Philox generator (CUDA) or the CPU generator, seeded from
    (workload seed, layer, request) so a row can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import math

import torch

CELL_4B, CELL_2B, CELL_SHARE = 0, 1, 2


@dataclasses.dataclass
class Workload:
    name: str
    n_layers: int
    n_loops: int
    H: int
    D: int
    B: int
    lengths: list          # history tokens per request at the start
    dtype: torch.dtype
    modes: list            # loop-major storage mode per cell
    tau: float
    tau_mode: int = 0      # 0 = relative to the row max, 1 = normalised weight
    append_steps: int = 0  # decode steps that append one token per request per cell
    seed: int = 0
    layer_windows: dict = dataclasses.field(default_factory=dict)  # layer -> sliding window (tokens)
    sink: int = 0          # BF16 sink tokens of every (cell, request)
    window: int = 0        # BF16 recent-window tokens (the near region holds window .. window + 31)

    @property
    def n_cells(self):
        return self.n_layers * self.n_loops

    @property
    def max_blocks(self):
        t = max(self.lengths) + self.append_steps + 32
        return 2 * math.ceil(t / 32)


def seeded_plan(n_layers, n_loops, loops, p2, psh, seed) -> list:
    """Storage modes for a plan: in `loops` (0-based), round(p2*N) 2-bit and round(psh*N)
    share cells by a seeded shuffle, the rest 4-bit; every other cell 4-bit."""
    modes = [CELL_4B] * (n_layers * n_loops)
    cells = [lp * n_layers + la for lp in loops for la in range(n_layers)]
    n = len(cells)
    n2, nsh = round(p2 * n), round(psh * n)
    g = torch.Generator().manual_seed(1000 + seed)
    perm = torch.randperm(n, generator=g).tolist()
    for k, idx in enumerate(perm):
        c = cells[idx]
        if k < n2:
            modes[c] = CELL_2B
        elif k < n2 + nsh:
            modes[c] = CELL_SHARE
    return modes


def workload(name: str, seed: int = 0) -> Workload:
    """The benchmark workloads by name: the five of the configuration list and the Ouro-2.6B
    fixed-length sweep."""
    if name == "tiny":
        return Workload("tiny", 1, 2, 2, 64, 1, [256], torch.float32, [CELL_4B, CELL_2B], 0.02, seed=seed)
    if name == "kivi4_8k":
        return Workload("kivi4_8k", 24, 4, 16, 128, 8, [8192] * 8, torch.bfloat16, [CELL_4B] * 96, 0.0, seed=seed)
    if name == "mixed_8k":
        modes = seeded_plan(24, 4, [1, 2], 0.30, 0.20, seed)
        return Workload("mixed_8k", 24, 4, 16, 128, 32, [8192] * 32, torch.bfloat16, modes, 0.01, seed=seed)
    if name == "long_16k":
        modes = seeded_plan(24, 4, [1, 2], 0.35, 0.25, seed)
        return Workload("long_16k", 24, 4, 16, 128, 32, [16384] * 32, torch.bfloat16, modes, 0.005,
                        append_steps=64, seed=seed)
    if name == "ragged_2p6b":
        g = torch.Generator().manual_seed(2000 + seed)
        lengths = torch.randint(4096, 32768 + 1, (8,), generator=g).tolist()
        modes = seeded_plan(48, 4, [0, 1, 2], 0.35, 0.25, seed)
        return Workload("ragged_2p6b", 48, 4, 16, 128, 8, lengths, torch.bfloat16, modes, 0.01, seed=seed)
    if name.startswith("ouro2p6b_"):
        # Ouro-2.6B fixed-length sweep (the paper's 8K / 16K / 32K throughput tables): 48 layers
        # x 4 loops, the ragged workload's plan, batch halving as the context doubles so that
        # the stored KV stays about 87 GB on one GPU
        T = {"ouro2p6b_8k": 8192, "ouro2p6b_16k": 16384, "ouro2p6b_32k": 32768}[name]
        B = 32 * 8192 // T
        modes = seeded_plan(48, 4, [0, 1, 2], 0.35, 0.25, seed)
        return Workload(name, 48, 4, 16, 128, B, [T] * B, torch.bfloat16, modes, 0.01, seed=seed)
    if name == "mixed_8k_sw":
        # mixed_8k with the paper's BF16 near region: a 32-token sink and a 256-token window
        # (LoopKV §2.3, §3.4); the history between them is quantized as in mixed_8k
        w = workload("mixed_8k", seed)
        w.name, w.sink, w.window = "mixed_8k_sw", 32, 256
        return w
    if name == "dory_16k":
        # Dory-4B-shaped recurrent block (LoopKV §2.1: 20 recurrent attention layers, 5 with full
        # attention and 15 with a sliding window).  The pages give neither the loop count, the
        # head shape nor the window size: 4 loops, 16 x 128 heads and a 4096-token window are
        # assumptions of this workload; every fourth layer attends fully
        modes = seeded_plan(20, 4, [1, 2], 0.35, 0.25, seed)
        windows = {la: 4096 for la in range(20) if la % 4 != 0}
        return Workload("dory_16k", 20, 4, 16, 128, 16, [16384] * 16, torch.bfloat16, modes, 0.01, seed=seed,
                        layer_windows=windows)
    raise KeyError(name)


WORKLOADS = ["tiny", "kivi4_8k", "mixed_8k", "long_16k", "ragged_2p6b", "ouro2p6b_8k", "ouro2p6b_16k",
             "ouro2p6b_32k", "dory_16k", "mixed_8k_sw"]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed & 0x7FFFFFFFFFFFFFFF)
    return g


def _mix(*xs) -> int:
    h = 1469598103934665603
    for x in xs:
        h = ((h ^ (int(x) & 0xFFFFFFFF)) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return h


def channel_scales(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Lognormal(0, 1) key scale per (head, channel) of a layer, float32 [H, D]."""
    g = _gen(_mix(w.seed, 11, layer), device)
    return torch.exp(torch.randn((w.H, w.D), generator=g, device=device, dtype=torch.float32))


def layer_history(w: Workload, layer: int, req: int, T: int | None = None, device="cpu"):
    """History keys and values of every loop of one (layer, request): lists of [T, H, D]
    tensors in the workload dtype, loop 0 first."""
    T = w.lengths[req] if T is None else T
    sc = channel_scales(w, layer, device)
    g = _gen(_mix(w.seed, 22, layer, req), device)
    ks, vs = [], []
    k = torch.randn((T, w.H, w.D), generator=g, device=device, dtype=torch.float32) * sc
    for lp in range(w.n_loops):
        if lp > 0:
            noise = torch.randn((T, w.H, w.D), generator=g, device=device, dtype=torch.float32) * sc
            k = 0.85 * k + 0.53 * noise
        v = torch.randn((T, w.H, w.D), generator=g, device=device, dtype=torch.float32)
        ks.append(k.to(w.dtype))
        vs.append(v.to(w.dtype))
    return ks, vs


def step_tokens(w: Workload, step: int, layer: int, device="cpu"):
    """Queries and new-token keys/values of one decode step for every loop of a layer:
    lists over loops of [B, H, D] tensors (q, k, v)."""
    sc = channel_scales(w, layer, device)
    g = _gen(_mix(w.seed, 33, step, layer), device)
    qs, ks, vs = [], [], []
    k = torch.randn((w.B, w.H, w.D), generator=g, device=device, dtype=torch.float32) * sc
    for lp in range(w.n_loops):
        if lp > 0:
            noise = torch.randn((w.B, w.H, w.D), generator=g, device=device, dtype=torch.float32) * sc
            k = 0.85 * k + 0.53 * noise
        qs.append(torch.randn((w.B, w.H, w.D), generator=g, device=device, dtype=torch.float32).to(w.dtype))
        ks.append(k.to(w.dtype))
        vs.append(torch.randn((w.B, w.H, w.D), generator=g, device=device, dtype=torch.float32).to(w.dtype))
    return qs, ks, vs
