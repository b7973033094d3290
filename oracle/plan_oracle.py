"""Brute-force oracle of LoopKV's offline plan search.

TEST INFRASTRUCTURE ONLY: the tests may import this module; the library never does.

LoopKV paper §3.1 "Allocation": each cell (loop, layer) takes one storage option -- 4-bit
codes, 2-bit codes, or sharing the final loop's history at the same layer (§3.2: a shared
cell stores nothing and reads the source's INT4 pages like an own INT4 cell) -- and the plan
minimizes the bytes read per token under a damage budget and, optionally, a storage budget,
with the per-cell damages of a profile adding up over cells (§3.1, §2.4).  The paper's plans
choose among the cells of loops 1..n-1 and keep the final loop in INT4 (read-optimized plan:
"INT2 in 25 of the 72 cells").  Bytes per token (§2.2 at H = 16, D = 128: a 4-bit cell 2.5 KiB,
a 2-bit cell 1.5 KiB) are taken per head as 1.25 D and 0.75 D bytes.

This module enumerates every plan -- 3^(cells of loops 1..n-1) of them, so tiny instances only
-- and returns the one with the fewest read bytes, then the least damage, then the least
storage.
"""
from __future__ import annotations

import itertools

CELL_4B, CELL_2B, CELL_SHARE = 0, 1, 2


def option_bytes(H: int, D: int):
    """(read, stored) bytes per token of one cell for each option."""
    b4, b2 = 1.25 * D * H, 0.75 * D * H
    return {CELL_4B: (b4, b4), CELL_2B: (b2, b2), CELL_SHARE: (b4, 0.0)}


def plan_search(n_layers: int, n_loops: int, H: int, D: int, damage, damage_budget: float,
                storage_budget: float = 0.0):
    """damage[cell][option], cells loop-major.  Returns (modes, read, stored, damage) of the
    best plan, or None if no plan meets the budgets."""
    M = (n_loops - 1) * n_layers
    ob = option_bytes(H, D)
    best_key, best_modes = None, None
    for combo in itertools.product((CELL_4B, CELL_2B, CELL_SHARE), repeat=M):
        modes = list(combo) + [CELL_4B] * n_layers
        read = stored = dmg = 0.0
        for c, o in enumerate(modes):
            read += ob[o][0]
            stored += ob[o][1]
            dmg += damage[c][o]
        if dmg > damage_budget:
            continue
        if storage_budget > 0.0 and stored > storage_budget:
            continue
        key = (read, dmg, stored)
        if best_key is None or key < best_key:
            best_key, best_modes = key, modes
    if best_key is None:
        return None
    return best_modes, best_key[0], best_key[2], best_key[1]
