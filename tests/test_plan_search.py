"""Offline plan search (LoopKV paper §3.1 "Allocation"): the library's exact dynamic program
against a brute-force oracle, and the oracle against hand-worked instances and the extremes.

Host-only: no GPU is needed (loopkv_plan_search touches no device).
"""
import os

import numpy as np
import pytest

from mixed_precision_kv_append_b200 import loopkv as L
from oracle import plan_oracle as P

GOLD = os.path.join(os.path.dirname(__file__), "golden", "plan_search_examples.txt")


def _cfg(layers, loops, H=16, D=128):
    return L.Config(layers, loops, H, D, 1, 2, L.DTYPE_BF16)


def _gold():
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, rest = line.split(None, 1)
        lhs, rhs = rest.split("->")
        head, dmg = lhs.split("|")
        layers, loops, budget, units = head.split()
        d = [float("nan") if x == "-" else float(x) for x in dmg.split()]
        damage = [d[3 * c:3 * c + 3] for c in range(len(d) // 3)]
        out = rhs.split()
        yield name, int(layers), int(loops), float(budget), int(units), damage, out


@pytest.mark.parametrize("case", list(_gold()), ids=lambda c: c[0])
def test_oracle_hand_worked(case):
    _, layers, loops, budget, units, damage, out = case
    H, D = 4, 64
    unit = H * D / 4
    damage = [[0.0 if np.isnan(x) else x for x in row] for row in damage]
    got = P.plan_search(layers, loops, H, D, damage, budget, units * unit)
    if out == ["infeasible"]:
        assert got is None
        return
    modes, read, stored, dmg = got
    assert modes == [int(m) for m in out[0].split(",")]
    assert read == int(out[1]) * unit and stored == int(out[2]) * unit
    assert dmg == pytest.approx(float(out[3]), abs=1e-12)


def test_oracle_extremes():
    rng = np.random.default_rng(3)
    layers, loops, H, D = 2, 3, 2, 64
    damage = rng.uniform(0.01, 1.0, size=(layers * loops, 3)).tolist()
    # unlimited damage budget: every choosable cell 2-bit (fewest reads)
    modes, *_ = P.plan_search(layers, loops, H, D, damage, 1e9)
    assert modes[:4] == [P.CELL_2B] * 4 and modes[4:] == [P.CELL_4B] * 2
    # budget = damage of the all-4B plan, with 2B and share costlier than 4B in every cell
    for row in damage:
        row[1] = row[0] + 0.5
        row[2] = row[0] + 0.25
    all4 = sum(row[0] for row in damage)
    modes, read, stored, dmg = P.plan_search(layers, loops, H, D, damage, all4 + 1e-12)
    assert modes == [P.CELL_4B] * 6 and dmg == pytest.approx(all4)


@pytest.mark.parametrize("case", list(_gold()), ids=lambda c: c[0])
def test_library_hand_worked(case):
    _, layers, loops, budget, units, damage, out = case
    H, D = 4, 64
    damage = [[0.0 if np.isnan(x) else x for x in row] for row in damage]
    cfg = _cfg(layers, loops, H, D)
    if out == ["infeasible"]:
        with pytest.raises(L.LoopKVError) as e:
            L.loopkv_plan_search(cfg, damage, budget, units * H * D / 4)
        assert e.value.code == -13
        return
    modes, rep = L.loopkv_plan_search(cfg, damage, budget, units * H * D / 4)
    assert modes == [int(m) for m in out[0].split(",")]
    assert rep["read_bytes_per_token"] == int(out[1]) * H * D / 4
    assert rep["stored_bytes_per_token"] == int(out[2]) * H * D / 4
    assert rep["damage"] == pytest.approx(float(out[3]), abs=1e-12)


@pytest.mark.parametrize("seed", range(40))
def test_library_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    layers = int(rng.integers(1, 4))
    loops = int(rng.integers(2, 4))
    while (loops - 1) * layers > 8:
        layers -= 1
    H, D = int(rng.choice([2, 16])), int(rng.choice([64, 128]))
    n = layers * loops
    damage = rng.uniform(0.0, 1.0, size=(n, 3))
    damage[:, 1] += rng.uniform(0.0, 1.0, size=n)  # 2-bit usually costlier
    damage = damage.tolist()
    all4 = sum(r[0] for r in damage)
    budget = all4 + float(rng.uniform(0.0, 2.0))
    storage = 0.0 if seed % 3 == 0 else float(rng.uniform(0.4, 1.0)) * 1.25 * D * H * n
    want = P.plan_search(layers, loops, H, D, damage, budget, storage)
    cfg = _cfg(layers, loops, H, D)
    if want is None:
        with pytest.raises(L.LoopKVError):
            L.loopkv_plan_search(cfg, damage, budget, storage)
        return
    modes, rep = L.loopkv_plan_search(cfg, damage, budget, storage)
    w_modes, w_read, w_stored, w_dmg = want
    assert rep["read_bytes_per_token"] == w_read
    assert rep["damage"] == pytest.approx(w_dmg, rel=1e-12, abs=1e-12)
    assert rep["stored_bytes_per_token"] == w_stored
    # the returned modes realise the reported totals and meet the budgets
    ob = P.option_bytes(H, D)
    assert sum(ob[m][0] for m in modes) == rep["read_bytes_per_token"]
    assert sum(ob[m][1] for m in modes) == rep["stored_bytes_per_token"]
    assert sum(damage[c][m] for c, m in enumerate(modes)) == pytest.approx(rep["damage"], rel=1e-12)
    assert modes[(loops - 1) * layers:] == [L.CELL_4B] * layers


def test_library_full_size_plan_is_valid():
    """Ouro-1.4B shape (24 layers x 4 loops) with a synthetic profile in the paper's pattern
    (middle layers more sensitive, loop 1 the most): the plan meets both budgets, its report
    matches its modes, and loopkv_plan_create accepts it."""
    layers, loops, H, D = 24, 4, 16, 128
    n = layers * loops
    damage = np.zeros((n, 3))
    for l in range(loops):
        for j in range(layers):
            edge = 1.0 if (j < 6 or j >= layers - 6) else 4.0
            damage[l * layers + j] = [0.01, 0.05 * edge * (3 - min(l, 2)), 0.03 * edge * (1 + (l == 0))]
    damage = damage.tolist()
    budget, storage = 2.0, 156 * 1024.0
    modes, rep = L.loopkv_plan_search(_cfg(layers, loops, H, D), damage, budget, storage)
    assert rep["damage"] <= budget and rep["stored_bytes_per_token"] <= storage
    ob = P.option_bytes(H, D)
    assert sum(ob[m][0] for m in modes) == rep["read_bytes_per_token"]
    assert sum(ob[m][1] for m in modes) == rep["stored_bytes_per_token"]
    assert sum(damage[c][m] for c, m in enumerate(modes)) == pytest.approx(rep["damage"], rel=1e-12)
    assert rep["stored_bytes_per_token"] < n * ob[L.CELL_4B][1]  # the storage budget forced cuts
    plan = L.Plan(layers, loops, H, D, 1, 2, modes, 0.01)
    del plan
