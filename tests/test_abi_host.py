"""Host-side checks of libloopkv that need no GPU: the library loads and exports every
function include/loopkv.h declares, plans are validated, and the byte accounting reproduces
the per-token KV byte totals printed on the LoopKV pages (tests/golden/bytes_per_token.txt)."""
import os
import re

import pytest
import torch

from mixed_precision_kv_append_b200 import build as B
from mixed_precision_kv_append_b200 import loopkv as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLD = os.path.join(ROOT, "tests", "golden", "bytes_per_token.txt")


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(loopkv_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    lib = L.lib()
    declared = _declared()
    assert "loopkv_decode" in declared and "loopkv_append" in declared and "loopkv_alloc" in declared
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, missing
    assert set(L.EXPORTS) == declared


def test_strerror_and_version():
    assert L.loopkv_strerror(0) == "ok"
    assert "flush" in L.loopkv_strerror(-9)
    assert L.lib().loopkv_version() >= 100


def _cfg(layers=2, loops=2, H=4, D=128, B=2, MB=8, dt=L.DTYPE_BF16):
    return L.Config(layers, loops, H, D, B, MB, dt)


def test_plan_validation():
    with pytest.raises(L.LoopKVError) as e:  # share cell in the final loop
        L.loopkv_plan_create(_cfg(), [0, 0, 2, 0], 0.01)
    assert e.value.code == -3
    with pytest.raises(L.LoopKVError) as e:
        L.loopkv_plan_create(_cfg(D=96), [0] * 4, 0.01)
    assert e.value.code == -2
    with pytest.raises(L.LoopKVError) as e:
        L.loopkv_plan_create(_cfg(MB=7), [0] * 4, 0.01)
    assert e.value.code == -2
    with pytest.raises(L.LoopKVError) as e:
        L.loopkv_plan_create(_cfg(), [0] * 4, -0.5)
    assert e.value.code == -1
    with pytest.raises(L.LoopKVError):
        L.loopkv_plan_create(_cfg(), [0, 3, 0, 0], 0.01)
    p = L.loopkv_plan_create(_cfg(), [2, 1, 0, 0], 0.01, L.TAU_ABS_PROB)
    L.lib().loopkv_plan_free(p)


def _modes_for(spec: str):
    parts = spec.split()
    loops, layers = map(int, parts[0].split("x"))
    if parts[1] == "bf16":
        return loops, layers, None
    counts = dict(p.split(":") for p in parts[1:])
    n4, n2, nsh = int(counts.get("4b", 0)), int(counts.get("2b", 0)), int(counts.get("share", 0))
    modes = [None] * (loops * layers)
    final = range((loops - 1) * layers, loops * layers)
    for c in final:
        modes[c] = 0
    n4 -= layers
    rest = [c for c in range(loops * layers) if modes[c] is None]
    for c in rest:
        if nsh:
            modes[c], nsh = 2, nsh - 1
        elif n2:
            modes[c], n2 = 1, n2 - 1
        else:
            modes[c], n4 = 0, n4 - 1
    assert n4 == 0 and n2 == 0 and nsh == 0, spec
    return loops, layers, modes


def _golden():
    for line in open(GOLD):
        if line.strip() and not line.startswith("#"):
            yield [f.strip() for f in line.split("|")]


@pytest.mark.parametrize("row", list(_golden()), ids=lambda r: r[0])
def test_page_byte_totals(row):
    name, spec, hot, stored, read, _src = row
    loops, layers, modes = _modes_for(spec)
    kib = 1024.0
    if modes is None:  # BF16: K and V of every cell, 16 heads x 128 dims x 2 bytes
        p = L.Plan(layers, loops, 16, 128, 1, 2, [0] * (loops * layers), 0.0)
        assert p.bytes()["bf16_bytes_per_token"] / kib == float(stored)
        return
    p = L.Plan(layers, loops, 16, 128, 1, 2, modes, 0.0)
    hf = None
    if hot != "1":
        per_loop = [float(x) for x in hot.split(",")]
        hf = [per_loop[c // layers] for c in range(loops * layers)]
    rep = p.bytes(hf)
    if stored != "-":
        assert rep["stored_bytes_per_token"] / kib == float(stored)
    if read != "-":
        digits = len(read.split(".")[1]) if "." in read else 0
        assert round(rep["read_bytes_per_token"] / kib, digits) == float(read), rep["read_bytes_per_token"] / kib


def test_skipping_lo_plane_saves_half_a_kib_per_token_and_layer():
    p = L.Plan(1, 1, 16, 128, 1, 2, [0], 0.0)
    rep = p.bytes([0.0])
    assert (rep["read_bytes_all_hot"] - rep["read_bytes_all_cold"]) == 512.0
    assert rep["read_bytes_per_token"] == rep["read_bytes_all_cold"]


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_alloc_without_device_fails_loudly():
    p = L.Plan(1, 1, 2, 64, 1, 2, [0], 0.0, in_dtype=torch.float32)
    buf = torch.empty(p.required_bytes(), dtype=torch.uint8)
    with pytest.raises(L.LoopKVError) as e:
        L.loopkv_alloc(p.handle, buf, stream=0)
    assert e.value.code in (-12, -8)
