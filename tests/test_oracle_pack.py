"""Pins of the oracle's packed byte order against hand-derived examples and block sizes.

The per-token byte totals are the pages' own: a 4-bit cell costs 2.5 KiB per token (240 KiB
over 96 cells, LoopKV paper §2.2), a 2-bit cell 1.5 KiB (§5.2, 168 = 72 x 1.5 + 24 x 2.5), and
skipping the lo plane saves 0.5 KiB per token and layer (§3.3).
"""
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "pack_examples.txt")


def _examples():
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, rest = line.split(None, 1)
        codes, out = rest.split("->")
        yield kind, [int(c) for c in codes.split(",")], bytes.fromhex(out.replace(" ", ""))


@pytest.mark.parametrize("ex", list(_examples()), ids=lambda e: e[0])
def test_hand_derived_rows(ex):
    kind, codes, expect = ex
    got = O.pack_row4(codes) if kind == "row4" else O.pack_row2(codes)
    assert bytes(got) == expect


@pytest.mark.parametrize("bits,width", [(4, 4), (2, 2)])
def test_one_hot_channels_land_on_distinct_bits(bits, width):
    D = 128
    seen = np.zeros(D * width // 8, np.uint8)
    for c in range(D):
        codes = np.zeros(D, np.uint8)
        codes[c] = (1 << width) - 1
        row = O.pack_row4(codes) if bits == 4 else O.pack_row2(codes)
        assert bin(int.from_bytes(row.tobytes(), "little")).count("1") == width
        assert not (row & seen).any()
        seen |= row
        # channel c sits inside 32-bit word c // (32 // width)
        word = np.flatnonzero(row)[0] // 4
        assert word == c // (32 // width)
    assert (seen == 0xFF).all()


def test_block_sizes_match_page_byte_totals():
    H, D = 16, 128
    per_token_4b = H * (O.head_main_bytes(4, D) + O.head_lo_bytes(4, D)) / 16
    per_token_2b = H * O.head_main_bytes(2, D) / 16
    lo_per_token = H * O.head_lo_bytes(4, D) / 16
    assert per_token_4b == 2.5 * 1024
    assert per_token_2b == 1.5 * 1024
    assert lo_per_token == 0.5 * 1024


def test_head_block_roundtrip_fields():
    """The packed block holds K codes, the group's K scales (even block) / zeros (odd block),
    V scale/zero pairs per token and channel group, and the hi/lo planes of the value codes."""
    rng = np.random.default_rng(5)
    D = 64
    k = rng.standard_normal((32, D)).astype(np.float32)
    v = rng.standard_normal((32, D)).astype(np.float32)
    h = O.HeadHistory(k, v, 4)
    mains, los = h.packed_blocks()
    assert mains.shape == (2, O.head_main_bytes(4, D)) and los.shape == (2, O.head_lo_bytes(4, D))
    kc_bytes = 16 * D // 2
    for b in range(2):
        m = mains[b]
        assert bytes(m[:D // 2]) == bytes(O.pack_row4(h.kc[16 * b]))
        meta = m[kc_bytes:kc_bytes + 2 * D].view(np.uint16)
        assert np.array_equal(meta, h.kz[0] if b else h.ks[0])
        vmeta = m[kc_bytes + 2 * D: kc_bytes + 2 * D + 16 * (D // 32) * 4].view(np.uint16).reshape(16, D // 32, 2)
        assert np.array_equal(vmeta[..., 0], h.vs[16 * b:16 * b + 16])
        assert np.array_equal(vmeta[..., 1], h.vz[16 * b:16 * b + 16])
        hi = m[-16 * D // 4:].reshape(16, D // 4)
        for t in range(16):
            assert bytes(hi[t]) == bytes(O.pack_row2(h.vc[16 * b + t] >> 2))
            assert bytes(los[b].reshape(16, D // 4)[t]) == bytes(O.pack_row2(h.vc[16 * b + t] & 3))
