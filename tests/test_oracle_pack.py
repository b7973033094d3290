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


def _lines(kind):
    for line in open(GOLD):
        line = line.strip()
        if line and not line.startswith("#") and line.split(None, 1)[0] == kind:
            yield line.split(None, 1)[1]


def _examples():
    for kind in ("row4", "row2"):
        for rest in _lines(kind):
            codes, out = rest.split("->")
            yield kind, [int(c) for c in codes.split(",")], bytes.fromhex(out.replace(" ", ""))


def _plane_examples():
    for rest in _lines("vplane"):
        lhs, rhs = rest.split("->")
        D, t, c, code = (int(x) for x in lhs.split())
        hb, hv, lb, lv = rhs.split()
        yield D, t, c, code, int(hb), int(hv, 16), int(lb), int(lv, 16)


@pytest.mark.parametrize("ex", list(_examples()), ids=lambda e: e[0])
def test_hand_derived_rows(ex):
    kind, codes, expect = ex
    got = O.pack_row4(codes) if kind == "row4" else O.pack_row2(codes)
    assert bytes(got) == expect


@pytest.mark.parametrize("ex", list(_plane_examples()), ids=lambda e: f"D{e[0]}_t{e[1]}_c{e[2]}")
def test_hand_derived_value_planes(ex):
    """One 4-bit value code in an otherwise zero block lands on the hand-derived bytes of the
    hi and lo planes, and nowhere else."""
    D, t, c, code, hbyte, hval, lbyte, lval = ex
    vc = np.zeros((16, D), np.uint8)
    vc[t, c] = code
    z16 = np.zeros(16 * (D // 32), np.uint16)
    main, lo = O.pack_head_block(4, D, np.zeros((16, D), np.uint8), np.zeros(D, np.uint16), vc, z16, z16)
    hi = main[-16 * D // 4:]
    assert np.flatnonzero(hi).tolist() == [hbyte] and hi[hbyte] == hval
    assert np.flatnonzero(lo).tolist() == [lbyte] and lo[lbyte] == lval


def _unpack_plane(words_bytes, D, kappa_major):
    """Decode a packed plane back to [16][D] 2-bit values by walking every field."""
    w = np.frombuffer(bytes(words_bytes), dtype="<u4")
    out = np.zeros((16, D), np.uint8)
    for kappa in range(D // 4):
        for tau in range(4):
            word = int(w[4 * kappa + tau] if kappa_major else w[tau * (D // 4) + kappa])
            for b in range(4):
                for i in range(4):
                    out[4 * tau + b, 4 * kappa + i] = (word >> (8 * b + 2 * i)) & 3
    return out


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
        # V meta pairs ordered [channel group][token]
        vmeta = m[kc_bytes + 2 * D: kc_bytes + 2 * D + 16 * (D // 32) * 4].view(np.uint16).reshape(D // 32, 16, 2)
        assert np.array_equal(vmeta[..., 0].T, h.vs[16 * b:16 * b + 16])
        assert np.array_equal(vmeta[..., 1].T, h.vz[16 * b:16 * b + 16])
        # every field of both planes decodes back to its (token, channel) code
        assert np.array_equal(_unpack_plane(m[-16 * D // 4:], D, True), h.vc[16 * b:16 * b + 16] >> 2)
        assert np.array_equal(_unpack_plane(los[b], D, False), h.vc[16 * b:16 * b + 16] & 3)
