"""Python access to the CPU oracle of the LoopKV decode hot path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline
and reference arms are the only callers.  The arithmetic lives in ``loopkv_oracle.c``
(plain C, fp64 attention, IEEE fp32 quantizer); this module only marshals NumPy arrays
and composes the per-row C routines into per-cell helpers.  It imports nothing from the
CUDA package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "loopkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, NONFINITE, RANGE, BADARG = 0, 1, 2, 3
TAU_REL_MAX, TAU_ABS_PROB = 0, 1
GROUP = 32

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain IEEE arithmetic, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
            L.orc_f16_to_f64.restype = ctypes.c_double
            L.orc_f64_to_f16.argtypes = [ctypes.c_double, ctypes.c_int]
            L.orc_f64_to_f16.restype = ctypes.c_uint16
            L.orc_quantize_group.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, _u16p,
                                             _u8p, ctypes.c_int]
            L.orc_quantize_group.restype = ctypes.c_int
            for name in ("orc_quantize_k", "orc_quantize_v"):
                f = getattr(L, name)
                f.argtypes = [_f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8p, _u16p, _u16p]
                f.restype = ctypes.c_int
            L.orc_pack_row4.argtypes = [_u8p, ctypes.c_int, _u8p]
            L.orc_pack_row2.argtypes = [_u8p, ctypes.c_int, _u8p]
            L.orc_head_main_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
            L.orc_head_main_bytes.restype = ctypes.c_int
            L.orc_head_lo_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
            L.orc_head_lo_bytes.restype = ctypes.c_int
            L.orc_pack_head_block.argtypes = [ctypes.c_int, ctypes.c_int, _u8p, _u16p, _u8p, _u16p, _u16p,
                                              _u8p, _u8p]
            L.orc_decode_row.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _u8p, _u16p, _u16p,
                                         _u8p, _u16p, _u16p, ctypes.c_int, _f64p, _f64p, ctypes.c_double,
                                         ctypes.c_int, _u32p, _f64p, _f64p, _f64p, _u32p, _f64p]
            L.orc_decode_row.restype = ctypes.c_int
            L.orc_decode_row_from.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, _u8p,
                                              _u16p, _u16p, _u8p, _u16p, _u16p, ctypes.c_int, _f64p, _f64p,
                                              ctypes.c_double, ctypes.c_int, _u32p, _f64p, _f64p, _f64p, _u32p,
                                              _f64p]
            L.orc_decode_row_from.restype = ctypes.c_int
            L.orc_stream_refine.argtypes = [ctypes.c_int, _f64p, ctypes.POINTER(ctypes.c_int), ctypes.c_int,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_double, _u32p]
            L.orc_stream_refine.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


# --------------------------------------------------------------------------- fp16

def f16_to_f64(h: int) -> float:
    return lib().orc_f16_to_f64(int(h))


def f64_to_f16(x: float, direction: int) -> int:
    """Round to binary16 bits: direction -1 down, +1 up, 0 nearest-even."""
    return int(lib().orc_f64_to_f16(float(x), int(direction)))


def f16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Vectorised value of fp16 bit patterns (exact)."""
    return np.asarray(a, dtype=np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------------- quantizer

def quantize_group(x, bits: int):
    """Quantize one group (1-D float32 array).  Returns (zero_bits, scale_bits, codes, status)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    z = ctypes.c_uint16()
    s = ctypes.c_uint16()
    codes = np.zeros(x.size, dtype=np.uint8)
    st = lib().orc_quantize_group(_p(x, _f32p), 1, x.size, bits, ctypes.byref(z), ctypes.byref(s),
                                  _p(codes, _u8p), 1)
    return int(z.value), int(s.value), codes, int(st)


def quantize_k(k: np.ndarray, bits: int):
    """Keys of one (request, head), k[T][D] float32 -> codes[T][D], scale[T/32][D], zero[T/32][D], status."""
    k = np.ascontiguousarray(k, dtype=np.float32)
    T, D = k.shape
    codes = np.zeros((T, D), np.uint8)
    sc = np.zeros((T // GROUP, D), np.uint16)
    ze = np.zeros((T // GROUP, D), np.uint16)
    st = lib().orc_quantize_k(_p(k, _f32p), T, D, bits, _p(codes, _u8p), _p(sc, _u16p), _p(ze, _u16p))
    return codes, sc, ze, int(st)


def quantize_v(v: np.ndarray, bits: int):
    """Values of one (request, head), v[T][D] float32 -> codes[T][D], scale[T][D/32], zero[T][D/32], status."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    T, D = v.shape
    codes = np.zeros((T, D), np.uint8)
    sc = np.zeros((T, D // GROUP), np.uint16)
    ze = np.zeros((T, D // GROUP), np.uint16)
    st = lib().orc_quantize_v(_p(v, _f32p), T, D, bits, _p(codes, _u8p), _p(sc, _u16p), _p(ze, _u16p))
    return codes, sc, ze, int(st)


# ----------------------------------------------------------------------- packing

def pack_row4(codes) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(codes.size // 2, np.uint8)
    lib().orc_pack_row4(_p(codes, _u8p), codes.size, _p(out, _u8p))
    return out


def pack_row2(codes) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(codes.size // 4, np.uint8)
    lib().orc_pack_row2(_p(codes, _u8p), codes.size, _p(out, _u8p))
    return out


def head_main_bytes(bits: int, D: int) -> int:
    return int(lib().orc_head_main_bytes(bits, D))


def head_lo_bytes(bits: int, D: int) -> int:
    return int(lib().orc_head_lo_bytes(bits, D))


def pack_head_block(bits, D, kcodes, kmeta, vcodes, vscale, vzero):
    """Pack one head of one 16-token block -> (main bytes, lo bytes)."""
    kcodes = np.ascontiguousarray(kcodes, np.uint8)
    kmeta = np.ascontiguousarray(kmeta, np.uint16)
    vcodes = np.ascontiguousarray(vcodes, np.uint8)
    vscale = np.ascontiguousarray(vscale, np.uint16)
    vzero = np.ascontiguousarray(vzero, np.uint16)
    main = np.zeros(head_main_bytes(bits, D), np.uint8)
    lo = np.zeros(max(head_lo_bytes(bits, D), 1), np.uint8)
    lib().orc_pack_head_block(bits, D, _p(kcodes, _u8p), _p(kmeta, _u16p), _p(vcodes, _u8p),
                              _p(vscale, _u16p), _p(vzero, _u16p), _p(main, _u8p), _p(lo, _u8p))
    return main, lo[: head_lo_bytes(bits, D)]


class HeadHistory:
    """Quantized history of one (cell, request, head): logical codes and fp16 metadata."""

    def __init__(self, k: np.ndarray, v: np.ndarray, bits: int):
        self.bits = bits
        self.T, self.D = k.shape
        self.kc, self.ks, self.kz, st_k = quantize_k(k, bits)
        self.vc, self.vs, self.vz, st_v = quantize_v(v, bits)
        self.status = st_k or st_v

    def packed_blocks(self):
        """Packed bytes of this head in every 16-token block: (main[nb][bytes], lo[nb][bytes])."""
        nb = self.T // 16
        mains, los = [], []
        for b in range(nb):
            g, odd = divmod(b, 2)
            kmeta = self.kz[g] if odd else self.ks[g]
            sl = slice(16 * b, 16 * b + 16)
            m, lo = pack_head_block(self.bits, self.D, self.kc[sl], kmeta, self.vc[sl], self.vs[sl], self.vz[sl])
            mains.append(m)
            los.append(lo)
        return np.stack(mains) if mains else np.zeros((0, head_main_bytes(self.bits, self.D)), np.uint8), \
            np.stack(los) if los else np.zeros((0, head_lo_bytes(self.bits, self.D)), np.uint8)


# ------------------------------------------------------------------------ decode

def decode_row(q, hist: HeadHistory | None, tail_k, tail_v, tau: float, tau_mode: int = TAU_REL_MAX,
               s_force: np.ndarray | None = None, bits: int | None = None, D: int | None = None,
               hist_first: int = 0):
    """Attention for one (request, head) row in fp64.

    q: [D]; hist: quantized history of the cell that is read (own or final loop's);
    tail_k/tail_v: [n_tail][D] raw tail; hist_first: history tokens before it are outside a
    sliding attention window (not attended).  Returns dict(o, m, l, s_bits, r).
    """
    q = np.ascontiguousarray(q, np.float64)
    D = q.size
    if hist is None or hist.T == 0:
        n_hist = 0
        bits = bits or 4
        kc = np.zeros((1, D), np.uint8)
        ks = kz = np.zeros((1, D), np.uint16)
        vc = np.zeros((1, D), np.uint8)
        vs = vz = np.zeros((1, D // GROUP), np.uint16)
    else:
        n_hist, bits = hist.T, hist.bits
        kc, ks, kz, vc, vs, vz = hist.kc, hist.ks, hist.kz, hist.vc, hist.vs, hist.vz
    tk = np.ascontiguousarray(np.asarray(tail_k, np.float64).reshape(-1, D))
    tv = np.ascontiguousarray(np.asarray(tail_v, np.float64).reshape(-1, D))
    n_tail = tk.shape[0]
    o = np.zeros(D, np.float64)
    m = ctypes.c_double()
    l_ = ctypes.c_double()
    s_bits = np.zeros(max(n_hist // 32, 1), np.uint32)
    r = np.zeros(max(n_hist + n_tail, 1), np.float64)
    sf = None
    if s_force is not None:
        sf = np.ascontiguousarray(s_force, np.uint32)
    if tk.size == 0:
        tk = np.zeros((1, D))
        tv = np.zeros((1, D))
    st = lib().orc_decode_row_from(D, bits, n_hist, int(hist_first), _p(q, _f64p), _p(kc, _u8p), _p(ks, _u16p),
                                   _p(kz, _u16p), _p(vc, _u8p), _p(vs, _u16p), _p(vz, _u16p), n_tail,
                                   _p(tk, _f64p), _p(tv, _f64p), float(tau), int(tau_mode),
                                   _p(sf, _u32p) if sf is not None else None, _p(o, _f64p), ctypes.byref(m),
                                   ctypes.byref(l_), _p(s_bits, _u32p), _p(r, _f64p))
    if st != OK:
        raise ValueError(f"oracle decode_row status {st}")
    return dict(o=o, m=m.value, l=l_.value, s_bits=s_bits[: n_hist // 32], r=r[: n_hist + n_tail])


def dequant_k(hist: HeadHistory) -> np.ndarray:
    """Dequantized keys z + s*code, fp64 [T][D] (for library cross-checks in tests)."""
    g = np.arange(hist.T) // GROUP
    return f16_bits_to_f64(hist.kz)[g] + f16_bits_to_f64(hist.ks)[g] * hist.kc.astype(np.float64)


def dequant_v(hist: HeadHistory, hot: np.ndarray | None) -> np.ndarray:
    """Dequantized values fp64 [T][D]; hot[T] bool selects full codes (4-bit), others mid-bin."""
    j = np.arange(hist.D) // GROUP
    z = f16_bits_to_f64(hist.vz)[:, j]
    s = f16_bits_to_f64(hist.vs)[:, j]
    code = hist.vc.astype(np.float64)
    if hist.bits == 2:
        return z + s * code
    cold = 4.0 * (hist.vc >> 2).astype(np.float64) + 1.5
    if hot is None:
        hot = np.ones(hist.T, bool)
    return np.where(hot[:, None], z + s * code, z + s * cold)


def stream_refine(scores, order, m0: float, tau: float, running: bool = True) -> np.ndarray:
    """Refine set of the streaming reader (seeded maximum, growing with the scores read when
    `running`; see orc_stream_refine): scores [n_hist] in natural-log units, order = group
    reading order.  Returns the bitmap [n_hist / 32] (uint32)."""
    s = np.ascontiguousarray(scores, np.float64)
    o = np.ascontiguousarray(order, np.int32)
    bits = np.zeros(max(s.size // GROUP, 1), np.uint32)
    st = lib().orc_stream_refine(int(s.size), _p(s, _f64p), o.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                 int(o.size), float(m0), int(bool(running)), float(tau), _p(bits, _u32p))
    if st != OK:
        raise ValueError(f"oracle stream_refine status {st}")
    return bits[: s.size // GROUP]
