"""Thin Python binding of libloopkv (the C ABI in include/loopkv.h).

Argument marshalling only: every step of the hot path runs in the library's CUDA kernels.
PyTorch supplies device memory and the current CUDA stream.  The module-level functions
carry the C names; ``Plan`` and ``Cache`` are small owners around them.  If the in-tree
``libloopkv.so`` is missing the import of this module still works, but the first call
raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# LOOPKV_LIB selects another build of the same library (for comparing builds)
LIB_PATH = os.environ.get("LOOPKV_LIB") or os.path.join(_PKG, "libloopkv.so")

LOOPKV_OK = 0
ERRORS = {
    -1: "INVALID_ARG", -2: "SHAPE", -3: "PLAN", -4: "POOL_EXHAUSTED", -5: "NONFINITE", -6: "RANGE",
    -7: "TIMEOUT", -8: "CUDA", -9: "TAIL_FULL", -10: "STATE", -11: "EMPTY_ROW", -12: "NO_DEVICE",
    -13: "INFEASIBLE",
}
CELL_4B, CELL_2B, CELL_SHARE = 0, 1, 2
TAU_REL_MAX, TAU_ABS_PROB, TAU_STREAM = 0, 1, 2
DTYPE_BF16, DTYPE_F32 = 0, 1
DEV_NONFINITE, DEV_RANGE, DEV_POOL_EXHAUSTED, DEV_TAIL_FULL, DEV_STATE, DEV_TIMEOUT, DEV_EMPTY_ROW = (
    0x01, 0x02, 0x04, 0x08, 0x10, 0x20, 0x40)

EXPORTS = [
    "loopkv_plan_create", "loopkv_plan_free", "loopkv_plan_bytes", "loopkv_required_bytes", "loopkv_alloc",
    "loopkv_free", "loopkv_ingest", "loopkv_append", "loopkv_flush", "loopkv_reset_request", "loopkv_decode",
    "loopkv_decode_debug", "loopkv_status", "loopkv_cell_view_get", "loopkv_decode_shape", "loopkv_strerror",
    "loopkv_version", "loopkv_plan_search", "loopkv_append_noalloc", "loopkv_set_wait_policy",
    "loopkv_plan_set_window",
]
INJECT_NONE, INJECT_STALLED_STAGE = 0, 1
NOALLOC_MAX_IDS = 4096


class LoopKVError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        name = ERRORS.get(code, str(code))
        super().__init__(f"{where}: LOOPKV_ERR_{name} ({code})" if where else f"LOOPKV_ERR_{name} ({code})")


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("n_loops", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("max_batch", ctypes.c_int), ("max_blocks_per_seq", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("sink_tokens", ctypes.c_int), ("window_tokens", ctypes.c_int)]


class ByteReport(ctypes.Structure):
    _fields_ = [("stored_bytes_per_token", ctypes.c_double), ("read_bytes_per_token", ctypes.c_double),
                ("read_bytes_all_hot", ctypes.c_double), ("read_bytes_all_cold", ctypes.c_double),
                ("bf16_bytes_per_token", ctypes.c_double)]


class PlanSearchReport(ctypes.Structure):
    _fields_ = [("read_bytes_per_token", ctypes.c_double), ("stored_bytes_per_token", ctypes.c_double),
                ("damage", ctypes.c_double)]


class CellView(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("src_cell", ctypes.c_int), ("src_mode", ctypes.c_int),
                ("head_main_bytes", ctypes.c_int), ("head_lo_bytes", ctypes.c_int),
                ("main_pool", ctypes.c_void_p), ("lo_pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("hist_len", ctypes.c_void_p), ("tail_len", ctypes.c_void_p), ("win_start", ctypes.c_void_p),
                ("tail", ctypes.c_void_p), ("near_cap", ctypes.c_int), ("pool_blocks", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the in-tree library (fails loudly if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with mixed_precision_kv_append_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, ip, i = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int), ctypes.c_int
        L.loopkv_plan_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_uint8), ctypes.c_float, i,
                                         ctypes.POINTER(vp)]
        L.loopkv_plan_free.argtypes = [vp]
        L.loopkv_plan_free.restype = None
        L.loopkv_plan_set_window.argtypes = [vp, i, i]
        L.loopkv_plan_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ByteReport)]
        L.loopkv_required_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t)]
        L.loopkv_alloc.argtypes = [vp, vp, ctypes.c_size_t, vp, ctypes.POINTER(vp)]
        L.loopkv_free.argtypes = [vp]
        L.loopkv_free.restype = None
        L.loopkv_ingest.argtypes = [vp, i, i, i, vp, vp, i, vp]
        L.loopkv_append.argtypes = [vp, i, i, vp, vp, ctypes.POINTER(ctypes.c_int32), i, vp]
        L.loopkv_append_noalloc.argtypes = [vp, i, i, vp, vp, ctypes.POINTER(ctypes.c_int32), i, vp]
        L.loopkv_flush.argtypes = [vp, vp]
        L.loopkv_reset_request.argtypes = [vp, i, vp]
        L.loopkv_decode.argtypes = [vp, i, i, vp, vp, vp, i, vp]
        L.loopkv_decode_debug.argtypes = [vp, i, i, vp, vp, vp, i, vp, vp, vp, vp]
        L.loopkv_status.argtypes = [vp, vp, ip]
        L.loopkv_set_wait_policy.argtypes = [vp, ctypes.c_uint64, i]
        L.loopkv_cell_view_get.argtypes = [vp, i, i, ctypes.POINTER(CellView)]
        L.loopkv_decode_shape.argtypes = [vp, i, ip, ip, ip]
        L.loopkv_strerror.argtypes = [i]
        L.loopkv_strerror.restype = ctypes.c_char_p
        L.loopkv_version.argtypes = []
        L.loopkv_plan_search.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_double), ctypes.c_double,
                                         ctypes.c_double, ctypes.POINTER(ctypes.c_uint8),
                                         ctypes.POINTER(PlanSearchReport)]
        for name in EXPORTS:
            if name not in ("loopkv_plan_free", "loopkv_free", "loopkv_strerror"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int, where: str):
    if rc != LOOPKV_OK:
        raise LoopKVError(rc, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return DTYPE_BF16
    if dt == torch.float32:
        return DTYPE_F32
    raise ValueError(f"unsupported input dtype {dt}")


# ------------------------------------------------------------ C-named functions

def loopkv_plan_search(cfg: Config, damage, damage_budget: float, storage_budget: float = 0.0):
    """Exact plan search (host-only).  damage: [n_loops * n_layers][3] per cell and option.
    Returns (modes list, report dict)."""
    n = cfg.n_loops * cfg.n_layers
    flat = [float(x) for row in damage for x in row]
    if len(flat) != 3 * n:
        raise ValueError("damage must hold 3 values per cell")
    d = (ctypes.c_double * len(flat))(*flat)
    modes = (ctypes.c_uint8 * n)()
    rep = PlanSearchReport()
    _check(lib().loopkv_plan_search(ctypes.byref(cfg), d, float(damage_budget), float(storage_budget), modes,
                                    ctypes.byref(rep)), "loopkv_plan_search")
    return list(modes), {"read_bytes_per_token": rep.read_bytes_per_token,
                         "stored_bytes_per_token": rep.stored_bytes_per_token, "damage": rep.damage}


def loopkv_plan_create(cfg: Config, modes, tau: float, tau_mode: int = TAU_REL_MAX) -> ctypes.c_void_p:
    arr = (ctypes.c_uint8 * len(modes))(*[int(m) for m in modes])
    out = ctypes.c_void_p()
    _check(lib().loopkv_plan_create(ctypes.byref(cfg), arr, ctypes.c_float(tau), tau_mode, ctypes.byref(out)),
           "loopkv_plan_create")
    return out


def loopkv_plan_bytes(plan, hot_fraction=None) -> dict:
    rep = ByteReport()
    hf = None
    if hot_fraction is not None:
        hf = (ctypes.c_float * len(hot_fraction))(*[float(x) for x in hot_fraction])
    _check(lib().loopkv_plan_bytes(plan, hf, ctypes.byref(rep)), "loopkv_plan_bytes")
    return {f: getattr(rep, f) for f, _ in ByteReport._fields_}


def loopkv_required_bytes(plan) -> int:
    n = ctypes.c_size_t()
    _check(lib().loopkv_required_bytes(plan, ctypes.byref(n)), "loopkv_required_bytes")
    return n.value


def loopkv_alloc(plan, buf: torch.Tensor, stream=None) -> ctypes.c_void_p:
    out = ctypes.c_void_p()
    _check(lib().loopkv_alloc(plan, _ptr(buf), buf.numel() * buf.element_size(), _stream(stream),
                              ctypes.byref(out)), "loopkv_alloc")
    return out


def loopkv_ingest(cache, loop: int, layer: int, req: int, k: torch.Tensor, v: torch.Tensor, stream=None):
    _check(lib().loopkv_ingest(cache, loop, layer, req, _ptr(k), _ptr(v), int(k.shape[0]), _stream(stream)),
           "loopkv_ingest")


def loopkv_append(cache, loop: int, layer: int, k: torch.Tensor, v: torch.Tensor, req_ids=None, stream=None):
    ids = None
    B = int(k.shape[0])
    if req_ids is not None:
        ids = (ctypes.c_int32 * B)(*[int(r) for r in req_ids])
    _check(lib().loopkv_append(cache, loop, layer, _ptr(k), _ptr(v), ids, B, _stream(stream)), "loopkv_append")


def loopkv_append_noalloc(cache, loop: int, layer: int, k: torch.Tensor, v: torch.Tensor, req_ids=None,
                          stream=None):
    """loopkv_append with the request ids staged in the library's fixed device array (the call
    allocates nothing)."""
    ids = None
    B = int(k.shape[0])
    if req_ids is not None:
        ids = (ctypes.c_int32 * B)(*[int(r) for r in req_ids])
    _check(lib().loopkv_append_noalloc(cache, loop, layer, _ptr(k), _ptr(v), ids, B, _stream(stream)),
           "loopkv_append_noalloc")


def loopkv_flush(cache, stream=None):
    _check(lib().loopkv_flush(cache, _stream(stream)), "loopkv_flush")


def loopkv_reset_request(cache, req: int, stream=None):
    _check(lib().loopkv_reset_request(cache, req, _stream(stream)), "loopkv_reset_request")


def loopkv_decode(plan, loop: int, layer: int, q: torch.Tensor, cache, out: torch.Tensor, stream=None):
    _check(lib().loopkv_decode(plan, loop, layer, _ptr(q), cache, _ptr(out), int(q.shape[0]), _stream(stream)),
           "loopkv_decode")


def loopkv_decode_debug(plan, loop, layer, q, cache, out, s_bitmap=None, row_max=None, row_sum=None, stream=None):
    _check(lib().loopkv_decode_debug(plan, loop, layer, _ptr(q), cache, _ptr(out), int(q.shape[0]), _stream(stream),
                                     _ptr(s_bitmap), _ptr(row_max), _ptr(row_sum)), "loopkv_decode_debug")


def loopkv_status(cache, stream=None) -> tuple[int, int]:
    bits = ctypes.c_int()
    rc = lib().loopkv_status(cache, _stream(stream), ctypes.byref(bits))
    return rc, bits.value


def loopkv_set_wait_policy(cache, wait_limit_ns: int, inject: int = INJECT_NONE):
    _check(lib().loopkv_set_wait_policy(cache, int(wait_limit_ns), int(inject)), "loopkv_set_wait_policy")


def loopkv_cell_view_get(cache, loop: int, layer: int) -> CellView:
    v = CellView()
    _check(lib().loopkv_cell_view_get(cache, loop, layer, ctypes.byref(v)), "loopkv_cell_view_get")
    return v


def loopkv_decode_shape(plan, B: int) -> dict:
    c, n, s = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().loopkv_decode_shape(plan, B, ctypes.byref(c), ctypes.byref(n), ctypes.byref(s)),
           "loopkv_decode_shape")
    return dict(cluster=c.value, ctas=n.value, smem=s.value)


def loopkv_strerror(code: int) -> str:
    return lib().loopkv_strerror(code).decode()


# -------------------------------------------------------------------- owners

class Plan:
    """A plan: config + one storage mode per (loop, layer) cell + tau (host object)."""

    def __init__(self, n_layers, n_loops, n_heads, head_dim, max_batch, max_blocks_per_seq, modes, tau,
                 tau_mode=TAU_REL_MAX, in_dtype=torch.bfloat16, sink_tokens=0, window_tokens=0):
        self.cfg = Config(n_layers, n_loops, n_heads, head_dim, max_batch, max_blocks_per_seq,
                          _dtype_code(in_dtype), sink_tokens, window_tokens)
        self.sink, self.window = sink_tokens, window_tokens
        self.in_dtype = in_dtype
        self.modes = [int(m) for m in modes]
        self.tau = float(tau)
        self.tau_mode = tau_mode
        self.handle = loopkv_plan_create(self.cfg, self.modes, self.tau, tau_mode)

    @property
    def n_cells(self):
        return self.cfg.n_loops * self.cfg.n_layers

    def cell(self, loop, layer):
        return loop * self.cfg.n_layers + layer

    def bytes(self, hot_fraction=None) -> dict:
        return loopkv_plan_bytes(self.handle, hot_fraction)

    def required_bytes(self) -> int:
        return loopkv_required_bytes(self.handle)

    def set_window(self, layer: int, window_tokens: int):
        """Sliding attention window of a layer (0 = full attention)."""
        _check(lib().loopkv_plan_set_window(self.handle, layer, window_tokens), "loopkv_plan_set_window")
        self.windows = getattr(self, "windows", {})
        self.windows[layer] = window_tokens

    def decode_shape(self, B) -> dict:
        return loopkv_decode_shape(self.handle, B)

    def close(self):
        if self.handle:
            lib().loopkv_plan_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cache:
    """A cache carved out of one torch-owned device buffer."""

    def __init__(self, plan: Plan, nbytes: int | None = None, device=None, stream=None):
        self.plan = plan
        if nbytes is None:
            nbytes = plan.required_bytes()
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
        self.handle = loopkv_alloc(plan.handle, self.buf, stream)

    def ingest(self, loop, layer, req, k, v, stream=None):
        loopkv_ingest(self.handle, loop, layer, req, k, v, stream)

    def append(self, loop, layer, k, v, req_ids=None, stream=None):
        loopkv_append(self.handle, loop, layer, k, v, req_ids, stream)

    def flush(self, stream=None):
        loopkv_flush(self.handle, stream)

    def reset_request(self, req, stream=None):
        loopkv_reset_request(self.handle, req, stream)

    def decode(self, loop, layer, q, out=None, stream=None, plan: Plan | None = None):
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        loopkv_decode((plan or self.plan).handle, loop, layer, q, self.handle, out, stream)
        return out

    def decode_debug(self, loop, layer, q, stream=None, plan: Plan | None = None):
        B, H = int(q.shape[0]), int(q.shape[1])
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        words = self.plan.cfg.max_blocks_per_seq // 2
        bm = torch.zeros((B, H, words), dtype=torch.int32, device=q.device)
        rm = torch.empty((B, H), dtype=torch.float32, device=q.device)
        rs = torch.empty((B, H), dtype=torch.float32, device=q.device)
        loopkv_decode_debug((plan or self.plan).handle, loop, layer, q, self.handle, out, bm, rm, rs, stream)
        return out, bm, rm, rs

    def status(self, stream=None) -> tuple[int, int]:
        return loopkv_status(self.handle, stream)

    def check(self, where="device"):
        rc, bits = self.status()
        if rc != LOOPKV_OK:
            raise LoopKVError(rc, f"{where} (status bits {bits:#x})")

    def cell_view(self, loop, layer) -> CellView:
        return loopkv_cell_view_get(self.handle, loop, layer)

    def _slice(self, addr: int, nbytes: int) -> torch.Tensor:
        off = addr - self.buf.data_ptr()
        assert 0 <= off and off + nbytes <= self.buf.numel()
        return self.buf[off: off + nbytes]

    def lengths(self, loop, layer) -> tuple[torch.Tensor, torch.Tensor]:
        """(history lengths of the source cell, near (sink + window) token counts of this cell),
        [max_batch] int32 on host."""
        v = self.cell_view(loop, layer)
        mb = self.plan.cfg.max_batch
        h = self._slice(v.hist_len, 4 * mb).view(torch.int32).cpu()
        t = self._slice(v.tail_len, 4 * mb).view(torch.int32).cpu()
        return h, t

    def block_table(self, loop, layer) -> torch.Tensor:
        v = self.cell_view(loop, layer)
        mb, nb = self.plan.cfg.max_batch, self.plan.cfg.max_blocks_per_seq
        return self._slice(v.block_table, 4 * mb * nb).view(torch.int32).view(mb, nb).cpu()

    def head_blocks(self, loop, layer, req) -> tuple[torch.Tensor, torch.Tensor]:
        """Packed bytes of the source cell's history of request `req`: main [n_blocks][H][head_main],
        lo [n_blocks][H][head_lo] (empty for 2-bit)."""
        v = self.cell_view(loop, layer)
        H = self.plan.cfg.n_heads
        hist, _ = self.lengths(loop, layer)
        nb = int(hist[req]) // 16
        ids = self.block_table(loop, layer)[req, :nb].tolist()
        mains, los = [], []
        for b in ids:
            mains.append(self._slice(v.main_pool + b * H * v.head_main_bytes, H * v.head_main_bytes)
                         .view(H, v.head_main_bytes))
            if v.head_lo_bytes:
                los.append(self._slice(v.lo_pool + b * H * v.head_lo_bytes, H * v.head_lo_bytes)
                           .view(H, v.head_lo_bytes))
        main = torch.stack(mains).cpu() if mains else torch.zeros((0, H, v.head_main_bytes), dtype=torch.uint8)
        lo = torch.stack(los).cpu() if los else torch.zeros((0, H, v.head_lo_bytes), dtype=torch.uint8)
        return main, lo

    def tail(self, loop, layer, req) -> torch.Tensor:
        """Unquantized near slots of this cell for `req`: [2][H][near_cap][D] in the input dtype
        (device view): the sink slots, then the window ring."""
        v = self.cell_view(loop, layer)
        c = self.plan.cfg
        esz = 2 if self.plan.in_dtype == torch.bfloat16 else 4
        per = 2 * c.n_heads * v.near_cap * c.head_dim * esz
        t = self._slice(v.tail + req * per, per)
        return t.view(self.plan.in_dtype).view(2, c.n_heads, v.near_cap, c.head_dim)

    def near_tokens(self, loop, layer, req) -> torch.Tensor:
        """The near tokens of this cell for `req` in arrival order: [2][H][n][D] (a copy): sink first,
        then the window from its oldest token."""
        v = self.cell_view(loop, layer)
        mb = self.plan.cfg.max_batch
        n = int(self._slice(v.tail_len, 4 * mb).view(torch.int32)[req])
        ws = int(self._slice(v.win_start, 4 * mb).view(torch.int32)[req])
        S, WR = self.plan.sink, self.plan.window + 32
        slots = [j if j < S else S + (ws + j - S) % WR for j in range(n)]
        return self.tail(loop, layer, req)[:, :, slots].clone()

    def close(self):
        if self.handle:
            lib().loopkv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
