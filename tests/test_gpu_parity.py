"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Every case feeds the same seeded inputs to libloopkv and to the oracle and checks:
  * packed history bytes (codes, fp16 scales and zeros, hi/lo planes) bit-exact;
  * the refine set S bit-exact except within 1e-6 of tau (tie band);
  * outputs within 2e-3 absolute, row max and row sum within 1e-4 relative.
"""
import numpy as np
import pytest
import torch

from lkv_helpers import bits_of, check_row, f32, words_from_bits
from mixed_precision_kv_append_b200 import loopkv as L
from mixed_precision_kv_append_b200 import synth
from oracle import oracle as O

pytestmark = pytest.mark.gpu

BITS = {L.CELL_4B: 4, L.CELL_2B: 2}


def _plan(n_layers, n_loops, H, D, B, max_blocks, modes, tau, tau_mode=L.TAU_REL_MAX, dtype=torch.bfloat16, sink=0,
          window=0):
    return L.Plan(n_layers, n_loops, H, D, B, max_blocks, modes, tau, tau_mode, dtype, sink, window)


class Model:
    """A small cache plus the raw token history of every (cell, request), as the oracle sees it."""

    def __init__(self, w: synth.Workload, max_blocks=None, tau=None, tau_mode=None, sink=0, window=0):
        self.w = w
        self.tau = w.tau if tau is None else tau
        self.tau_mode = w.tau_mode if tau_mode is None else tau_mode
        self.sink = sink
        self.plan = _plan(w.n_layers, w.n_loops, w.H, w.D, w.B, max_blocks or w.max_blocks, w.modes, self.tau,
                          self.tau_mode, w.dtype, sink, window)
        self.cache = L.Cache(self.plan)
        self.tokens = {}  # (cell, req) -> (K [n, H, D] float32, V)
        self._hist_cache = {}

    def cell(self, loop, layer):
        return loop * self.w.n_layers + layer

    def src(self, loop, layer):
        c = self.cell(loop, layer)
        if self.w.modes[c] == L.CELL_SHARE:
            return self.cell(self.w.n_loops - 1, layer)
        return c

    def ingest(self, T_override=None):
        w = self.w
        for layer in range(w.n_layers):
            for req in range(w.B):
                T = w.lengths[req] if T_override is None else T_override[req]
                ks, vs = synth.layer_history(w, layer, req, T=T, device="cuda")
                for lp in range(w.n_loops):
                    self.cache.ingest(lp, layer, req, ks[lp].contiguous(), vs[lp].contiguous())
                    self.tokens[(self.cell(lp, layer), req)] = (f32(ks[lp]), f32(vs[lp]))
        self.cache.check("ingest")

    def append_step(self, step):
        w = self.w
        self.cache.flush()
        for layer in range(w.n_layers):
            _, ks, vs = synth.step_tokens(w, step, layer, device="cuda")
            for lp in range(w.n_loops):
                self.cache.append(lp, layer, ks[lp].contiguous(), vs[lp].contiguous())
                c = self.cell(lp, layer)
                for req in range(w.B):
                    K, V = self.tokens[(c, req)]
                    self.tokens[(c, req)] = (np.concatenate([K, f32(ks[lp][req:req + 1])]),
                                             np.concatenate([V, f32(vs[lp][req:req + 1])]))
        self._hist_cache.clear()

    def head_history(self, cell, req, h, n_hist):
        """Quantized history of a head: the n_hist tokens after the sink."""
        key = (cell, req, h, n_hist)
        if key not in self._hist_cache:
            K, V = self.tokens[(cell, req)]
            S = self.sink
            self._hist_cache[key] = O.HeadHistory(K[S:S + n_hist, h], V[S:S + n_hist, h], BITS[self.w.modes[cell]]) \
                if n_hist else None
        return self._hist_cache[key]

    def raw_tokens(self, K, V, n_hist, n_near):
        """The unquantized tokens of a sequence: the sink, then the window after the history."""
        if n_hist == 0:
            return K[:n_near], V[:n_near]
        S = self.sink
        return np.concatenate([K[:S], K[S + n_hist:]]), np.concatenate([V[:S], V[S + n_hist:]])

    def check_cell(self, loop, layer, q, rows=None, where=""):
        """Decode cell (loop, layer) on the GPU and compare the given (req, head) rows."""
        w = self.w
        out, bm, rm, rs = self.cache.decode_debug(loop, layer, q)
        self.cache.check(f"decode {where}")
        hist, tail = self.cache.lengths(loop, layer)
        c, s = self.cell(loop, layer), self.src(loop, layer)
        out, bm, rm, rs = f32(out), bm.cpu().numpy().view(np.uint32), f32(rm), f32(rs)
        qn = f32(q)
        rows = rows if rows is not None else [(r, h) for r in range(w.B) for h in range(w.H)]
        worst, ties = 0.0, 0
        for req, h in rows:
            n_hist, n_tail = int(hist[req]), int(tail[req])
            K, V = self.tokens[(c, req)]
            n_own = K.shape[0]
            assert n_own == n_hist + n_tail, (n_own, n_hist, n_tail)
            hh = self.head_history(s, req, h, n_hist)
            Kr, Vr = self.raw_tokens(K, V, n_hist, n_tail)
            win = getattr(self.plan, "windows", {}).get(layer, 0)
            h0 = 0
            if win:  # sliding window: the last `win` positions (sink, history, window in order)
                n = n_hist + n_tail
                h0 = min(max(n - win - self.sink, 0), n_hist)
                pos = np.array([j if j < self.sink else n_hist + j for j in range(n_tail)])
                keep = pos >= n - win
                Kr, Vr = Kr[keep], Vr[keep]
            err, nt = check_row(out[req, h], bm[req, h], rm[req, h], rs[req, h], qn[req, h].astype(np.float64),
                                hh, Kr[:, h], Vr[:, h], self.tau, self.tau_mode,
                                where=f"{where} cell ({loop},{layer}) req {req} head {h}", hist_first=h0)
            worst, ties = max(worst, err), ties + nt
        return worst, ties

    def check_bytes(self, loop, layer, reqs=None, heads=None):
        """Packed bytes of the cell's own pages against the oracle's packing."""
        w = self.w
        c = self.cell(loop, layer)
        assert w.modes[c] != L.CELL_SHARE
        hist, _ = self.cache.lengths(loop, layer)
        for req in (reqs if reqs is not None else range(w.B)):
            main, lo = self.cache.head_blocks(loop, layer, req)
            n_hist = int(hist[req])
            assert main.shape[0] == n_hist // 16
            for h in (heads if heads is not None else range(w.H)):
                hh = self.head_history(c, req, h, n_hist)
                if hh is None:
                    continue
                om, ol = hh.packed_blocks()
                assert np.array_equal(main[:, h].numpy(), om), f"main bytes differ: cell {c} req {req} head {h}"
                if BITS[w.modes[c]] == 4:
                    assert np.array_equal(lo[:, h].numpy(), ol), f"lo bytes differ: cell {c} req {req} head {h}"


def _q(w, step, layer, loop):
    qs, _, _ = synth.step_tokens(w, step, layer, device="cuda")
    return qs[loop].contiguous()


def test_tiny_config_bytes_and_decode():
    w = synth.workload("tiny")
    m = Model(w)
    m.ingest()
    for lp in range(2):
        m.check_bytes(lp, 0)
        m.check_cell(lp, 0, _q(w, 0, 0, lp), where="tiny")


@pytest.mark.parametrize("tau,tau_mode", [(0.0, 0), (0.01, 0), (0.3, 0), (1.5, 0), (0.002, 1), (0.05, 1)])
def test_ragged_rows_tails_and_share_cells(tau, tau_mode):
    # loop 0: [share of a 4-bit cell, 4-bit]; loop 1: [2-bit, share of a 2-bit cell]; loop 2 (final): [4b, 2b]
    modes = [L.CELL_SHARE, L.CELL_4B, L.CELL_2B, L.CELL_SHARE, L.CELL_4B, L.CELL_2B]
    w = synth.Workload("ragged_small", 2, 3, 4, 128, 5, [5, 37, 300, 1000, 64], torch.bfloat16, modes, tau,
                       tau_mode=tau_mode, seed=3)
    m = Model(w)
    m.ingest()
    for layer in range(2):
        for lp in range(3):
            if modes[m.cell(lp, layer)] != L.CELL_SHARE:
                m.check_bytes(lp, layer)
            m.check_cell(lp, layer, _q(w, 1, layer, lp), where=f"tau={tau} mode={tau_mode}")


def test_head_dim_64_bf16_and_fp32_tails():
    for dtype in (torch.float32, torch.bfloat16):
        w = synth.Workload("d64", 1, 2, 2, 64, 2, [100, 257], dtype, [L.CELL_2B, L.CELL_4B], 0.05, seed=5)
        m = Model(w)
        m.ingest()
        for lp in range(2):
            m.check_bytes(lp, 0)
            m.check_cell(lp, 0, _q(w, 0, 0, lp), where=f"d64 {dtype}")


def test_append_flush_sequence():
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # 2 layers x 2 loops
    w = synth.Workload("append", 2, 2, 4, 128, 3, [20, 64, 95], torch.bfloat16, modes, 0.02, append_steps=70,
                       seed=7)
    m = Model(w)
    m.ingest()
    for step in range(70):
        m.append_step(step)
        if step % 9 == 0 or step in (11, 12, 43, 44, 69):
            for layer in range(2):
                for lp in range(2):
                    m.check_cell(lp, layer, _q(w, step, layer, lp), where=f"step {step}")
    m.cache.check("append sequence")
    for layer in range(2):
        for lp in range(2):
            if modes[m.cell(lp, layer)] != L.CELL_SHARE:
                m.check_bytes(lp, layer)
            hist, tail = m.cache.lengths(lp, layer)
            for req in range(w.B):
                n = w.lengths[req] + 70
                assert int(tail[req]) >= 1 and int(hist[req]) % 32 == 0 and int(hist[req]) + int(tail[req]) == n


@pytest.mark.parametrize("lengths", [[4096, 1000, 33], [2048] * 3])
def test_repeated_single_pass_decode_is_bit_identical(lengths):
    # 2-bit cells and tau = 0 reads (single-pass reader, rows split over the CTAs of a cluster
    # and merged through distributed shared memory): a second launch must repeat the first.
    modes = [L.CELL_2B, L.CELL_4B]
    w = synth.Workload("repeat", 1, 2, 4, 128, 3, lengths, torch.bfloat16, modes, 0.0, seed=11)
    m = Model(w)
    m.ingest()
    for lp in range(2):
        q = _q(w, 0, 0, lp)
        first = m.cache.decode(lp, 0, q)
        second = m.cache.decode(lp, 0, q)
        m.cache.check("repeat")
        assert torch.equal(first, second)
        m.check_cell(lp, 0, q, where=f"repeat loop {lp}")


def test_share_cell_with_final_loop_query_is_bit_identical():
    modes = [L.CELL_SHARE, L.CELL_4B]
    w = synth.Workload("share", 1, 2, 4, 128, 2, [512, 1024], torch.bfloat16, modes, 0.01, seed=9)
    m = Model(w)
    m.ingest()  # multiples of 32: every tail is empty
    q = _q(w, 0, 0, 1)
    a = m.cache.decode(0, 0, q)
    b = m.cache.decode(1, 0, q)
    m.cache.check("share")
    assert torch.equal(a, b)


@pytest.mark.parametrize("tau,tau_mode,D,dtype,sink,window", [
    (0.01, 0, 128, torch.bfloat16, 0, 0), (0.05, 1, 128, torch.bfloat16, 0, 0), (0.0, 0, 128, torch.bfloat16, 0, 0),
    (0.02, 0, 64, torch.float32, 0, 0), (0.01, 0, 128, torch.bfloat16, 32, 64), (0.02, 0, 64, torch.float32, 32, 96)])
def test_lean_build_matches_general_build(tau, tau_mode, D, dtype, sink, window):
    """loopkv_decode without debug outputs runs the lean kernel builds (no refine-set bitmap,
    streaming rule, sliding window or test hook on their per-group path; with a sink or window, the
    build that streams the near region); they must give the outputs of the general builds, which
    the other cases check against the oracle, bit for bit."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("lean", 2, 2, 4, D, 3, [4096, 1000, 33], dtype, modes, tau, tau_mode=tau_mode,
                       append_steps=5, seed=21)
    m = Model(w, sink=sink, window=window)
    m.ingest()
    for step in range(5):
        m.append_step(step)
    for la in range(2):
        for lp in range(2):
            q = _q(w, 4, la, lp)
            lean = m.cache.decode(lp, la, q)
            general, _, _, _ = m.cache.decode_debug(lp, la, q)
            m.cache.check("lean vs general build")
            assert torch.equal(lean, general), f"cell ({lp},{la})"
    m.check_cell(0, 0, _q(w, 4, 0, 0), where="lean")


@pytest.mark.parametrize("name,B,T,modes,tau,steps", [
    ("kivi4_8k", 8, [8192] * 8, [0, 0, 0, 0], 0.0, 0),
    ("mixed_8k", 32, [8192] * 32, [0, 1, 2, 0], 0.01, 0),
    ("long_16k", 32, [16384] * 32, [0, 2, 1, 0], 0.005, 2),
    ("ragged_2p6b", 8, None, [1, 2, 0, 0], 0.01, 0),
    ("ouro2p6b_32k", 8, [32768] * 8, [2, 1, 0, 0], 0.01, 0),
])
def test_full_size_sampled_rows(name, B, T, modes, tau, steps):
    """Benchmark shapes (one layer of four loops): the launch configuration the benchmark times,
    checked on sampled rows of every cell and on the packed bytes of sampled heads."""
    base = synth.workload(name)
    lengths = T if T is not None else base.lengths
    w = synth.Workload(name, 1, 4, 16, 128, B, lengths, torch.bfloat16, modes, tau, append_steps=steps, seed=1)
    m = Model(w, max_blocks=base.max_blocks)
    m.ingest()
    for s in range(steps):
        m.append_step(s)
    rng = np.random.default_rng(0)
    for lp in range(4):
        rows = [(int(rng.integers(B)), int(rng.integers(16))) for _ in range(5)] + [(B - 1, 15), (0, 0)]
        m.check_cell(lp, 0, _q(w, steps, 0, lp), rows=rows, where=name)
        if modes[lp] != L.CELL_SHARE:
            m.check_bytes(lp, 0, reqs=[0, B - 1], heads=[0, 7])


@pytest.mark.parametrize("score_bufs", ["1", "2"])
def test_two_phase_score_buffer_orders(monkeypatch, score_bufs):
    """The decide path (4-bit, tau > 0) with one score buffer (a cluster's rows in sequence)
    and with two (the next row's keys overlapping the current row's values), forced through
    the launch-shape override on a batch with more rows than clusters."""
    base = synth.workload("mixed_8k")
    w = synth.Workload("mixed_8k", 1, 4, 16, 128, 32, [8192] * 32, torch.bfloat16, [0, 1, 2, 0], 0.01, seed=2)
    shapes = {}
    for nb in ("1", "2"):  # the override takes effect: two score buffers take more shared memory
        monkeypatch.setenv("LOOPKV_DECODE_SHAPE", f"4,0,0,{nb},0")  # clusters of 4 in both
        shapes[nb] = L.Plan(1, 4, 16, 128, 32, base.max_blocks, [0, 1, 2, 0], 0.01).decode_shape(32)
    assert shapes["2"]["smem"] > shapes["1"]["smem"]
    monkeypatch.setenv("LOOPKV_DECODE_SHAPE", f"4,0,0,{score_bufs},0")
    # more rows (32 requests x 16 heads) than clusters: every cluster reads several rows in order
    assert 32 * 16 > shapes[score_bufs]["ctas"] // shapes[score_bufs]["cluster"]
    m = Model(w, max_blocks=base.max_blocks)
    m.ingest()
    rng = np.random.default_rng(1)
    for lp in (0, 2, 3):  # 4-bit, share of a 4-bit source, final loop
        rows = [(int(rng.integers(32)), int(rng.integers(16))) for _ in range(6)] + [(31, 15), (0, 0)]
        m.check_cell(lp, 0, _q(w, 0, 0, lp), rows=rows, where=f"score buffers {score_bufs}")


def test_graph_replay_matches_eager():
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("graph", 2, 2, 4, 128, 3, [33, 64, 200], torch.bfloat16, modes, 0.01, append_steps=40,
                       seed=11)
    m = Model(w)
    m.ingest()
    qs = [[_q(w, 0, layer, lp) for lp in range(2)] for layer in range(2)]
    _, ks, vs = synth.step_tokens(w, 0, 0, device="cuda")
    outs = [[torch.empty_like(qs[0][0], dtype=torch.float32) for _ in range(2)] for _ in range(2)]
    for layer in range(2):  # eager decodes fix each cell's launch shape before the capture
        for lp in range(2):
            m.cache.decode(lp, layer, qs[layer][lp])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        m.cache.flush(stream=s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            m.cache.flush(stream=s)
            for layer in range(2):
                for lp in range(2):
                    m.cache.append(lp, layer, ks[lp], vs[lp], stream=s)
                    L.loopkv_decode(m.plan.handle, lp, layer, qs[layer][lp], m.cache.handle, outs[layer][lp],
                                    stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(35):
        g.replay()
        torch.cuda.synchronize()
        for layer in range(2):
            for lp in range(2):
                c = m.cell(lp, layer)
                for req in range(w.B):
                    K, V = m.tokens[(c, req)]
                    m.tokens[(c, req)] = (np.concatenate([K, f32(ks[lp][req:req + 1])]),
                                          np.concatenate([V, f32(vs[lp][req:req + 1])]))
        m._hist_cache.clear()
        if rep in (0, 30, 34):
            for layer in range(2):
                for lp in range(2):
                    ref = outs[layer][lp].clone()
                    eager = m.cache.decode(lp, layer, qs[layer][lp])
                    assert torch.equal(ref, eager)
                    m.check_cell(lp, layer, qs[layer][lp], where=f"graph replay {rep}")
    m.cache.check("graph")


def test_device_errors_are_reported():
    modes = [L.CELL_4B, L.CELL_4B]
    w = synth.Workload("err", 1, 2, 2, 64, 2, [64, 64], torch.float32, modes, 0.01, seed=13)
    m = Model(w, max_blocks=8)
    m.ingest()
    # ingest into a non-empty (cell, request)
    k = torch.zeros((32, 2, 64), device="cuda")
    m.cache.ingest(0, 0, 0, k, k)
    assert m.cache.status() == (-10, L.DEV_STATE)
    # a 33rd token in a tail without flush
    for _ in range(33):
        m.cache.append(0, 0, torch.zeros((2, 2, 64), device="cuda"), torch.zeros((2, 2, 64), device="cuda"))
    rc, bits = m.cache.status()
    assert rc == -9 and bits & L.DEV_TAIL_FULL
    # non-finite and out-of-range groups
    m.cache.reset_request(1)
    bad = torch.randn((32, 2, 64), device="cuda")
    bad[3, 1, 7] = float("nan")
    m.cache.ingest(1, 0, 1, bad, torch.randn((32, 2, 64), device="cuda"))
    rc, bits = m.cache.status()
    assert rc == -5 and bits & L.DEV_NONFINITE
    m.cache.reset_request(1)
    big = torch.randn((32, 2, 64), device="cuda")
    big[0, 0, 0] = -1e6
    m.cache.ingest(1, 0, 1, big, torch.randn((32, 2, 64), device="cuda"))
    rc, bits = m.cache.status()
    assert rc == -6 and bits & L.DEV_RANGE
    # host-side argument errors come back before any launch
    with pytest.raises(L.LoopKVError):
        m.cache.ingest(5, 0, 0, k, k)
    with pytest.raises(L.LoopKVError):
        m.cache.ingest(0, 0, 0, torch.zeros((10 * 32, 2, 64), device="cuda"), torch.zeros((320, 2, 64),
                                                                                          device="cuda"))


def test_pool_exhaustion_and_reset():
    modes = [L.CELL_4B]
    w = synth.Workload("pool", 1, 1, 2, 64, 4, [64] * 4, torch.float32, modes, 0.0, seed=17)
    plan = _plan(1, 1, 2, 64, 4, 8, modes, 0.0, dtype=torch.float32)
    need = plan.required_bytes()
    per_block = 2 * (1024 + 256)
    cache = L.Cache(plan, nbytes=need - 20 * per_block)  # room for fewer than 16 blocks
    ks, vs = synth.layer_history(w, 0, 0, T=64, device="cuda")
    for req in range(4):
        cache.ingest(0, 0, req, ks[0], vs[0])
    rc, bits = cache.status()
    assert rc == -4 and bits & L.DEV_POOL_EXHAUSTED
    hist, _ = cache.lengths(0, 0)
    full = [r for r in range(4) if int(hist[r]) == 64]
    assert len(full) >= 1
    cache.reset_request(full[0])
    hist, _ = cache.lengths(0, 0)
    assert int(hist[full[0]]) == 0
    missing = [r for r in range(4) if int(hist[r]) == 0 and r != full[0]][0]
    cache.ingest(0, 0, missing, ks[0], vs[0])
    assert cache.status() == (0, 0)


def test_empty_row_is_reported():
    plan = _plan(1, 1, 2, 64, 1, 4, [L.CELL_4B], 0.0, dtype=torch.float32)
    cache = L.Cache(plan)
    out = cache.decode(0, 0, torch.randn((1, 2, 64), device="cuda"))
    rc, bits = cache.status()
    assert rc == -11 and bits & L.DEV_EMPTY_ROW
    assert torch.all(out == 0)


def test_decode_shape_reports_cluster_launch():
    p = L.Plan(24, 4, 16, 128, 8, 514, [0] * 96, 0.0)
    shp = p.decode_shape(8)
    assert shp["cluster"] in (1, 2, 3, 4, 5, 6, 7, 8, 16) and shp["ctas"] % shp["cluster"] == 0
    assert shp["ctas"] >= 148 and 0 < shp["smem"] <= 227 * 1024


@pytest.mark.parametrize("modes,tau", [([L.CELL_4B, L.CELL_4B], 0.01), ([L.CELL_2B, L.CELL_4B], 0.0)])
def test_bounded_wait_gives_up_and_recovers(modes, tau):
    """A stage armed for bytes that are never requested (the injection hook) makes its wait run
    out after the short limit: the decode reports LOOPKV_ERR_TIMEOUT, the stream completes, and
    the next decode with the normal policy matches the oracle.  Both kernels: the exact-maximum
    reader (4-bit, tau > 0) and the single-pass reader (2-bit / tau = 0)."""
    w = synth.Workload("timeout", 1, 2, 4, 128, 3, [512, 96, 1000], torch.bfloat16, modes, tau, seed=23)
    m = Model(w)
    m.ingest()
    q = _q(w, 0, 0, 0)
    L.loopkv_set_wait_policy(m.cache.handle, 200_000, L.INJECT_STALLED_STAGE)
    m.cache.decode(0, 0, q)
    torch.cuda.synchronize()
    rc, bits = m.cache.status()
    assert rc == -7 and bits & L.DEV_TIMEOUT
    L.loopkv_set_wait_policy(m.cache.handle, 500_000_000, L.INJECT_NONE)
    m.check_cell(0, 0, q, where="after a timed-out decode")
    assert m.cache.status() == (0, 0)
    with pytest.raises(L.LoopKVError):
        L.loopkv_set_wait_policy(m.cache.handle, 0, L.INJECT_NONE)


@pytest.mark.parametrize("graph", [False, True])
def test_flush_then_decode_without_append(graph):
    """A decode launched right after a flush on the same stream (no append between) reads the
    lengths and block tables the flush wrote, in eager mode and inside a captured graph."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("flushdec", 2, 2, 4, 128, 3, [20, 64, 95], torch.bfloat16, modes, 0.01, append_steps=40,
                       seed=29)
    m = Model(w)
    m.ingest()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    outs = {}
    qs = {(lp, la): _q(w, 5, la, lp) for lp in range(2) for la in range(2)}
    for step in range(36):  # every tail fills up at least once
        _, ks, vs = synth.step_tokens(w, step, 0, device="cuda")
        with torch.cuda.stream(s):
            m.cache.flush(stream=s)
            for la in range(2):
                for lp in range(2):
                    m.cache.append(lp, la, ks[lp].contiguous(), vs[lp].contiguous(), stream=s)
        s.synchronize()
        for la in range(2):
            for lp in range(2):
                c = m.cell(lp, la)
                for req in range(w.B):
                    K, V = m.tokens[(c, req)]
                    m.tokens[(c, req)] = (np.concatenate([K, f32(ks[lp][req:req + 1])]),
                                          np.concatenate([V, f32(vs[lp][req:req + 1])]))
    m._hist_cache.clear()
    for la in range(2):  # launch shapes fixed before any capture
        for lp in range(2):
            outs[(lp, la)] = m.cache.decode(lp, la, qs[(lp, la)])
    torch.cuda.synchronize()

    def step(stream):
        m.cache.flush(stream=stream)
        for la in range(2):
            for lp in range(2):
                L.loopkv_decode(m.plan.handle, lp, la, qs[(lp, la)], m.cache.handle, outs[(lp, la)], stream=stream)

    with torch.cuda.stream(s):
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                step(s)
            g.replay()
        else:
            step(s)
    s.synchronize()
    m.cache.check("flush then decode")
    for la in range(2):
        for lp in range(2):
            hist, tail = m.cache.lengths(lp, la)
            assert all(int(tail[r]) < 32 for r in range(w.B))
            ref = outs[(lp, la)].clone()
            again = m.cache.decode(lp, la, qs[(lp, la)])
            assert torch.equal(ref, again)
            m.check_cell(lp, la, qs[(lp, la)], where=f"flush then decode graph={graph}")


@pytest.mark.parametrize("sink,window", [(32, 64), (32, 256), (0, 96)])
def test_sink_window_sequence(sink, window):
    """Sink and window stay unquantized (LoopKV §2.3, §3.4): requests whose tokens are all in the
    sink, that have a window but no history, and that have history between sink and window;
    appends fill the window ring and each flush quantizes its oldest page.  Packed pages are
    bit-exact with the oracle's quantization of the tokens after the sink, decodes match."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("sinkwin", 2, 2, 4, 128, 3, [20, sink + window + 4, 600], torch.bfloat16, modes, 0.02,
                       append_steps=80, seed=31)
    m = Model(w, sink=sink, window=window)
    m.ingest()
    for lp in range(2):
        for la in range(2):
            m.check_cell(lp, la, _q(w, 0, la, lp), where=f"ingest s={sink} w={window}")
    for step in range(80):
        m.append_step(step)
        if step % 17 == 0 or step in (31, 32, 33, 79):
            for la in range(2):
                for lp in range(2):
                    m.check_cell(lp, la, _q(w, step, la, lp), where=f"s={sink} w={window} step {step}")
    m.cache.check("sink/window sequence")
    for la in range(2):
        for lp in range(2):
            c = m.cell(lp, la)
            if modes[c] != L.CELL_SHARE:
                m.check_bytes(lp, la)
            hist, near = m.cache.lengths(lp, la)
            for req in range(w.B):
                n = w.lengths[req] + 80
                h, nn = int(hist[req]), int(near[req])
                assert h + nn == n and h % 32 == 0
                if h:
                    assert sink + window <= nn <= sink + window + 32  # a full window is flushed at the next step
                # the near slots hold exactly the sink and the window, in arrival order
                K, _ = m.tokens[(c, req)]
                Kr, _ = m.raw_tokens(K, K, h, nn)
                got = f32(m.cache.near_tokens(lp, la, req)[0]).transpose(1, 0, 2)
                assert np.array_equal(got, Kr.astype(np.float32)), (lp, la, req)


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_sink_window_single_pass_all_hot(D, dtype):
    """tau = 0 on 4-bit cells (every lo plane read: the single-pass reader) with a sink and a window:
    the near region streams through that reader's ring in chunks of 8 (bf16) or 4 (fp32) rows next
    to 4-row chunks of the 2-bit cells; outputs, row maxima and sums against the oracle through
    appends and flushes."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("sw1p", 2, 2, 4, D, 3, [20, 32 + 64 + 9, 700], dtype, modes, 0.0, append_steps=40, seed=37)
    m = Model(w, sink=32, window=64)
    m.ingest()
    for step in range(40):
        m.append_step(step)
        if step in (0, 17, 33, 39):
            for la in range(2):
                for lp in range(2):
                    m.check_cell(lp, la, _q(w, step, la, lp), where=f"1p sink/window step {step}")
    m.cache.check("single-pass sink/window")


def test_sink_window_ouro_shape():
    """The paper's geometry (32-token sink, 256-token window) at Ouro-1.4B head shape, 8K
    context, sampled rows of a 4-bit, a share and a 2-bit cell, tau = 0.01."""
    w = synth.Workload("sinkwin_8k", 1, 4, 16, 128, 4, [8192, 8000, 5000, 300], torch.bfloat16, [0, 1, 2, 0], 0.01,
                       append_steps=40, seed=37)
    m = Model(w, sink=32, window=256)
    m.ingest()
    for s in range(40):
        m.append_step(s)
    rng = np.random.default_rng(3)
    for lp in range(4):
        rows = [(int(rng.integers(4)), int(rng.integers(16))) for _ in range(6)] + [(3, 15), (0, 0)]
        m.check_cell(lp, 0, _q(w, 40, 0, lp), rows=rows, where="sink/window 8K")
    m.check_bytes(0, 0, reqs=[0, 2], heads=[0, 9])


def _stream_expected(scores, m0, C, tau, n_hist):
    """The streaming refine set as the kernel reads a row (LOOPKV_TAU_STREAM): group g to CTA
    g mod C as its local group g // C, local group i to warp i mod 4 in increasing i; per warp,
    the oracle's streaming rule over its groups in that order, seeded with m0."""
    ng = n_hist // 32
    bits = np.zeros(n_hist, bool)
    for c in range(C):
        for wp in range(4):
            groups = [c + i * C for i in range(wp, (ng + C - 1) // C + 4, 4) if c + i * C < ng]
            if not groups:
                continue
            sub = np.concatenate([scores[32 * g:32 * g + 32] for g in groups])
            words = O.stream_refine(sub, list(range(len(groups))), m0, tau, running=True)
            for k, g in enumerate(groups):
                bits[32 * g:32 * g + 32] = bits_of(words[k:k + 1], 32)
    return bits


@pytest.mark.parametrize("tau", [0.05, 0.01])
def test_streaming_refine_rule(tau):
    """LOOPKV_TAU_STREAM (the paper's running maximum seeded with the sink maximum): the GPU's set
    equals the oracle's streaming rule in the order the kernel reads (ties within 1e-6 of tau
    aside), contains the exact set, and the output matches the oracle on the GPU's set."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]
    w = synth.Workload("stream", 2, 2, 4, 128, 4, [2000, 700, 130, 1500], torch.bfloat16, modes, tau, seed=41,
                       tau_mode=L.TAU_STREAM)
    m = Model(w, sink=32, window=64)
    m.ingest()
    C = m.plan.decode_shape(w.B)["cluster"]
    for lp, la in [(0, 0), (0, 1), (1, 1)]:  # 4-bit cells and the share cell of a 4-bit source
        assert BITS[w.modes[m.src(lp, la)]] == 4
        if True:
            q = _q(w, 0, la, lp)
            out, bm, _, _ = m.cache.decode_debug(lp, la, q)
            m.cache.check("stream decode")
            out, bm, qn = f32(out), bm.cpu().numpy().view(np.uint32), f32(q)
            hist, near = m.cache.lengths(lp, la)
            c, src = m.cell(lp, la), m.src(lp, la)
            for req in range(w.B):
                n_hist, n_near = int(hist[req]), int(near[req])
                K, V = m.tokens[(c, req)]
                Kr, Vr = m.raw_tokens(K, V, n_hist, n_near)
                for h in range(w.H):
                    qq = qn[req, h].astype(np.float64)
                    hh = m.head_history(src, req, h, n_hist)
                    got = bits_of(bm[req, h], n_hist)
                    if n_hist == 0:
                        continue
                    g = np.arange(n_hist) // 32
                    kq = O.f16_bits_to_f64(hh.kz)[g] + O.f16_bits_to_f64(hh.ks)[g] * hh.kc.astype(np.float64)
                    s = kq @ qq / np.sqrt(w.D)
                    m0 = float((Kr[:32, h].astype(np.float64) @ qq).max() / np.sqrt(w.D))
                    want = _stream_expected(s, m0, C, tau, n_hist)
                    exact = O.decode_row(qq, hh, Kr[:, h], Vr[:, h], tau)
                    ex_bits = bits_of(exact["s_bits"], n_hist)
                    assert not (ex_bits & ~got).any(), "streaming set must contain the exact set"
                    diff = np.flatnonzero(want != got)
                    if diff.size:  # only ties: recompute the running maximum each differing token saw
                        run = np.full(n_hist, -np.inf)
                        for c2 in range(C):
                            for wp in range(4):
                                mr = m0
                                for i in range(wp, n_hist // 32, 4):
                                    gg = c2 + i * C
                                    if gg >= n_hist // 32:
                                        break
                                    mr = max(mr, s[32 * gg:32 * gg + 32].max())
                                    run[32 * gg:32 * gg + 32] = mr
                        far = diff[np.abs(np.exp(s[diff] - run[diff]) - tau) > 1e-6]
                        assert far.size == 0, f"streaming set differs at {far[:8]}"
                    ref = O.decode_row(qq, hh, Kr[:, h], Vr[:, h], tau, s_force=words_from_bits(got))
                    assert np.abs(out[req, h] - ref["o"]).max() <= 2e-3


def _exact_scores(K, q):
    """Oracle quantization of keys K [T, D] and the exact scores (natural log) of query q."""
    hh = O.HeadHistory(K, np.zeros_like(K), 4)
    g = np.arange(K.shape[0]) // 32
    kq = O.f16_bits_to_f64(hh.kz)[g] + O.f16_bits_to_f64(hh.ks)[g] * hh.kc.astype(np.float64)
    return kq @ q / np.sqrt(K.shape[1])


def _threshold_row(rng, d_rel, tau_target, D=128, T=256):
    """Keys of one row with a cluster of tokens whose scores are spaced by about d_rel (natural
    log) around m + ln(tau_target), m the row maximum: group 3 holds 32 copies of one key except
    channel c*, which steps through 16 codes; every other channel of that group is constant
    (scale 0).  The other groups are random keys with wide (lognormal, sigma 1.5) channel
    scales, so that the fixed-point factors of those groups are coarse and the row maximum lies
    there.  Returns bf16 keys [T, D] and query [D] as float32 arrays of bf16 values."""
    bf = lambda x: torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).float().numpy()  # noqa: E731
    sc = np.exp(1.5 * rng.standard_normal(D))
    k = rng.standard_normal((T, D)) * sc
    cstar = 5
    u = rng.standard_normal(D) * sc
    u[cstar] = 0.0
    q = rng.standard_normal(D)
    q[cstar] = d_rel * np.sqrt(D)  # one code step (scale ~0.5 below) moves the score by ~d_rel / 2
    q = bf(q)

    def build(alpha):
        kk = k.copy()
        kk[96:128] = alpha * u
        kk[96:128, cstar] = 1.0 + np.arange(32) * 0.5
        return bf(kk)

    s = _exact_scores(build(1.0), q)
    m = np.delete(s, np.arange(96, 128)).max()
    s0 = _exact_scores(build(0.0), q)[96:128].mean()  # the cluster's score without the base key
    alpha = (m + np.log(tau_target) - s0) / ((s[96:128].mean() - s0))
    return build(alpha), q


@pytest.mark.parametrize("d_rel", [1e-5, 1e-4, 1e-3])
@pytest.mark.parametrize("tau_target", [0.01, 0.3])
def test_refine_set_exact_near_threshold(d_rel, tau_target):
    """Tokens placed at r = tau * exp(j * d), around the threshold, with wide channel scales: the
    decide path's refine set may differ from the oracle's only within 1e-6 of tau."""
    rng = np.random.default_rng(int(d_rel * 1e7) + int(tau_target * 100))
    K, qv = _threshold_row(rng, d_rel, tau_target)
    s = _exact_scores(K, qv.astype(np.float64))
    m = s.max()
    assert s[96:128].max() < m  # the row maximum lies in another group
    mid = np.sort(np.unique(s[96:128]))
    tau = float(np.exp(mid[len(mid) // 2] - m))  # a cluster token exactly at the threshold
    assert 0.3 * tau_target < tau < 3 * tau_target
    V = torch.randn((256, 128), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    k = torch.tensor(K).to(torch.bfloat16)
    q = torch.tensor(qv).to(torch.bfloat16)
    plan = _plan(1, 1, 1, 128, 1, 32, [L.CELL_4B], tau)
    cache = L.Cache(plan)
    cache.ingest(0, 0, 0, k.view(256, 1, 128).contiguous().cuda(), V.view(256, 1, 128).contiguous().cuda())
    out, bm, _, _ = cache.decode_debug(0, 0, q.view(1, 1, 128).contiguous().cuda())
    cache.check("near-threshold decode")
    got = bits_of(bm.cpu().numpy().view(np.uint32)[0, 0], 256)
    hh = O.HeadHistory(K, V.float().numpy(), 4)
    res = O.decode_row(qv.astype(np.float64), hh, np.zeros((0, 128)), np.zeros((0, 128)), tau)
    want = bits_of(res["s_bits"], 256)
    r = res["r"][:256]
    assert (np.abs(r[96:128] / tau - 1) < 20 * d_rel).sum() >= 8  # many tokens close to the threshold
    diff = np.flatnonzero(got != want)
    assert np.all(np.abs(r[diff] - tau) <= 1e-6), (diff, r[diff] / tau - 1)




@pytest.mark.parametrize("win", [40, 100, 333, 5000])
@pytest.mark.parametrize("tau", [0.02, 0.0])
@pytest.mark.parametrize("sink,window", [(32, 64), (0, 0)])
def test_sliding_window_layer(win, tau, sink, window):
    """A layer whose cells attend only to their last `win` positions (Dory's sliding-window
    layers, LoopKV §2.1) next to a full-attention layer: windows that start inside a history
    group, inside the near region, and beyond the sequence; both readers (tau > 0 and tau = 0)."""
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # loop 0: [4b, share], loop 1: [2b, 4b]
    w = synth.Workload("slide", 2, 2, 4, 128, 3, [20, 150, 700], torch.bfloat16, modes, tau, append_steps=40, seed=43)
    m = Model(w, sink=sink, window=window)
    m.plan.set_window(1, win)
    m.ingest()
    for step in range(40):
        m.append_step(step)
        if step in (0, 13, 39):
            for la in range(2):
                for lp in range(2):
                    m.check_cell(lp, la, _q(w, step, la, lp), where=f"win={win} step {step}")
    m.cache.check("sliding window")
