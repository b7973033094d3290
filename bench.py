"""Benchmark of the LoopKV decode hot path on B200: fused loop-aware decode attention.

One step = one decode step of the whole looped model's attention: for every (loop, layer)
cell in model order, [append this step's token when the workload appends, after a flush of
full tails at the start of the step] and one fused decode launch, replayed as one CUDA
graph (the pages replay a whole decode step as one graph).  Inputs are resident in HBM;
the per-step KV working set (16 GB and up) is far larger than L2, so no flush is needed.

Prints one JSON line.  `value` = algorithmic KV bytes read per step / step time (GB/s) of the
headline workload (default long_16k, the largest single-GPU configuration, with appends);
`e2e` = the same through the public API with the step's inputs (queries, and the new keys and
values of an appending workload) copied from pinned host memory and the outputs copied back
inside the timed region, every step; the copies run on their own streams into and out of two
buffer sets (one graph per set), so that step i + 1's inputs and step i - 1's outputs move while
step i computes, as a serving loop would; `workloads` = the other workloads measured the same
way (device time only).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config long_16k] [--workloads kivi4_8k,mixed_8k]
                  [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from mixed_precision_kv_append_b200 import synth  # noqa: E402

METRIC = "fused loop-aware decode attention: KV GB/s (% of HBM peak) and decode steps/s"


def _code_digest(paths) -> str:
    """sha256 of source files with comments and blank lines removed: an edit of comments
    leaves the compiled kernels, and so the counters taken from them, unchanged."""
    import hashlib
    import re

    h = hashlib.sha256()
    for p in paths:
        text = open(p, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("\n".join(line.rstrip() for line in text.splitlines() if line.strip()).encode())
    return h.hexdigest()


def _profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary of this workload, if the
    decode kernel code is unchanged since the capture (else None)."""
    import re

    path = os.path.join(ROOT, "profiles", f"decode_kernel_{workload}.md")
    csrc = os.path.join(ROOT, "mixed_precision_kv_append_b200", "csrc")
    try:
        text = open(path).read()
        traffic = int(re.search(r"traffic_bytes_per_launch: (\d+)", text).group(1))
        want = re.search(r"kernel_code_sha256: ([0-9a-f]+)", text).group(1)
        got = _code_digest([os.path.join(csrc, f) for f in ("decode_kernel.cu", "lkv_device.cuh")])
    except Exception:
        return None
    return traffic if got == want else None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = threading.Event()
        self._proc = None

    def __enter__(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self._proc = None
        return self

    def _read(self):
        for line in self._proc.stdout:
            self.samples.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self._proc:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in self.samples:
            for n, v in zip(names, s[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.samples)}


def max_over_ranks(values, device=None):
    """Element-wise maximum over all ranks of per-rank timings (identity without a process group).
    Every rank must call it at the same point; the tensor lives on `device` (CUDA for NCCL, CPU for gloo)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ----------------------------------------------------------------------------- workload

class Runner:
    """Builds the cache of one workload on this GPU and captures one decode step as a graph."""

    def __init__(self, w: synth.Workload, device):
        from mixed_precision_kv_append_b200 import loopkv as L

        self.L = L
        self.w = w
        self.dev = device
        self.plan = L.Plan(w.n_layers, w.n_loops, w.H, w.D, w.B, w.max_blocks, w.modes, w.tau, w.tau_mode,
                           w.dtype, w.sink, w.window)
        for layer, win in w.layer_windows.items():  # sliding-window layers
            self.plan.set_window(layer, win)
        self.cache = L.Cache(self.plan, device=device)
        for layer in range(w.n_layers):
            for req in range(w.B):
                ks, vs = synth.layer_history(w, layer, req, device=device)
                for lp in range(w.n_loops):
                    self.cache.ingest(lp, layer, req, ks[lp], vs[lp])
                del ks, vs
        self.cache.check("ingest")
        n = w.n_cells
        # queries of every cell (fixed over steps), new tokens of the appending workloads
        self.q = torch.empty((n, w.B, w.H, w.D), dtype=w.dtype, device=device)
        self.knew = torch.empty_like(self.q)
        self.vnew = torch.empty_like(self.q)
        for layer in range(w.n_layers):
            qs, ks, vs = synth.step_tokens(w, 0, layer, device=device)
            for lp in range(w.n_loops):
                c = lp * w.n_layers + layer
                self.q[c], self.knew[c], self.vnew[c] = qs[lp], ks[lp], vs[lp]
        self.out = torch.empty((n, w.B, w.H, w.D), dtype=torch.float32, device=device)
        self.order = [(lp, layer) for lp in range(w.n_loops) for layer in range(w.n_layers)]  # model order
        self.stream = torch.cuda.Stream(device=device)
        self.launches_per_step = len(self.order) * (2 if w.append_steps else 1) + (1 if w.append_steps else 0)

    def _step(self, s, bufs=None):
        L, w = self.L, self.w
        q, knew, vnew, out = bufs or (self.q, self.knew, self.vnew, self.out)
        if w.append_steps:
            self.cache.flush(stream=s)
        for lp, layer in self.order:
            c = lp * w.n_layers + layer
            if w.append_steps:
                self.cache.append(lp, layer, knew[c], vnew[c], stream=s)
            L.loopkv_decode(self.plan.handle, lp, layer, q[c], self.cache.handle, out[c], stream=s)

    def capture_second_set(self):
        """A second set of input and output buffers and the step graph on it (end-to-end timing
        alternates the two sets, so that copies of one overlap the compute of the other)."""
        self.bufs2 = (self.q.clone(), self.knew.clone(), self.vnew.clone(), torch.empty_like(self.out))
        self.graph2 = torch.cuda.CUDAGraph()
        s = self.stream
        with torch.cuda.stream(s):
            with torch.cuda.graph(self.graph2, stream=s):
                self._step(s, self.bufs2)
        s.synchronize()

    def capture(self):
        s = self.stream
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            self._step(s)  # sets the launch attributes outside the capture
        s.synchronize()
        if self.w.append_steps:  # undo the eager step: not needed for timing, lengths only grow by one
            pass
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(self.graph, stream=s):
                self._step(s)
        s.synchronize()

    def hot_fraction_and_bytes(self):
        """Algorithmic bytes read by one step, from the refine sets of one debug pass."""
        L, w = self.L, self.w
        D, H, esz = w.D, w.H, (2 if w.dtype == torch.bfloat16 else 4)
        total = 0.0
        hot_tokens = all_tokens = 0
        with torch.cuda.stream(self.stream):
            for lp, layer in self.order:
                c = lp * w.n_layers + layer
                _, bm, _, _ = self.cache.decode_debug(lp, layer, self.q[c], stream=self.stream)
                self.stream.synchronize()
                hist, tail = self.cache.lengths(lp, layer)
                v = self.cache.cell_view(lp, layer)
                per_tok = v.head_main_bytes / 16.0
                win = w.layer_windows.get(layer, 0)
                # history tokens read: all, or those inside a sliding window (from its first group)
                nh = sum(int(hist[r]) - (min(max(int(hist[r]) + int(tail[r]) - win, 0), int(hist[r])) // 32) * 32
                         if win else int(hist[r]) for r in range(w.B))
                hot = 0
                if v.head_lo_bytes:
                    bits = bm.view(torch.int32).cpu()
                    hot = int(sum(bin(x & 0xFFFFFFFF).count("1") for x in bits.flatten().tolist()))
                    hot_tokens += hot
                    all_tokens += nh * H
                total += H * nh * per_tok + hot * (v.head_lo_bytes / 16.0)
                total += int(tail[: w.B].sum()) * H * D * esz * 2
                total += w.B * H * D * (esz + 4)  # q in, out
        self.cache.check("debug pass")
        return total, (hot_tokens / all_tokens if all_tokens else 0.0)


def _time_graph(runner: Runner, steps: int):
    """Device time of `steps` graph replays on the runner's stream (CUDA events on that stream)."""
    s = runner.stream
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for _ in range(steps):
            runner.graph.replay()
        ev1.record(s)
    ev1.synchronize()
    return ev0.elapsed_time(ev1) / 1e3  # seconds


def _time_e2e(runner: Runner, steps: int, host):
    """Device time of `steps` end-to-end steps, from the first input copy to the last output copy.
    Step i uses buffer set i % 2: its inputs are copied from pinned host memory on a copy stream,
    its graph runs on the compute stream, and all its outputs are copied back to pinned host
    memory on a third stream.  A set is refilled only after the graph that read it finished, and
    a graph writes a set's outputs only after their previous copy-back finished."""
    s = runner.stream
    cin, cout = runner.copy_in, runner.copy_out
    graphs = (runner.graph, runner.graph2)
    outs = (runner.out, runner.bufs2[3])
    done_in = [torch.cuda.Event() for _ in range(2)]
    done_comp = [torch.cuda.Event() for _ in range(2)]
    done_out = [torch.cuda.Event() for _ in range(2)]
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(cin)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(cin):
            if i >= 2:
                cin.wait_event(done_comp[b])
            for dev_t, host_t in host["in"][b]:
                dev_t.copy_(host_t, non_blocking=True)
            done_in[b].record(cin)
        with torch.cuda.stream(s):
            s.wait_event(done_in[b])
            if i >= 2:
                s.wait_event(done_out[b])
            graphs[b].replay()
            done_comp[b].record(s)
        with torch.cuda.stream(cout):
            cout.wait_event(done_comp[b])
            host["out"][b].copy_(outs[b], non_blocking=True)
            done_out[b].record(cout)
    s.wait_event(done_out[(steps - 1) % 2])
    ev1.record(s)
    ev1.synchronize()
    return ev0.elapsed_time(ev1) / 1e3  # seconds


def _workload(name, args):
    w = synth.workload(name, seed=args.seed)
    if w.append_steps:  # room for every appended token of this run (warm-up, timing, e2e, setup)
        w.append_steps = max(w.append_steps, 2 * (args.steps + args.warmup) + 8)
    if args.layers and args.layers < w.n_layers:
        n = args.layers
        w.modes = [w.modes[lp * w.n_layers + la] for lp in range(w.n_loops) for la in range(n)]
        w.n_layers = n
        w.layer_windows = {la: win for la, win in w.layer_windows.items() if la < n}
        w.name = f"{w.name}[{n} layer{'s' if n > 1 else ''}]"
    return w


def measure(w, args, rank, world, device, e2e: bool):
    """One workload: build the cache, capture a step, time it.  Returns (result dict, runner)."""
    runner = Runner(w, device)
    algo_bytes, hot = runner.hot_fraction_and_bytes()
    runner.capture()
    for _ in range(args.warmup):
        runner.graph.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t = _time_graph(runner, args.steps)
    torch.cuda.synchronize(device)
    t_e2e, h2d = None, 0
    if e2e:
        runner.capture_second_set()
        runner.copy_in = torch.cuda.Stream(device=device)
        runner.copy_out = torch.cuda.Stream(device=device)
        host = {"in": [[], []], "out": [torch.empty(runner.out.shape, dtype=torch.float32, pin_memory=True)
                                        for _ in range(2)]}
        for b, (q, knew, vnew, _) in enumerate([(runner.q, runner.knew, runner.vnew, None), runner.bufs2]):
            for dev_t in [q] + ([knew, vnew] if w.append_steps else []):
                h = torch.empty(dev_t.shape, dtype=dev_t.dtype, pin_memory=True)
                h.copy_(dev_t)
                host["in"][b].append((dev_t, h))
                if b == 0:
                    h2d += dev_t.numel() * dev_t.element_size()
        for _ in range(2):
            runner.graph.replay()
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
        t_e2e = _time_e2e(runner, args.steps, host)
    runner.cache.check("timed steps")
    t, t_e2e = max_over_ranks([t, t_e2e if t_e2e is not None else 0.0], device)
    peak, peak_kind = _peaks()
    ms = t / args.steps * 1e3
    gbs = algo_bytes * world * args.steps / t / 1e9
    # per decode launch: algorithmic bytes of one launch / (step time / decode launches); the
    # step's flush and append launches are counted in the time, so this is a lower bound
    n_decode = len(runner.order)
    achieved = (algo_bytes / n_decode) / (t / args.steps / n_decode) / 1e9
    shape = runner.plan.decode_shape(w.B)
    res = {
        "value": round(gbs, 2), "ms_per_step": round(ms, 4), "steps_per_s": round(1e3 / ms, 2),
        "pct_hbm_peak": round(100.0 * gbs / world / peak, 2), "hot_fraction": round(hot, 4),
        "frac": round(achieved / peak, 4), "traffic": _profiled_traffic(w.name) if not args.layers else None,
        "algorithmic_bytes_per_step": int(algo_bytes), "cluster": shape["cluster"], "ctas_per_launch": shape["ctas"],
        "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "clocks": clk.summary(),
        "launches_per_step": runner.launches_per_step,
    }
    if e2e:
        res["e2e"] = {"value": round(algo_bytes * world * args.steps / t_e2e / 1e9, 2), "unit": "GB/s",
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(runner.out.numel() * 4),
                      "ms_per_step": round(t_e2e / args.steps * 1e3, 4),
                      "copies": "every step's inputs in and outputs out, on their own streams, double-buffered, "
                                "overlapping the neighbouring steps' compute"}
    return res, runner


def run_ours(args, rank, world, device):
    w = _workload(args.config, args)
    head, runner = measure(w, args, rank, world, device, e2e=True)
    algo_bytes = head["algorithmic_bytes_per_step"]
    del runner
    torch.cuda.empty_cache()
    result = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "steps_per_s": head["steps_per_s"],
        "pct_hbm_peak": head["pct_hbm_peak"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in, 4/2-bit KV codes, fp32 accumulate" if w.dtype == torch.bfloat16 else "fp32",
        "data": "synthetic (seeded Ouro-shaped Q/K/V, lognormal key channel scales, loop correlation 0.85)",
        "config": {"workload": w.name, "layers": w.n_layers, "loops": w.n_loops, "heads": w.H, "head_dim": w.D,
                   "batch_per_gpu": w.B, "global_batch": w.B * world, "context": max(w.lengths),
                   "tau": w.tau, "cells_4b_2b_share": [w.modes.count(0), w.modes.count(1), w.modes.count(2)],
                   "append": bool(w.append_steps), "hot_fraction": head["hot_fraction"],
                   "algorithmic_bytes_per_step": algo_bytes, "cluster": head["cluster"],
                   "ctas_per_launch": head["ctas_per_launch"],
                   "l2": "per-step working set >> 126 MB L2 (no flush needed)",
                   "parallelism": f"dp{world} (request-sharded replicas)"},
        "e2e": head["e2e"],
        "roofline": {"bound": "hbm", "achieved": head["achieved"], "peak": head["peak"], "unit": "GB/s",
                     "frac": head["frac"], "traffic": head["traffic"],
                     "peak_source": f"{head['peak_kind']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "gpu_launches": head["launches_per_step"] * args.steps * 2,
        "clocks": head["clocks"],
    }
    if args.workloads:
        result["workloads"] = {}
        for name in [n for n in args.workloads.split(",") if n and n != args.config]:
            wl, r = measure(_workload(name, args), args, rank, world, device, e2e=False)
            del r
            torch.cuda.empty_cache()
            result["workloads"][name] = {k: wl[k] for k in ("value", "ms_per_step", "steps_per_s", "hot_fraction",
                                                            "frac", "traffic", "algorithmic_bytes_per_step",
                                                            "cluster", "ctas_per_launch", "clocks")}
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, algo_bytes, budget_s=args.cpu_seconds)
    return result


# ------------------------------------------------------------------- CPU oracle timing

def _cpu_rows(w: synth.Workload, n_rows: int):
    """Rows (request, head) of the workload at its context for the CPU oracle, drawn from the
    cells of layer 0 in loop order: (query, quantized history of the cell read, bytes the GPU
    path counts for the row).  Share cells read the final loop's history."""
    import numpy as np

    from oracle import oracle as O

    rows = []
    req = 0
    T = w.lengths[req] // 32 * 32
    ks, vs = synth.layer_history(w, 0, req, T=T, device="cpu")
    qs, _, _ = synth.step_tokens(w, 0, 0, device="cpu")
    cells = list(range(w.n_loops))
    hists = {}
    h = 0
    while len(rows) < n_rows:
        lp = cells[(len(rows) // w.H) % len(cells)]
        mode = w.modes[lp * w.n_layers]
        src = w.n_loops - 1 if mode == synth.CELL_SHARE else lp
        bits = 4 if w.modes[src * w.n_layers] == synth.CELL_4B else 2
        if (src, h % w.H) not in hists:
            hists[(src, h % w.H)] = O.HeadHistory(ks[src][:, h % w.H].float().numpy(),
                                                  vs[src][:, h % w.H].float().numpy(), bits)
        hh = hists[(src, h % w.H)]
        per_tok = (128.0 if bits == 4 else 96.0) * (w.D / 128.0)  # + lo bytes of hot tokens, added below
        rows.append((qs[lp][req, h % w.H].float().numpy().astype(np.float64), hh, per_tok, bits))
        h += 1
    return rows


def _time_oracle(w, rows, threads: int):
    """Decode the rows with the oracle on `threads` host threads (the oracle is C; its calls
    run in parallel).  Returns (seconds, algorithmic bytes of the rows)."""
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor

    from oracle import oracle as O

    empty = np.zeros((0, w.D))

    def one(r):
        q, hh, per_tok, bits = r
        res = O.decode_row(q, hh, empty, empty, w.tau, w.tau_mode)
        hot = int(sum(bin(int(x)).count("1") for x in res["s_bits"])) if bits == 4 else 0
        return hh.T * per_tok + hot * (w.D / 4.0)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        nbytes = sum(ex.map(one, rows))
    return time.perf_counter() - t0, nbytes


def cpu_baseline(w: synth.Workload, step_bytes: float, budget_s: float = 15.0):
    """The CPU oracle's decode on the host cores, on a bounded sample of the workload's rows,
    in the benchmark's unit; steps/s extrapolated linearly in bytes to a whole step."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    probe = _cpu_rows(w, cores)
    t1, _ = _time_oracle(w, probe, cores)  # one row per thread: sizes the sample to the budget
    n = max(cores, int(budget_s / max(t1, 1e-3)) * cores)
    rows = _cpu_rows(w, n)
    secs, nbytes = _time_oracle(w, rows, cores)
    gbs = nbytes / secs / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "extrapolated_steps_per_s": round(nbytes / secs / step_bytes, 6),
            "sample": f"{n} rows (request 0, every head) of the layer-0 cells in loop order at {w.lengths[0] // 32 * 32} "
                      f"tokens, decode only, fp64 oracle on {cores} host threads, {secs:.1f} s; bytes counted as "
                      f"the GPU path's algorithmic bytes; steps/s extrapolated linearly in bytes"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: K steps of a bounded sample on the host cores."""
    w = _workload(args.config, args)
    if rank != 0:
        return None
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    rows = _cpu_rows(w, cores)
    for _ in range(args.warmup):
        _time_oracle(w, rows[:1], 1)
    secs = nbytes = 0.0
    for _ in range(args.steps):
        t, b = _time_oracle(w, rows, cores)
        secs += t
        nbytes += b
    value = nbytes / secs / 1e9
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Ouro-shaped Q/K/V)",
        "config": {"workload": w.name, "context": max(w.lengths), "tau": w.tau},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {len(rows)} rows (request 0, every head) of the layer-0 cells, "
                                   f"decode only, on {cores} host threads"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="long_16k", choices=synth.WORKLOADS[1:])
    ap.add_argument("--workloads", default="kivi4_8k,mixed_8k",
                    help="further workloads measured after the headline one and reported under 'workloads' "
                         "(comma-separated; empty for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="keep only the first N layers (small profiling cases)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    from datetime import timedelta

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    from mixed_precision_kv_append_b200 import build as B

    if rank == 0 or world == 1:
        B.build()
    if world > 1:
        dist.barrier()
    res = run_ours(args, rank, world, device)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
