"""Benchmark of the LoopKV decode hot path on B200: fused loop-aware decode attention.

One step = one decode step of the whole looped model's attention: for every (loop, layer)
cell in model order, [append this step's token when the workload appends, after a flush of
full tails at the start of the step] and one fused decode launch, replayed as one CUDA
graph (the pages replay a whole decode step as one graph).  Inputs are resident in HBM;
the per-step KV working set (16 GB and up) is far larger than L2, so no flush is needed.

Prints one JSON line.  `value` = algorithmic KV bytes read per step / step time (GB/s);
`e2e` = the same through the public API with the step's queries copied from pinned host
memory and the outputs copied back inside the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config kivi4_8k] [--impl ours|reference]
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
                           w.dtype)
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

    def _step(self, s):
        L, w = self.L, self.w
        if w.append_steps:
            self.cache.flush(stream=s)
        for lp, layer in self.order:
            c = lp * w.n_layers + layer
            if w.append_steps:
                self.cache.append(lp, layer, self.knew[c], self.vnew[c], stream=s)
            L.loopkv_decode(self.plan.handle, lp, layer, self.q[c], self.cache.handle, self.out[c], stream=s)

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
                nh = int(hist[: w.B].sum())
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


def _time_graph(runner: Runner, steps: int, e2e: bool, host_q=None, host_out=None):
    s = runner.stream
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        ev0.record(s)
        for _ in range(steps):
            if e2e:
                runner.q.copy_(host_q, non_blocking=True)
            runner.graph.replay()
            if e2e:
                host_out.copy_(runner.out, non_blocking=True)
        ev1.record(s)
    ev1.synchronize()
    return ev0.elapsed_time(ev1) / 1e3  # seconds


def _workload(args):
    w = synth.workload(args.config, seed=args.seed)
    if args.layers and args.layers < w.n_layers:
        n = args.layers
        w.modes = [w.modes[lp * w.n_layers + la] for lp in range(w.n_loops) for la in range(n)]
        w.n_layers = n
        w.name = f"{w.name}[{n} layer{'s' if n > 1 else ''}]"
    return w


def run_ours(args, rank, world, device):
    w = _workload(args)
    runner = Runner(w, device)
    algo_bytes, hot = runner.hot_fraction_and_bytes()
    runner.capture()
    host_q = torch.empty(runner.q.shape, dtype=runner.q.dtype, pin_memory=True)
    host_q.copy_(runner.q)
    host_out = torch.empty(runner.out.shape, dtype=torch.float32, pin_memory=True)
    for _ in range(args.warmup):
        runner.graph.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t = _time_graph(runner, args.steps, False)
    torch.cuda.synchronize(device)
    for _ in range(2):
        runner.graph.replay()
    if world > 1:
        dist.barrier()
    t_e2e = _time_graph(runner, args.steps, True, host_q, host_out)
    runner.cache.check("timed steps")
    t, t_e2e = max_over_ranks([t, t_e2e], device)
    peak, peak_kind = _peaks()
    ms = t / args.steps * 1e3
    gbs = algo_bytes * world * args.steps / t / 1e9
    gbs_e2e = algo_bytes * world * args.steps / t_e2e / 1e9
    n_decode = len(runner.order)
    per_launch_s = t / args.steps / n_decode
    per_launch_bytes = algo_bytes / n_decode
    achieved = per_launch_bytes / per_launch_s / 1e9 if not w.append_steps else gbs / world
    shape = runner.plan.decode_shape(w.B)
    result = {
        "metric": METRIC,
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "steps_per_s": round(1e3 / ms, 2),
        "pct_hbm_peak": round(100.0 * gbs / world / peak, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in, 4/2-bit KV codes, fp32 accumulate" if w.dtype == torch.bfloat16 else "fp32",
        "data": "synthetic (seeded Ouro-shaped Q/K/V, lognormal key channel scales, loop correlation 0.85)",
        "config": {"workload": w.name, "layers": w.n_layers, "loops": w.n_loops, "heads": w.H, "head_dim": w.D,
                   "batch_per_gpu": w.B, "global_batch": w.B * world, "context": max(w.lengths),
                   "tau": w.tau, "cells_4b_2b_share": [w.modes.count(0), w.modes.count(1), w.modes.count(2)],
                   "append": bool(w.append_steps), "hot_fraction": round(hot, 4),
                   "algorithmic_bytes_per_step": int(algo_bytes), "cluster": shape["cluster"],
                   "ctas_per_launch": shape["ctas"], "l2": "per-step working set >> 126 MB L2 (no flush needed)",
                   "parallelism": f"dp{world} (request-sharded replicas)"},
        "e2e": {"value": round(gbs_e2e, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(runner.q.numel() * runner.q.element_size()),
                "d2h_bytes_per_step": int(runner.out.numel() * 4),
                "ms_per_step": round(t_e2e / args.steps * 1e3, 4)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": _profiled_traffic(w.name) if not args.layers else None,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "gpu_launches": runner.launches_per_step * args.steps * 2,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return result


# ------------------------------------------------------------------- CPU oracle timing

def cpu_baseline(w: synth.Workload, budget_s: float = 15.0, rows_max: int | None = None):
    """Time the CPU oracle's decode (single thread) on whole rows of cell (0, 0) at the
    workload's context, and express it in the benchmark's unit."""
    import numpy as np

    from oracle import oracle as O

    bits = 4 if w.modes[0] == 0 else 2
    T = w.lengths[0] // 32 * 32
    ks, vs = synth.layer_history(w, 0, 0, T=T, device="cpu")
    K, V = ks[0].float().numpy(), vs[0].float().numpy()
    qs, _, _ = synth.step_tokens(w, 0, 0, device="cpu")
    q = qs[0].float().numpy()
    per_tok = (160.0 if bits == 4 else 96.0) * (w.D / 128.0)
    rows, secs = 0, 0.0
    h = 0
    while (rows < rows_max) if rows_max is not None else (secs < budget_s):
        hist = O.HeadHistory(K[:, h % w.H], V[:, h % w.H], bits)
        t0 = time.perf_counter()
        O.decode_row(q[0, h % w.H].astype(np.float64), hist, np.zeros((0, w.D)), np.zeros((0, w.D)), w.tau,
                     w.tau_mode)
        secs += time.perf_counter() - t0
        rows += 1
        h += 1
    gbs = rows * T * per_tok / secs / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} rows (request, head) of cell (loop 1, layer 1) at {T} tokens, decode only, "
                      f"{secs:.1f} s single-threaded fp64; bytes counted as the GPU path's algorithmic bytes"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: K steps of a bounded sample on the host cores."""
    w = _workload(args)
    if rank != 0:
        return None
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=0.0, rows_max=1)
    t0 = time.perf_counter()
    vals = [cpu_baseline(w, budget_s=0.0, rows_max=2) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(wall / args.steps * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Ouro-shaped Q/K/V)",
        "config": {"workload": w.name, "context": max(w.lengths), "tau": w.tau},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: 2 rows (request, head) of cell (loop 1, layer 1), decode only"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="kivi4_8k", choices=synth.WORKLOADS[1:])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
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
