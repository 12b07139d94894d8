#!/usr/bin/env python
"""Throughput of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over one synthetic sequence (CSA:
compress KV, compress indexer keys, indexer scores, top-k, sparse attention;
HCA: compress, dense attention; decode: indexer, top-k, sparse and HCA
attention over a batch of long caches). With N GPUs (one process per GPU,
launched by torchrun) every rank runs its own sequence: the units are
independent, so there is no data-path collective and scaling is weak.

Printed by rank 0: one JSON line (see the keys below). ``value`` is tokens/s
(prefill) or queries/s (decode) over all ranks, from CUDA-event time with
inputs resident in HBM and L2 flushed between steps; ``e2e`` is the same
metric with the step's inputs copied from pinned host memory and its output
read back inside the timed region; ``roofline`` describes the dominant kernel;
``cpu_baseline`` is the float64 CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import datetime
import json
import hashlib
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_07_b200 import workloads as W  # noqa: E402
from long_context_sparse_07_b200 import work  # noqa: E402

METRIC = "CSA/HCA tokens/s (prefill), queries/s (decode) and % of roofline on 1 B200"
DEFAULT_WORKLOAD = "csa_bf16_n4096"
L2_FLUSH_BYTES = 512 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index = period, index
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------------- our arm


def rank_workload(w, rank):
    """The workload of one rank: every rank runs its own independent sequence
    (same shapes, seed + 1000 * rank), so no data crosses ranks."""
    return W.scaled(w, seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(x, dist, device):
    """x reduced with max over the ranks of `dist` (the value itself without it)."""
    t = torch.tensor([x], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(local_ms, units_per_rank, world, dist, device):
    """Whole-job throughput: the units of all ranks over the slowest rank's
    mean step time. Returns (rate per second, that time in ms)."""
    ms = max_over_ranks(local_ms, dist, device)
    return units_per_rank * world / (ms * 1e-3), ms


def build_path(w, rank):
    from long_context_sparse_07_b200 import path
    wr = rank_workload(w, rank)
    if w.kind == "csa":
        return path.CsaPrefill(wr, W.csa_operands(wr))
    if w.kind == "hca":
        return path.HcaPrefill(wr, W.hca_operands(wr))
    return path.Decode(wr, W.decode_operands(wr))


def units_per_step(w):
    return w.batch if w.kind == "decode" else w.n


def algorithmic(w, p):
    if w.kind == "csa":
        return work.csa_prefill(w)
    if w.kind == "hca":
        return work.hca_prefill(w)
    return work.decode(w, p.E, p.E_hca)


# DRAM bytes (read + write) per launch of the dominant kernel from one ncu capture
# (summarised under profiles/), keyed by workload and kernel; each entry holds the
# SHA-1 of the kernel source it was taken on and counts only while that source is
# unchanged.
MEASURED_TRAFFIC = {
    ("csa_bf16_n4096", "attend"): ("attend_tc.cu", "7eeca1bf5e32ae25532dfa810103adaea4c2bcfc",
                                   143.875840e6 + 95.943936e6),
}


def measured_traffic(workload, kernel):
    ent = MEASURED_TRAFFIC.get((workload, kernel))
    if ent is None:
        return None
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "long_context_sparse_07_b200",
                       "csrc", ent[0])
    try:
        with open(src, "rb") as f:
            digest = hashlib.sha1(f.read()).hexdigest()
    except OSError:
        return None
    return ent[2] if digest == ent[1] else None


def time_steps(p, steps, flush, stream):
    """Device time of each step and of each kernel, L2 flushed in between."""
    names = [n for n, _ in p.phases()]
    per_kernel = {n: [] for n in names}
    per_step = []
    for _ in range(steps):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        evs[0].record(stream)
        for i, (_, f) in enumerate(p.phases()):
            f(stream)
            evs[i + 1].record(stream)
        per_step.append(evs)
    torch.cuda.synchronize()
    out = []
    for evs in per_step:
        out.append(evs[0].elapsed_time(evs[-1]))
        for i, n in enumerate(names):
            per_kernel[n].append(evs[i].elapsed_time(evs[i + 1]))
    return out, per_kernel


def time_steps_graph(p, steps, flush, stream):
    """time_steps with the step captured once in a CUDA graph and replayed:
    the graph launches every kernel of the step, so kernels of a few
    microseconds are timed without host launch gaps between them."""
    names = [n for n, _ in p.phases()]
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)]
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        evs[0].record()
        for i, (_, f) in enumerate(p.phases()):
            f(None)
            evs[i + 1].record()
    torch.cuda.synchronize()
    per_kernel = {n: [] for n in names}
    out = []
    for _ in range(steps):
        flush.zero_()
        g.replay()
        torch.cuda.synchronize()
        out.append(evs[0].elapsed_time(evs[-1]))
        for i, n in enumerate(names):
            per_kernel[n].append(evs[i].elapsed_time(evs[i + 1]))
    del g
    return out, per_kernel


def time_e2e(p, steps, stream):
    """Same step with inputs copied from pinned host memory and the result
    read back, inside the timed region."""
    dev_in = p.inputs()
    host_in = {k: v.cpu().pin_memory() for k, v in dev_in.items()}
    res = p.result()
    host_out = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = res.numel() * res.element_size()
    times = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for k, v in host_in.items():
            dev_in[k].copy_(v, non_blocking=True)
        p.step(stream)
        host_out.copy_(res, non_blocking=True)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in times], h2d, d2h


def cpu_baseline(w, p_rows=None):
    """The oracle as it stands on a bounded sample, extrapolated linearly."""
    import oracle
    from oracle import pipeline
    cores = os.cpu_count()
    if w.kind == "decode":
        wd = W.scaled(w, batch=1)
        ops = W.decode_operands(wd)
        t0 = time.perf_counter()
        pipeline.decode(ops, wd)
        dt = time.perf_counter() - t0
        return {"value": 1.0 / dt, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": "1 of %d decode queries (full cache), scaled per query" % w.batch}
    ops = W.csa_operands(w) if w.kind == "csa" else W.hca_operands(w)
    rows = p_rows or 128
    sel = np.random.default_rng(0).choice(w.n, size=rows, replace=False)
    # compression is linear in tokens: time it on the first n/8 tokens
    ns = max(w.m, (w.n // 8) // w.m * w.m)
    t0 = time.perf_counter()
    if w.kind == "csa":
        oracle.compress(ops["Ca"][:ns], ops["Cb"][:ns], ops["Za"][:ns], ops["Zb"][:ns],
                        ops["Ba"], ops["Bb"], w.m, True)
        oracle.compress(ops["CIa"][:ns], ops["CIb"][:ns], ops["ZIa"][:ns], ops["ZIb"][:ns],
                        ops["BIa"], ops["BIb"], w.m, True)
    else:
        oracle.compress(ops["C"][:ns], None, ops["Z"][:ns], None, ops["B"], None, w.m, False)
    t_comp = (time.perf_counter() - t0) * (w.n / ns)
    fn = pipeline.csa_prefill if w.kind == "csa" else pipeline.hca_prefill
    t0 = time.perf_counter()
    fn(ops, w, sel)
    t_all = time.perf_counter() - t0
    # the pipeline call also compresses the whole sequence once: subtract it
    t_rows = max(t_all - t_comp, 1e-3)
    total = t_comp + t_rows * (w.n / rows)
    return {"value": w.n / total, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "compression on %d of %d tokens and %d of %d query rows, extrapolated "
                      "linearly" % (ns, w.n, rows, w.n)}


def run_ours(args, w):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    from long_context_sparse_07_b200 import abi
    abi.load()
    p = build_path(w, rank)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        p.step(stream)
    torch.cuda.synchronize()
    abi.csa_get_error()

    def barrier():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()

    barrier()
    graph = args.graph == "on" or (args.graph == "auto" and w.kind == "decode")
    with ClockSampler(local) as clk:
        if graph:
            step_ms, kern_ms = time_steps_graph(p, args.steps, flush, stream)
        else:
            step_ms, kern_ms = time_steps(p, args.steps, flush, stream)
    barrier()
    abi.csa_get_error()
    mean_ms = sum(step_ms) / len(step_ms)
    value, ms = job_rate(mean_ms, units_per_step(w), world, dist, "cuda")

    # end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, 20))
    p.step(stream)
    e_ms, h2d, d2h = time_e2e(p, e2e_steps, stream)
    e2e_value, _ = job_rate(sum(e_ms) / len(e_ms), units_per_step(w), world, dist, "cuda")

    # roofline of the dominant kernel
    pk = peaks()
    alg = algorithmic(w, p)
    kavg = {n: sum(v) / len(v) for n, v in kern_ms.items()}
    dom = max(kavg, key=kavg.get)
    a = alg[dom]
    if a["flops"] > 0 and a["flops"] / pk["bf16"] > a["bytes"] / (pk["hbm"] * 1e9 / 1e12):
        achieved = a["flops"] / (kavg[dom] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s"}
    else:
        achieved = a["bytes"] / (kavg[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(w.name, dom)
    roof["kernel"] = dom
    roof["peak_source"] = pk["source"]
    roof["kernel_ms"] = {n: round(v, 5) for n, v in kavg.items()}

    if rank == 0:
        unit = "queries/s" if w.kind == "decode" else "tokens/s"
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded generators; random-init projection outputs)",
            "config": {"workload": w.name, "n": w.n, "c": w.c, "m": w.m, "k": w.k,
                       "h": w.h, "hI": w.hI, "cI": w.cI, "n_win": w.n_win,
                       "indexer_dtype": w.idx_dtype, "batch_per_gpu": w.batch,
                       "l2": "flushed between timed steps (512 MiB write)",
                       "launch": "CUDA graph replay" if graph else "eager",
                       "parallelism": "dp%d (independent sequences)" % world},
            "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": p.launches_per_step * args.steps,
            "roofline": roof,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- reference arm


def run_reference(args, w):
    """The CPU oracle timed as the reference arm (bounded sample per step)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    from oracle import pipeline
    cores = os.cpu_count()
    total_steps = args.steps + args.warmup
    budget = 90.0 / max(total_steps, 1)          # seconds of CPU work per step
    if w.kind == "decode":
        raise SystemExit("reference arm: decode workload not wired")
    ops = W.csa_operands(w) if w.kind == "csa" else W.hca_operands(w)
    fn = pipeline.csa_prefill if w.kind == "csa" else pipeline.hca_prefill
    # calibrate: one row costs about this much (compression included once)
    g = np.random.default_rng(0)
    t0 = time.perf_counter()
    fn(ops, w, g.choice(w.n, size=8, replace=False))
    t_cal = time.perf_counter() - t0
    ns = max(w.m, min(w.n, int(w.n * min(1.0, budget / max(t_cal, 1e-3) / 4))) // w.m * w.m)
    rows = 4
    times = []
    for i in range(total_steps):
        sel = g.choice(w.n, size=rows, replace=False)
        t0 = time.perf_counter()
        if w.kind == "csa":
            oracle.compress(ops["Ca"][:ns], ops["Cb"][:ns], ops["Za"][:ns], ops["Zb"][:ns],
                            ops["Ba"], ops["Bb"], w.m, True)
        else:
            oracle.compress(ops["C"][:ns], None, ops["Z"][:ns], None, ops["B"], None, w.m,
                            False)
        t1 = time.perf_counter()
        fn(ops, w, sel)
        t2 = time.perf_counter()
        if i >= args.warmup:
            t_comp = (t1 - t0) * w.n / ns
            t_rows = max((t2 - t1) - t_comp, 1e-4) * w.n / rows
            times.append(t_comp + t_rows)
    ms = 1e3 * sum(times) / len(times)
    value = w.n / (ms * 1e-3)
    unit = "tokens/s"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded generators)",
            "config": {"workload": w.name, "n": w.n, "c": w.c, "m": w.m, "k": w.k,
                       "h": w.h},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": "per step: compression on %d of %d tokens and %d query "
                                       "rows, extrapolated linearly" % (ns, w.n, rows)},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--n", type=int, default=None,
                    help="run the workload on a shorter sequence of n tokens (small profiling cases)")
    ap.add_argument("--graph", default="auto", choices=["auto", "on", "off"],
                    help="replay the timed step from a CUDA graph (auto: decode only)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = W.WORKLOADS[args.workload]
    if args.n is not None:
        # a shorter sequence of the same workload (profiling captures), named as such
        if args.n % w.m or args.n <= 0:
            sys.exit("--n must be a positive multiple of m = %d" % w.m)
        w = W.scaled(w, n=args.n, name="%s@n%d" % (w.name, args.n))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
