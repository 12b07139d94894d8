#!/usr/bin/env python
"""Throughput of the CSA / HCA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-per-workload] [--no-extras]
                    [--no-cpu-baseline] [--n N] [--graph auto|on|off]

One step = one pass of the whole path over one synthetic sequence (CSA:
compress KV, compress indexer keys, indexer scores and top-k in one call
(csa_indexer_topk, which does not write the score rows), sparse attention;
HCA: compress, dense attention; decode: indexer, top-k, sparse and HCA
attention over a batch of long caches). The default workload is the largest
prefill that fits one GPU: a 131072-token CSA prefill with an e4m3 indexer
(64 indexer heads, top-1024, 64 query heads). With N GPUs (one process per
GPU, launched by torchrun) every rank runs its own sequence: the units are
independent, so there is no data-path collective and scaling is weak.

Printed by rank 0: one JSON line. ``value`` is tokens/s (prefill) or
queries/s (decode) over all ranks, from CUDA-event time with inputs resident
in HBM and L2 flushed between steps; ``e2e`` is the same metric with the
step's inputs copied from pinned host memory and its output read back inside
the timed region; ``roofline`` describes the dominant kernel of the default
workload; ``per_workload`` times every workload of the suite in the same run
(step time, per-kernel times and roofline fractions, and for decode the HBM
fraction of the CSA step); ``cpu_baseline`` is the float64 CPU oracle on a
bounded sample, timed on inputs converted to float64 beforehand.

``--impl reference`` times that same oracle sample as the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
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
DEFAULT_WORKLOAD = "csa_fp8idx_n131072"
SUITE = ("csa_fp32_n256", "csa_bf16_n4096", "hca_bf16_n65536", "csa_fp8idx_n131072",
         "decode_b8_ctx1m")
L2_FLUSH_BYTES = 512 << 20
# query rows of the oracle's bounded sample, per workload (prefill: the
# quadratic steps run on these rows, stratified over the sequence)
ORACLE_ROWS = {"csa_fp32_n256": 256, "csa_bf16_n4096": 256, "hca_bf16_n65536": 64,
               "csa_fp8idx_n131072": 32}


def peaks():
    """Roofline denominators: measured HBM copy bandwidth and dense bf16
    throughput when present; e4m3 contractions take twice the bf16 figure
    (the nominal dense fp8 : bf16 ratio of B200) until fp8 is measured."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        bf16 = d["bf16_tflops"]
        return {"hbm": d["hbm_gbs"], "bf16": bf16,
                "bf16_sustained": d.get("bf16_tflops_sustained", bf16),
                "fp8": d.get("fp8_tflops", 2.0 * bf16),
                "fp8_source": "measured" if "fp8_tflops" in d else "nominal-ratio (2 x measured bf16)",
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "fp8": 3180.0,
            "fp8_source": "nominal-ratio (2 x fallback bf16)", "source": "fallback"}


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


# --------------------------------------------------------------------------- host logic


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


def units_per_step(w):
    if w.kind == "decode":
        return w.batch
    return LAST_N if (LAST_N and w.kind == "csa") else w.n


def unit_of(w):
    return "queries/s" if w.kind == "decode" else "tokens/s"


# --fp4-keys: the indexer keys are stored in FP4 (e2m1 + a power-of-two scale
# per 32 channels) instead of the workload's e4m3 keys
FP4_KEYS = False
# --last N: a CSA prefill step runs only the last N queries of the sequence
# (its longest rows) over the whole sequence's entries (profiling cases)
LAST_N = None


def config_of(w, world=1):
    """The workload description both arms print (same keys, same values)."""
    cfg = {"workload": w.name, "n": w.n, "c": w.c, "m": w.m, "k": w.k, "h": w.h,
           "hI": w.hI, "cI": w.cI, "n_win": w.n_win, "dtype": w.dtype,
           "indexer_dtype": w.idx_dtype, "batch_per_gpu": w.batch,
           "l2": "flushed between timed steps (512 MiB write)",
           "parallelism": "dp%d (independent sequences)" % world}
    if FP4_KEYS and w.hI:
        cfg["indexer_keys"] = "e2m1, one power-of-two scale per 32 channels"
    if LAST_N and w.kind == "csa":
        cfg["queries"] = "the last %d positions" % LAST_N
    return cfg


def build_path(w, rank, keep_ops=False):
    """The device-resident step of rank `rank` (and, with keep_ops, the host
    operands it was built from)."""
    from long_context_sparse_07_b200 import path
    wr = rank_workload(w, rank)
    if w.kind == "csa" and LAST_N:
        q_lo = wr.n - LAST_N
        ops = W.csa_operands(wr, parts=("kv", "indexer"))
        for k in ("qI", "qI_scale", "wI"):
            if k in ops:
                ops[k] = ops[k][q_lo:].contiguous()
        ops.update(W.csa_operands(wr, lo=q_lo, parts=("query",)))
        p = path.CsaPrefill(wr, ops, fused=True, fp4_keys=FP4_KEYS and w.idx_dtype == "e4m3",
                            q_lo=q_lo)
    elif w.kind == "csa":
        ops = W.csa_operands(wr)
        p = path.CsaPrefill(wr, ops, fused=True, fp4_keys=FP4_KEYS and w.idx_dtype == "e4m3")
    elif w.kind == "hca":
        ops = W.hca_operands(wr)
        p = path.HcaPrefill(wr, ops)
    else:
        ops = W.decode_operands(wr, fp4_keys=FP4_KEYS)
        p = path.Decode(wr, ops)
    return (p, ops) if keep_ops else p


def algorithmic(w, p):
    if w.kind == "csa":
        return work.csa_prefill(w, fp4_keys=getattr(p, "fp4_keys", False), q_lo=w.n - p.nq)
    if w.kind == "hca":
        return work.hca_prefill(w)
    return work.decode(w, p.E, p.E_hca, fp4_keys=getattr(p, "fp4_keys", False))


def kernel_roofline(w, name, a, ms, pk):
    """Roofline of one kernel from its algorithmic work `a` ({"flops",
    "bytes"}) and its mean launch time: bound = the slower of the tensor-core
    time (at the peak of its operand dtype) and the HBM time; frac = that
    ideal time over the measured one."""
    if w.dtype == "f32":
        # CUDA-core float32 path of the parity-sized workload: no tensor peak
        # applies; report against HBM only
        tensor_peak, pdt = None, None
    elif name in ("indexer", "indexer_topk") and w.idx_dtype == "e4m3":
        tensor_peak, pdt = pk["fp8"], "e4m3"
    else:
        tensor_peak, pdt = pk["bf16"], "bf16"
    t_hbm = a["bytes"] / (pk["hbm"] * 1e9)
    t_ten = a["flops"] / (tensor_peak * 1e12) if tensor_peak and a["flops"] else 0.0
    sec = ms * 1e-3
    if t_ten > t_hbm:
        r = {"bound": "tensor", "achieved": a["flops"] / sec / 1e12, "peak": tensor_peak,
             "unit": "TFLOP/s", "peak_dtype": pdt}
    else:
        r = {"bound": "hbm", "achieved": a["bytes"] / sec / 1e9, "peak": pk["hbm"],
             "unit": "GB/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["ideal_ms"] = max(t_ten, t_hbm) * 1e3
    return r


# DRAM bytes (read + write) per launch of a kernel from one ncu capture
# (summarised under profiles/), keyed by workload and kernel; each entry holds the
# SHA-1 of the kernel source it was taken on and the number of launches it covers
# scaled to a full launch, and counts only while that source is unchanged.
MEASURED_TRAFFIC = {
    # attention at n = 16384 (1.16 GB read + 1.04 GB write, q / out dominated),
    # scaled by 131072 / 16384 = 8 queries per captured query
    ("csa_fp8idx_n131072", "attend"): ("attend_tc.cu", "99901d1152b0dc2bdd984b72efca53cb4622615e",
                                       8 * (1.163732e9 + 1.040877e9)),
}


def measured_traffic(workload, kernel):
    ent = MEASURED_TRAFFIC.get((workload, kernel))
    if ent is None:
        return None
    src = os.path.join(ROOT, "long_context_sparse_07_b200", "csrc", ent[0])
    try:
        with open(src, "rb") as f:
            digest = hashlib.sha1(f.read()).hexdigest()
    except OSError:
        return None
    return ent[2] if digest == ent[1] else None


# --------------------------------------------------------------------------- timing


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
    if hasattr(p, "step_from_host"):
        # one untimed step first: its copy streams and chunk workspaces are
        # created on the first call
        p.step_from_host(host_in, host_out, stream)
        torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if hasattr(p, "step_from_host"):
            # the copies overlap the computation (queries in chunks)
            p.step_from_host(host_in, host_out, stream)
        else:
            for k, v in host_in.items():
                dev_in[k].copy_(v, non_blocking=True)
            p.step(stream)
            host_out.copy_(res, non_blocking=True)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    del host_in, host_out
    return [a.elapsed_time(b) for a, b in times], h2d, d2h


def measure(p, w, steps, warmup, graph, flush, stream, barrier, clk=None):
    """Warm-up, then `steps` timed steps; returns (mean step ms, mean kernel
    ms by name, whether a graph was replayed)."""
    from long_context_sparse_07_b200 import abi
    for _ in range(warmup):
        p.step(stream)
    torch.cuda.synchronize()
    abi.csa_get_error()
    barrier()
    use_graph = graph == "on" or (graph == "auto" and w.kind == "decode")
    if clk is not None:
        with clk:
            f = time_steps_graph if use_graph else time_steps
            step_ms, kern_ms = f(p, steps, flush, stream)
    else:
        f = time_steps_graph if use_graph else time_steps
        step_ms, kern_ms = f(p, steps, flush, stream)
    barrier()
    abi.csa_get_error()
    kavg = {n: sum(v) / len(v) for n, v in kern_ms.items()}
    return sum(step_ms) / len(step_ms), kavg, use_graph


def workload_summary(w, p, step_ms, kavg, use_graph, pk, steps):
    """Per-kernel rooflines and the whole step's fraction of its ideal time
    (sum of the kernels' ideal times over the measured step time)."""
    alg = algorithmic(w, p)
    kernels = {n: kernel_roofline(w, n, alg[n], kavg[n], pk) for n in kavg}
    ideal = sum(r["ideal_ms"] for r in kernels.values())
    out = {"ms_per_step": step_ms, "value": units_per_step(w) / (step_ms * 1e-3),
           "unit": unit_of(w), "steps": steps,
           "launch": "CUDA graph replay" if use_graph else "eager",
           "kernel_ms": {n: round(v, 5) for n, v in kavg.items()},
           "kernels": {n: {k: (round(v, 4) if isinstance(v, float) else v)
                           for k, v in r.items()} for n, r in kernels.items()},
           "step_frac": ideal / step_ms if w.dtype != "f32" else None,
           "dominant": max(kavg, key=kavg.get)}
    if w.kind == "decode":
        names = ("indexer", "topk", "attend")
        ms = sum(kavg[n] for n in names)
        by = sum(alg[n]["bytes"] for n in names)
        out["csa_step"] = {"kernels": list(names), "ms": ms, "bytes": by,
                           "achieved": by / (ms * 1e-3) / 1e9, "peak": pk["hbm"],
                           "unit": "GB/s", "frac": by / (ms * 1e-3) / 1e9 / pk["hbm"]}
    return out


def time_norm_rope(p, w, pk, stream, steps=5):
    """Device time of the RMSNorm + partial RoPE calls on a CSA step's own
    tensors (entries and window rows; queries; the output turned back), each
    read and written once: bytes = 2 x the tensor's bytes."""
    from long_context_sparse_07_b200 import abi
    kwin = torch.empty_like(p.d["Ca"])
    calls = {
        "rope_entries": (lambda: abi.csa_norm_rope(p.entries.body, 64, pos=None, pos_mul=w.m,
                                                   pos_add=w.m - 1), p.entries.body),
        "rope_window": (lambda: abi.csa_norm_rope(kwin, 64, pos=None), kwin),
        "rope_q": (lambda: abi.csa_norm_rope(p.d["q"], 64, pos=p.q_pos), p.d["q"]),
        "rotate_back": (lambda: abi.csa_norm_rope(p.out[0], 64, pos=p.q_pos, pos_mul=-1,
                                                  normalise=False), p.out),
    }
    res = {}
    for name, (f, t) in calls.items():
        f()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            f()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        by = 2 * t.numel() * t.element_size()
        res[name] = {"ms": ms, "bytes": by, "achieved": by / (ms * 1e-3) / 1e9,
                     "peak": pk["hbm"], "unit": "GB/s", "frac": by / (ms * 1e-3) / 1e9 / pk["hbm"]}
    abi.csa_get_error()
    del kwin
    return res


def time_out_proj(p, w, pk, stream, steps=3, g=8, dg=1024, d=4096):
    """Device time of the grouped output projection (g groups of d_g, then
    d; the Flash configuration) on the step's own attention output; random
    N(0, 0.02^2) weights. Work: 2 n (h c d_g + g d_g d) FLOPs."""
    from long_context_sparse_07_b200 import abi
    n = w.n
    gen = torch.Generator(device="cuda").manual_seed(5)
    Wg = (torch.randn(g * dg, w.h * w.c // g, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    Wo = (torch.randn(d, g * dg, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    u = torch.empty(n, g * dg, device="cuda", dtype=torch.bfloat16)
    out = torch.empty(n, d, device="cuda", dtype=torch.bfloat16)
    o = p.out[0]
    abi.csa_grouped_out_proj(o, Wg, Wo, g, u, out)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        abi.csa_grouped_out_proj(o, Wg, Wo, g, u, out)
    b.record(stream)
    torch.cuda.synchronize()
    abi.csa_get_error()
    ms = a.elapsed_time(b) / steps
    fl = 2.0 * n * (w.h * w.c * dg + g * dg * d)
    del Wg, Wo, u, out
    return {"ms": ms, "flops": fl, "achieved": fl / (ms * 1e-3) / 1e12, "peak": pk["bf16"],
            "unit": "TFLOP/s", "frac": fl / (ms * 1e-3) / 1e12 / pk["bf16"],
            "shape": {"n": n, "h": w.h, "c": w.c, "g": g, "dg": dg, "d": d}}


def _fp4_keys(rows, cI, seed):
    """Random FP4 indexer keys on the device: packed e2m1 codes and block
    exponents within a span of 8."""
    from long_context_sparse_07_b200.abi import Entries
    gen = torch.Generator(device="cuda").manual_seed(seed)
    body = torch.randint(0, 256, (rows, cI // 2), device="cuda", dtype=torch.uint8, generator=gen)
    exps = torch.randint(118, 127, (rows, cI // 32), device="cuda", dtype=torch.uint8,
                         generator=gen)
    return Entries(body, cI, scale=exps, scale_group=32, fp4=True)


def _event_ms(f, stream, flush, steps):
    ts = []
    for _ in range(steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        f()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return sum(ts) / len(ts)


def time_fp4_prefill(p, w, pk, stream, flush, steps=3):
    """The step's indexer and top-k in one call with FP4 keys (random codes
    of the same shape) in place of its e4m3 keys, L2 flushed in between."""
    from long_context_sparse_07_b200 import abi
    kI = _fp4_keys(w.E, w.cI, 11)
    d = p.d
    qs = d.get("qI_scale")
    f = lambda: abi.csa_indexer_topk(d["qI"][None], qs[None], d["wI"][None], kI, p.q_pos[None],
                                     w.m, w.k, p.idx, w.E, workspace=p.fused_ws)
    f()
    torch.cuda.synchronize()
    ms = _event_ms(f, stream, flush, steps)
    abi.csa_get_error()
    fl = work.csa_prefill(w)["indexer_topk"]["flops"]
    return {"ms": ms, "flops": fl, "achieved": fl / (ms * 1e-3) / 1e12, "peak": pk["fp8"],
            "unit": "TFLOP/s", "frac": fl / (ms * 1e-3) / 1e12 / pk["fp8"],
            "keys": "e2m1 + one power-of-two scale per 32 channels (68 bytes per key)"}


def time_fp4_decode(pk, stream, flush, steps=20):
    """Decode indexer over FP4 keys against the same call over e4m3 keys, on
    the decode workload's queries and cache length (HBM-bound: the keys are
    most of the bytes)."""
    from long_context_sparse_07_b200 import abi
    w = W.WORKLOADS["decode_b8_ctx1m"]
    B, E, sd = w.batch, w.n // w.m, w.seed
    # the decode workload's queries (the same generators and seeds)
    qI = W.e4m3_codes(sd, "qI", B, w.hI * w.cI).view(B, 1, w.hI, w.cI).cuda()
    qs = W.e4m3_scales(sd, "qI_scale", B, w.hI, w.std_q).view(B, 1, w.hI).cuda()
    wI = W.to_storage(W.normal(sd, "wI", B, w.hI, w.std_w), "f32").view(B, 1, w.hI).cuda()
    q_pos = torch.full((B, 1), w.n - 1, dtype=torch.int64, device="cuda")
    scores = torch.empty(B, 1, E, device="cuda")
    res = {}
    for name, kI, kbytes in (("e4m3", None, w.cI + 4), ("e2m1", _fp4_keys(B * E, w.cI, 12),
                                                         w.cI // 2 + w.cI // 32)):
        if kI is None:
            from long_context_sparse_07_b200.abi import Entries
            body = torch.randint(-100, 100, (B * E, w.cI), device="cuda",
                                 dtype=torch.int8).view(torch.float8_e4m3fn)
            sc = torch.rand(B * E, device="cuda") + 0.5
            kI = Entries(body, w.cI, scale=sc, scale_group=w.cI)
        f = lambda: abi.csa_indexer_scores(qI, qs, wI, kI, q_pos, w.m, scores, E)
        f()
        torch.cuda.synchronize()
        ms = _event_ms(f, stream, flush, steps)
        by = B * E * kbytes + B * w.hI * (w.cI + 8) + B * E * 4
        res[name] = {"ms": ms, "bytes": by, "achieved": by / (ms * 1e-3) / 1e9,
                     "peak": pk["hbm"], "unit": "GB/s", "frac": by / (ms * 1e-3) / 1e9 / pk["hbm"],
                     "key_bytes": kbytes}
        del kI
    abi.csa_get_error()
    res["speedup"] = res["e4m3"]["ms"] / res["e2m1"]["ms"]
    return res


# --------------------------------------------------------------------------- CPU oracle


def stratified_rows(n, count, seed):
    """`count` query positions, one uniform pick in each of `count` equal
    strata of [0, n) (all positions when count >= n)."""
    if count >= n:
        return np.arange(n, dtype=np.int64)
    g = np.random.default_rng(seed)
    lo = (np.arange(count) * n) // count
    hi = ((np.arange(count) + 1) * n) // count
    return (lo + np.floor(g.random(count) * (hi - lo))).astype(np.int64)


class OracleSample:
    """A bounded sample of one workload for the float64 CPU oracle, with
    every input converted to float64 before any timing.

    Prefill: the linear compression steps run over the whole sequence, the
    quadratic steps (indexer, top-k, attention) over `rows` stratified query
    positions; the whole workload's time is estimated as
    t_compress + t_rows * n / rows. Decode: one query (sequence 0) over its
    full cache, every step of the decode path; the batch takes B times that.
    """

    def __init__(self, w, seed=0, ops=None):
        import oracle
        from oracle import pipeline
        self.oracle, self.pipeline, self.w = oracle, pipeline, w
        f64 = oracle.f64
        if w.kind == "decode":
            ws = W.scaled(w, batch=1)
            if ops is None:
                ops = W.decode_operands(ws)
            else:
                # sequence 0 of a batch: every operand but the sink is batched
                ops = {k: (v if k == "sink" else v[:1]) for k, v in ops.items()}
            self.rows = 1
            self.qI = oracle.dequantize(ops["qI"], ops["qI_scale"].reshape(1, 1, w.hI, 1), w.cI)
            self.kI = oracle.dequantize(ops["kI"], ops["kI_scale"].reshape(1, -1, 1), w.cI)
            self.ent = pipeline.split_entries(ops["kv_nope"], ops["kv_scale"], ops["kv_rope"],
                                              w.scale_group)
            self.hent = pipeline.split_entries(ops["hca_nope"], ops["hca_scale"],
                                               ops["hca_rope"], w.scale_group)
            self.wI, self.q, self.kwin = f64(ops["wI"]), f64(ops["q"]), f64(ops["kwin"])
            self.sink = f64(ops["sink"])
            self.pos = ops["q_pos"].numpy()
            self.win_pos0 = ops["win_pos0"].numpy()
            self.sample = ("1 of %d decode queries (sequence 0 over its full %d-token cache: "
                           "indexer, top-k, CSA and HCA attention), caches decoded to float64 "
                           "before timing; batch time = %d x that"
                           % (w.batch, w.n, w.batch))
            return
        self.rows = stratified_rows(w.n, ORACLE_ROWS.get(w.name, 64), seed)
        R = self.rows
        if w.kind == "csa":
            ops = W.csa_operands(w) if ops is None else ops
            self.kv = [f64(ops[k]) for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")]
            self.ki = [f64(ops[k]) for k in ("CIa", "CIb", "ZIa", "ZIb", "BIa", "BIb")]
            self.qI, self.wI = pipeline._indexer_operands(ops, R, w)
            self.win = self.kv[0]
        else:
            ops = W.hca_operands(w) if ops is None else ops
            self.kv = [f64(ops[k]) for k in ("C", "Z", "B")]
            self.win = self.kv[0]
        self.q = f64(ops["q"][torch.as_tensor(R)])
        self.sink = f64(ops["sink"])
        self.sample = ("compression over all %d tokens; indexer, top-k and attention over %d "
                       "stratified query rows of %d; whole-sequence time = t_compress + "
                       "t_rows x n / rows; inputs converted to float64 before timing"
                       % (w.n, len(R), w.n) if len(R) < w.n else
                       "the whole workload (all %d query rows)" % w.n)

    def run(self):
        """Times one pass of the sample; returns the estimated seconds of the
        whole workload (one step) and the seconds actually spent."""
        o, pl, w = self.oracle, self.pipeline, self.w
        scale = 1.0 / math.sqrt(w.c)
        t0 = time.perf_counter()
        if w.kind == "decode":
            sc = o.indexer(self.qI, self.wI, self.kI, self.pos, w.m)
            sel = o.topk(sc.reshape(1, -1).astype(np.float32), self.pos.reshape(1), w.m, w.k)
            o.attend(self.q, self.ent, sel, w.k, w.m, self.kwin, self.win_pos0, w.n_win,
                     self.pos, self.sink, scale)
            o.attend(self.q, self.hent, None, 0, w.m_hca, self.kwin, self.win_pos0, w.n_win,
                     self.pos, self.sink, scale)
            dt = time.perf_counter() - t0
            return dt * w.batch, dt
        R = self.rows
        pos = R.reshape(1, -1)
        if w.kind == "csa":
            ent = pl.store(o.compress(*self.kv, w.m, True), w.dtype)
            k64 = o.compress(*self.ki, w.m, True)
            if w.idx_dtype == "e4m3":
                codes, scales = o.quantize_e4m3(k64, w.cI)
                kI = o.dequantize(codes, scales, w.cI)
            else:
                kI = pl.store(k64, w.idx_dtype)
            t1 = time.perf_counter()
            sc = o.indexer(self.qI[None], self.wI[None], kI[None], pos, w.m)[0]
            sel = o.topk(sc.astype(np.float32), R, w.m, w.k)
            o.attend(self.q[None], ent[None], sel, w.k, w.m, self.win[None], [0], w.n_win, pos,
                     self.sink, scale)
        else:
            C, Z, B = self.kv
            ent = pl.store(o.compress(C, None, Z, None, B, None, w.m, False), w.dtype)
            t1 = time.perf_counter()
            o.attend(self.q[None], ent[None], None, 0, w.m, self.win[None], [0], w.n_win, pos,
                     self.sink, scale)
        t2 = time.perf_counter()
        return (t1 - t0) + (t2 - t1) * w.n / len(R), t2 - t0


def oracle_cores():
    """Threads the oracle's OpenMP loops use."""
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else os.cpu_count()


def host_operands(w):
    """The workload's operands on the host (decode: sequence 0 only, the
    part the oracle sample reads)."""
    if w.kind == "csa":
        return W.csa_operands(w)
    if w.kind == "hca":
        return W.hca_operands(w)
    return W.decode_operands(W.scaled(w, batch=1))


def cpu_baseline(w, ops=None):
    """The oracle as it stands on a bounded sample (OracleSample)."""
    s = OracleSample(w, ops=ops)
    s.run()                                   # first pass: page-in, thread start-up
    est, spent = s.run()
    return {"value": units_per_step(w) / est, "unit": unit_of(w), "cores": oracle_cores(),
            "kind": "oracle", "sample": s.sample, "sample_s": round(spent, 3)}


# --------------------------------------------------------------------------- our arm


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
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    pk = peaks()

    def barrier():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()

    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    p, host_ops = build_path(w, rank, keep_ops=True)
    if not want_cpu:
        host_ops = None
    clk = ClockSampler(local)
    mean_ms, kavg, use_graph = measure(p, w, args.steps, args.warmup, args.graph, flush, stream,
                                       barrier, clk)
    value, ms = job_rate(mean_ms, units_per_step(w), world, dist, "cuda")
    summ = workload_summary(w, p, mean_ms, kavg, use_graph, pk, args.steps)

    # end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, 20 if units_per_step(w) * w.h * w.c < (1 << 30) else 3))
    e_ms, h2d, d2h = time_e2e(p, e2e_steps, stream)
    e2e_value, _ = job_rate(sum(e_ms) / len(e_ms), units_per_step(w), world, dist, "cuda")

    # the Module D normalisation and partial RoPE (outside the configs' step):
    # timed on this workload's own buffers, after the step measurements
    extras = {}
    if w.kind == "csa" and w.c >= 64 and not args.no_extras:
        extras["norm_rope"] = time_norm_rope(p, w, pk, stream)
        if w.dtype == "bf16" and w.h % 8 == 0:
            extras["grouped_out_proj"] = time_out_proj(p, w, pk, stream)
        if w.idx_dtype == "e4m3" and w.cI == 128 and p.fused:
            extras["fp4_keys_prefill"] = time_fp4_prefill(p, w, pk, stream, flush)
        extras["fp4_keys_decode"] = time_fp4_decode(pk, stream, flush)

    dom = summ["dominant"]
    roof = dict(summ["kernels"][dom])
    roof.pop("ideal_ms", None)
    roof["traffic"] = measured_traffic(w.name, dom) if not (LAST_N or FP4_KEYS) else None
    roof["kernel"] = dom
    roof["peak_source"] = pk["source"] if roof.get("peak_dtype") != "e4m3" else pk["fp8_source"]
    roof["kernel_ms"] = summ["kernel_ms"]
    launches = p.launches_per_step * args.steps
    del p
    torch.cuda.empty_cache()

    # every other workload of the suite, each on its own (rank-local) inputs
    per = {}
    if not args.no_per_workload and args.n is None:
        for name in SUITE:
            if name == w.name:
                per[name] = summ
                continue
            wn = W.WORKLOADS[name]
            pn = build_path(wn, rank)
            steps_n = max(3, min(args.steps, 10))
            m_n, k_n, g_n = measure(pn, wn, steps_n, args.warmup, args.graph, flush, stream,
                                    barrier)
            per[name] = workload_summary(wn, pn, m_n, k_n, g_n, pk, steps_n)
            launches += pn.launches_per_step * steps_n
            del pn
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": unit_of(w), "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded generators; random-init projection outputs)",
            "config": config_of(w, world),
            "launch": "CUDA graph replay" if use_graph else "eager",
            "e2e": {"value": e2e_value, "unit": unit_of(w), "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "ms_per_step": [round(x, 3) for x in e_ms]},
            "gpu_launches": launches,
            "roofline": roof,
            "step_frac": summ["step_frac"],
            "clocks": clk.summary(),
            "peaks": {k: pk[k] for k in ("hbm", "bf16", "bf16_sustained", "fp8", "source",
                                         "fp8_source")},
        }
        if per:
            line["per_workload"] = per
        if extras:
            line["extras"] = extras
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, host_ops)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- reference arm


def run_reference(args, w):
    """The CPU oracle timed as the reference arm: each step is one pass of the
    same bounded sample as ``cpu_baseline`` (new stratified rows per step)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    ops = host_operands(w)
    samples = [OracleSample(w, seed=s, ops=ops) for s in range(2)]
    del ops
    est, spent = [], []
    for i in range(args.steps + args.warmup):
        e, s = samples[i % 2].run()
        if i >= args.warmup:
            est.append(e)
            spent.append(s)
    t_est = sum(est) / len(est)
    value = units_per_step(w) / t_est
    unit = unit_of(w)
    cores = oracle_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(spent) / len(spent),
            "ms_per_workload_estimated": 1e3 * t_est,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded generators)",
            "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": samples[0].sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the selected workload")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the RMSNorm/RoPE and grouped-projection timings")
    ap.add_argument("--fp4-keys", action="store_true",
                    help="store the indexer keys in FP4 (e2m1 + a scale per 32 channels); "
                         "no CPU baseline or reference arm in this mode")
    ap.add_argument("--last", type=int, default=None,
                    help="CSA prefill: run only the last N queries over the whole sequence's "
                         "entries (profiling cases; no CPU baseline or reference arm)")
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
    if args.last is not None:
        if args.impl == "reference" or w.kind != "csa" or not 0 < args.last <= w.n:
            sys.exit("--last takes 0 < N <= n on a CSA prefill workload, our arm only")
        global LAST_N
        LAST_N = args.last
        args.no_cpu_baseline = True
        args.no_extras = True
        args.no_per_workload = True
    if args.fp4_keys:
        if args.impl == "reference":
            sys.exit("--fp4-keys has no reference arm")
        global FP4_KEYS
        FP4_KEYS = True
        args.no_cpu_baseline = True
        args.no_extras = True
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
