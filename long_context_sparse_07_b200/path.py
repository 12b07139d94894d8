"""Device-resident steps of the hot path, built on the C ABI.

``CsaPrefill``, ``HcaPrefill`` and ``Decode`` hold one workload's operands and
outputs in device memory and run one pass of the path per ``step()``:

* CSA prefill: compress KV entries -> compress indexer keys -> indexer scores
  -> top-k -> sparse shared-KV attention (window + sink); with ``fused`` the
  scores and the top-k are one call (``csa_indexer_topk``) that does not
  write the score rows;
* HCA prefill: compress (m' = 128, no overlap) -> dense shared-KV attention;
* decode: indexer scores -> top-k -> sparse attention, and HCA dense
  attention, for a batch of single-token queries over long caches.

Only buffer management and argument marshalling live here; every step runs
in ``libcsa.so``. The raw window KV of a prefill is the pre-compression KV
(C^a for CSA, C for HCA).
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import torch

from . import abi
from .abi import Entries

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _dev(ops: Dict[str, torch.Tensor], device) -> Dict[str, torch.Tensor]:
    return {k: v.to(device, non_blocking=False).contiguous() for k, v in ops.items()}


class CsaPrefill:
    """One causal CSA prefill of a single sequence (batch 1)."""

    kind = "csa"

    @property
    def launches_per_step(self):
        """Kernels launched by one step (top-k of long rows takes four; the
        normalisation and RoPE add four)."""
        if self.fused:
            sel = abi.csa_indexer_topk_launches(1, self.nq, self.w.E, self.w.hI, self.w.cI,
                                                self.w.k, self.d["qI"])
        else:
            sel = 1 + (4 if self.topk_ws is not None else 1)
        return 3 + sel + (4 if self.rope_dims else 0)

    def __init__(self, w, ops: Dict[str, torch.Tensor], device="cuda", rope_dims: int = 0,
                 fused: bool = False, fp4_keys: bool = False, q_lo: int = 0):
        """`ops` as ``workloads.csa_operands``; with q_lo > 0 the queries (q,
        qI, qI_scale, wI) are only those of positions q_lo .. n - 1 (the
        sequence's longest rows), the KV side the whole sequence."""
        self.w = w
        self.fused = fused
        self.fp4_keys = fp4_keys
        d = self.d = _dev(ops, device)
        c, E = w.c, w.E
        n = self.nq = w.n - q_lo
        # with rope_dims > 0 the step also applies Module D's RMSNorm and
        # partial RoPE to the entries, the window rows (a copy of C^a) and the
        # queries, and turns the output back by the query position
        self.rope_dims = rope_dims
        self.kwin = torch.empty_like(d["Ca"]) if rope_dims else d["Ca"]
        self.q_pos = torch.arange(q_lo, w.n, device=device, dtype=torch.int64)
        self.win_pos0 = torch.zeros(1, device=device, dtype=torch.int64)
        self.entries = Entries(torch.empty(E, c, device=device, dtype=DT[w.dtype]), c)
        if fp4_keys:
            # FP4 indexer keys (e2m1 + a power-of-two scale per 32 channels),
            # written by the compressor; the queries stay e4m3
            self.kI = Entries(torch.empty(E, w.cI // 2, device=device, dtype=torch.uint8), w.cI,
                              scale=torch.empty(E, w.cI // 32, device=device, dtype=torch.uint8),
                              scale_group=32, fp4=True)
        elif w.idx_dtype == "e4m3":
            self.kI = Entries(torch.empty(E, w.cI, device=device, dtype=torch.float8_e4m3fn),
                              w.cI, scale=torch.empty(E, device=device, dtype=torch.float32),
                              scale_group=w.cI)
        else:
            self.kI = Entries(torch.empty(E, w.cI, device=device, dtype=DT[w.idx_dtype]), w.cI)
        self.idx = torch.empty(n, w.k, device=device, dtype=torch.int32)
        if fused:
            self.scores = self.topk_ws = None
            nf = abi.csa_indexer_topk_workspace_size(1, n, E, w.hI, w.cI, w.k, d["qI"])
            self.fused_ws = torch.empty(nf, device=device, dtype=torch.uint8) if nf else None
        else:
            self.scores = torch.empty(1, n, E, device=device, dtype=torch.float32)
            nt = abi.csa_topk_workspace_size(n, E, w.k)
            self.topk_ws = torch.empty(nt, device=device, dtype=torch.uint8) if nt else None
        self.out = torch.empty(1, n, w.h, c, device=device, dtype=DT[w.dtype])
        self.lse = torch.empty(1, n, w.h, device=device, dtype=torch.float32)
        self.scale = 1.0 / math.sqrt(c)

    def compress_kv(self, stream=None):
        d, w = self.d, self.w
        abi.csa_compress_kv(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], w.m, True,
                            self.entries, stream)

    def compress_index(self, stream=None):
        d, w = self.d, self.w
        abi.csa_compress_kv(d["CIa"], d["CIb"], d["ZIa"], d["ZIb"], d["BIa"], d["BIb"], w.m,
                            True, self.kI, stream)

    def index(self, stream=None):
        d, w = self.d, self.w
        qs = d.get("qI_scale")
        abi.csa_indexer_scores(d["qI"][None], qs[None] if qs is not None else None,
                               d["wI"][None], self.kI, self.q_pos[None], w.m, self.scores,
                               w.E, stream)

    def select(self, stream=None):
        w = self.w
        abi.csa_topk(self.scores[0], self.q_pos, w.m, w.k, self.idx, w.E, workspace=self.topk_ws,
                     stream=stream)

    def index_select(self, stream=None):
        """Indexer scores and top-k in one call (no score rows written)."""
        d, w = self.d, self.w
        qs = d.get("qI_scale")
        abi.csa_indexer_topk(d["qI"][None], qs[None] if qs is not None else None, d["wI"][None],
                             self.kI, self.q_pos[None], w.m, w.k, self.idx, w.E,
                             workspace=self.fused_ws, stream=stream)

    def attend(self, stream=None):
        d, w = self.d, self.w
        abi.csa_sparse_mqa(d["q"][None], self.entries, w.E, w.m, self.idx, w.k, self.kwin[None],
                           self.win_pos0, w.n_win, self.q_pos[None], d["sink"], self.scale,
                           self.out, self.lse, stream=stream)

    def rope_kv(self, stream=None):
        """RMSNorm + RoPE of the entries (at their blocks' last tokens) and of
        the window rows (a copy of C^a, at their own positions)."""
        w = self.w
        abi.csa_norm_rope(self.entries.body, self.rope_dims, pos=None, pos_mul=w.m,
                          pos_add=w.m - 1, stream=stream)
        self.kwin.copy_(self.d["Ca"])
        abi.csa_norm_rope(self.kwin, self.rope_dims, pos=None, stream=stream)

    def rope_q(self, stream=None):
        abi.csa_norm_rope(self.d["q"], self.rope_dims, pos=self.q_pos, stream=stream)

    def rotate_back(self, stream=None):
        abi.csa_norm_rope(self.out[0], self.rope_dims, pos=self.q_pos, pos_mul=-1,
                          normalise=False, stream=stream)

    def phases(self):
        """The kernels of one step, in order: (name, launch)."""
        sel = [("indexer_topk", self.index_select)] if self.fused else \
            [("indexer", self.index), ("topk", self.select)]
        ph = [("compress_kv", self.compress_kv), ("compress_index", self.compress_index)] + sel + \
            [("attend", self.attend)]
        if self.rope_dims:
            ph = ph[:1] + [("rope_kv", self.rope_kv)] + ph[1:-1] + [("rope_q", self.rope_q)] + \
                ph[-1:] + [("rotate_back", self.rotate_back)]
        return ph

    def inputs(self):
        """Device operands a step reads (copied from the host in end-to-end runs)."""
        return {k: v for k, v in self.d.items()}

    def result(self):
        return self.out

    def step(self, stream=None):
        for _, f in self.phases():
            f(stream)

    QUERY_SIDE = ("q", "qI", "qI_scale", "wI")

    @staticmethod
    def chunk_plan(nq: int, chunk: int, small: int = 2048):
        """Query chunk sizes for ``step_from_host``: doubling from ``small`` up
        to ``chunk`` at the start (the first output leaves early, so the
        device-to-host copies run beside the host-to-device ones for most of
        the step), full chunks in the middle, and halving back to ``small`` at
        the end (little computation and output are left once the last queries
        have arrived)."""
        ramp = []
        s = small
        while s < chunk:
            ramp.append(s)
            s *= 2
        mid = nq - 2 * sum(ramp)
        if not ramp or mid < chunk:
            return [min(chunk, nq - lo) for lo in range(0, nq, chunk)]
        sizes = list(ramp) + [chunk] * (mid // chunk)
        if mid % chunk:
            sizes.append(mid % chunk)
        return sizes + ramp[::-1]

    def step_from_host(self, host_in: Dict[str, torch.Tensor], host_out: torch.Tensor,
                       stream=None, chunk: int = 8192):
        """One step from pinned host operands (keys as ``inputs()``) to a
        pinned host output (shaped like ``result()``), the copies overlapped
        with the computation: the KV side arrives first and is compressed;
        then the queries come in chunks (``chunk_plan``), each chunk's
        selection and attention running while the next chunk's queries arrive
        and the previous chunk's output leaves on a second copy stream
        (host-to-device and device-to-host copies run at the same time). The
        result equals ``step()``'s: every query's work is the same, only
        grouped by chunk."""
        cur = stream if stream is not None else torch.cuda.current_stream()
        d, w = self.d, self.w
        if self.rope_dims or not self.fused:
            for k, v in host_in.items():
                d[k].copy_(v, non_blocking=True)
            self.step(cur)
            host_out.copy_(self.out, non_blocking=True)
            return
        if not hasattr(self, "_h2d"):
            self._h2d, self._d2h = torch.cuda.Stream(), torch.cuda.Stream()
            self._chunk_ws = {}
        h2d, d2h = self._h2d, self._d2h
        h2d.wait_stream(cur)                      # earlier work on these buffers is done
        d2h.wait_stream(cur)
        qside = [k for k in self.QUERY_SIDE if k in d]
        with torch.cuda.stream(h2d):
            for k, v in host_in.items():
                if k not in qside:
                    d[k].copy_(v, non_blocking=True)
        cur.wait_event(h2d.record_event())
        self.compress_kv(cur)
        self.compress_index(cur)
        qs = d.get("qI_scale")
        plan = self.chunk_plan(self.nq, chunk)
        # one workspace pair, for the largest chunk (the chunks run one after
        # another on one stream)
        big = max(plan)
        if big not in self._chunk_ws:
            nf = max(abi.csa_indexer_topk_workspace_size(1, r, w.E, w.hI, w.cI, w.k, d["qI"])
                     for r in set(plan))
            na = max(abi.csa_mqa_workspace_size(1, r, w.h, w.c, w.k + w.n_win) for r in set(plan))
            self._chunk_ws = {big: (
                torch.empty(nf, device=self.out.device, dtype=torch.uint8) if nf else None,
                torch.empty(na, device=self.out.device, dtype=torch.uint8) if na else None)}
        fws, aws = self._chunk_ws[big]
        lo = 0
        for rows in plan:
            hi = lo + rows
            with torch.cuda.stream(h2d):
                for k in qside:
                    d[k][lo:hi].copy_(host_in[k][lo:hi], non_blocking=True)
            cur.wait_event(h2d.record_event())
            abi.csa_indexer_topk(d["qI"][lo:hi][None], qs[lo:hi][None] if qs is not None else None,
                                 d["wI"][lo:hi][None], self.kI, self.q_pos[lo:hi][None], w.m, w.k,
                                 self.idx[lo:hi], w.E, workspace=fws, stream=cur)
            abi.csa_sparse_mqa(d["q"][lo:hi][None], self.entries, w.E, w.m, self.idx[lo:hi], w.k,
                               self.kwin[None], self.win_pos0, w.n_win, self.q_pos[lo:hi][None],
                               d["sink"], self.scale, self.out[:, lo:hi], self.lse[:, lo:hi],
                               workspace=aws, stream=cur)
            d2h.wait_event(cur.record_event())
            with torch.cuda.stream(d2h):
                host_out[:, lo:hi].copy_(self.out[:, lo:hi], non_blocking=True)
            lo = hi
        cur.wait_stream(d2h)


class HcaPrefill:
    """One causal HCA prefill of a single sequence (batch 1)."""

    launches_per_step = 2
    kind = "hca"

    def __init__(self, w, ops: Dict[str, torch.Tensor], device="cuda"):
        self.w = w
        self.d = _dev(ops, device)
        n, c, E = w.n, w.c, w.E
        self.q_pos = torch.arange(n, device=device, dtype=torch.int64)
        self.win_pos0 = torch.zeros(1, device=device, dtype=torch.int64)
        self.entries = Entries(torch.empty(E, c, device=device, dtype=DT[w.dtype]), c)
        self.out = torch.empty(1, n, w.h, c, device=device, dtype=DT[w.dtype])
        self.lse = torch.empty(1, n, w.h, device=device, dtype=torch.float32)
        self.scale = 1.0 / math.sqrt(c)

    def compress(self, stream=None):
        d, w = self.d, self.w
        abi.csa_compress_kv(d["C"], None, d["Z"], None, d["B"], None, w.m, False,
                            self.entries, stream)

    def attend(self, stream=None):
        d, w = self.d, self.w
        abi.hca_dense_mqa(d["q"][None], self.entries, w.E, w.m, d["C"][None], self.win_pos0,
                          w.n_win, self.q_pos[None], d["sink"], self.scale, self.out, self.lse,
                          stream=stream)

    def phases(self):
        return [("compress_kv", self.compress), ("attend", self.attend)]

    def inputs(self):
        return {k: v for k, v in self.d.items()}

    def result(self):
        return self.out

    def step(self, stream=None):
        for _, f in self.phases():
            f(stream)


class Decode:
    """One batched decode step over long CSA and HCA caches."""

    kind = "decode"

    @property
    def launches_per_step(self):
        """indexer + top-k (4 for long rows) + two attention calls, each with
        a combine launch when it splits the keys of each query."""
        return (1 + (4 if self.topk_ws is not None else 1) + (2 if self.ws is not None else 1)
                + (2 if self.hws is not None else 1))

    def __init__(self, w, ops: Dict[str, torch.Tensor], device="cuda"):
        self.w = w
        d = self.d = _dev(ops, device)
        B = w.batch
        self.E = d["kI"].shape[1]
        self.E_hca = d["hca_nope"].shape[1]
        self.fp4_keys = "kI_exp" in d
        if self.fp4_keys:
            self.kI = Entries(d["kI"].view(B * self.E, w.cI // 2), w.cI,
                              scale=d["kI_exp"].view(B * self.E, w.cI // 32), scale_group=32,
                              fp4=True)
        else:
            self.kI = Entries(d["kI"].view(B * self.E, w.cI), w.cI,
                              scale=d["kI_scale"].view(B * self.E), scale_group=w.cI)
        self.kv = Entries(d["kv_nope"].view(B * self.E, -1), w.c,
                          scale=d["kv_scale"].view(B * self.E, -1),
                          rope=d["kv_rope"].view(B * self.E, -1), rope_dims=w.rope_dims,
                          scale_group=w.scale_group)
        self.hkv = Entries(d["hca_nope"].view(B * self.E_hca, -1), w.c,
                           scale=d["hca_scale"].view(B * self.E_hca, -1),
                           rope=d["hca_rope"].view(B * self.E_hca, -1), rope_dims=w.rope_dims,
                           scale_group=w.scale_group)
        self.scores = torch.empty(B, 1, self.E, device=device, dtype=torch.float32)
        self.idx = torch.empty(B, w.k, device=device, dtype=torch.int32)
        self.out = torch.empty(B, 1, w.h, w.c, device=device, dtype=torch.bfloat16)
        self.lse = torch.empty(B, 1, w.h, device=device, dtype=torch.float32)
        self.hout = torch.empty_like(self.out)
        self.hlse = torch.empty_like(self.lse)
        self.scale = 1.0 / math.sqrt(w.c)
        maxk = w.k + w.n_win
        nt = abi.csa_topk_workspace_size(B, self.E, w.k)
        self.topk_ws = torch.empty(nt, device=device, dtype=torch.uint8) if nt else None
        self.ws = self._workspace(B, w, maxk, device)
        self.hws = self._workspace(B, w, self.E_hca + w.n_win, device)

    @staticmethod
    def _workspace(B, w, keys, device) -> Optional[torch.Tensor]:
        n = abi.csa_mqa_workspace_size(B, 1, w.h, w.c, keys)
        return torch.empty(max(n, 1), device=device, dtype=torch.uint8) if n else None

    def index(self, stream=None):
        d, w = self.d, self.w
        abi.csa_indexer_scores(d["qI"], d["qI_scale"], d["wI"], self.kI, d["q_pos"], w.m,
                               self.scores, self.E, stream)

    def select(self, stream=None):
        w = self.w
        abi.csa_topk(self.scores.view(w.batch, self.E), self.d["q_pos"].view(-1), w.m, w.k,
                     self.idx, self.E, workspace=self.topk_ws, stream=stream)

    def attend(self, stream=None):
        d, w = self.d, self.w
        abi.csa_sparse_mqa(d["q"], self.kv, self.E, w.m, self.idx, w.k, d["kwin"],
                           d["win_pos0"], w.n_win, d["q_pos"], d["sink"], self.scale,
                           self.out, self.lse, workspace=self.ws, stream=stream)

    def attend_hca(self, stream=None):
        d, w = self.d, self.w
        abi.hca_dense_mqa(d["q"], self.hkv, self.E_hca, w.m_hca, d["kwin"], d["win_pos0"],
                          w.n_win, d["q_pos"], d["sink"], self.scale, self.hout, self.hlse,
                          workspace=self.hws, stream=stream)

    def phases(self):
        return [("indexer", self.index), ("topk", self.select), ("attend", self.attend),
                ("attend_hca", self.attend_hca)]

    def inputs(self):
        return {k: v for k, v in self.d.items()}

    def result(self):
        return self.out

    def step(self, stream=None):
        for _, f in self.phases():
            f(stream)
