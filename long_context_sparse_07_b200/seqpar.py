"""One CSA prefill sequence split over several ranks (sequence parallelism).

The method itself is per sequence; what shards is the token axis:

* Compression (Eq. 9-12) is local to blocks of m tokens, except that entry i
  also reads the m rows of block i - 1 through C^b / Z^b: a rank that owns
  tokens [a, b) (a, b multiples of m) computes entries a/m .. b/m - 1 from its
  own rows plus the m rows before a (the compression halo).
* The indexer, top-k and attention of a query at position t read every
  visible compressed entry (s < V_t) and the n_win raw rows before t: after
  one all-gather of the compressed entries and the compressed indexer keys,
  a rank runs them for its own queries, with the n_win - 1 rows before each of
  its chunks as the window halo.

Balance: tokens are cut into 2P chunks of whole m-blocks and rank r owns
chunks r and 2P - 1 - r (zig-zag), so every rank gets about the same share of
the causal triangle (the indexer work of a query grows with its position).

Exchanges per prefill, all through ``torch.distributed`` (NCCL between GPUs):
one all-gather of the chunk tails (the halos), one all-gather of the entries
and indexer keys. Nothing else crosses ranks: each rank writes the outputs of
its own queries.

The per-rank steps are the five calls of the path, given as a ``backend``
object with ``compress``, ``indexer``, ``topk`` and ``attend`` methods;
``AbiBackend`` runs them through the C ABI on the rank's GPU.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import torch


def chunks(n: int, m: int, world: int) -> List[Tuple[int, int]]:
    """The 2P token chunks [a, b), each a whole number of m-blocks."""
    E = n // m
    P2 = 2 * world
    return [((E * j // P2) * m, (E * (j + 1) // P2) * m) for j in range(P2)]


def owned(world: int, rank: int) -> Tuple[int, int]:
    """The two chunk numbers of rank `rank` (zig-zag)."""
    return rank, 2 * world - 1 - rank


def halo_rows(m: int, n_win: int) -> int:
    """Rows before a chunk that its owner needs: m for the compression of
    its first entry, n_win - 1 for the windows of its first queries."""
    return max(m, n_win - 1)


def _gather_equal(t: torch.Tensor, dist, group=None) -> List[torch.Tensor]:
    """all-gather of one tensor per rank with possibly different first
    dimensions (padded to the largest, then trimmed)."""
    world = dist.get_world_size(group)
    n = torch.tensor([t.shape[0]], dtype=torch.int64, device=t.device)
    ns = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(ns, n, group=group)
    ns = [int(x.item()) for x in ns]
    mx = max(ns)
    pad = torch.zeros((mx,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[:t.shape[0]] = t
    outs = [torch.empty_like(pad) for _ in range(world)]
    # the collective moves bytes: any storage dtype (bf16, e4m3 codes) travels
    # as its raw bytes
    dist.all_gather([o.view(torch.uint8) for o in outs], pad.view(torch.uint8), group=group)
    return [o[:k] for o, k in zip(outs, ns)]


class SeqParallelCsa:
    """CSA prefill of one sequence of n tokens over the ranks of `dist`.

    ``run(ops)`` takes this rank's operand rows (see ``local_operands``) and
    returns {chunk number: (positions, out, lse, idx)} for its two chunks.
    """

    def __init__(self, w, backend, dist, group=None):
        self.w, self.be, self.dist, self.group = w, backend, dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.ch = chunks(w.n, w.m, self.world)
        self.mine = owned(self.world, self.rank)
        self.halo = halo_rows(w.m, w.n_win)

    def local_operands(self, ops: Dict[str, torch.Tensor]) -> Dict[int, Dict[str, torch.Tensor]]:
        """This rank's rows of full-sequence operands: per owned chunk, the
        token rows of C/Z (KV and indexer), q, q^I, w^I. Position biases
        and sinks are shared. (A real deployment produces these rows by its
        own projections; the slicing stands in for that.)"""
        out = {}
        for j in self.mine:
            a, b = self.ch[j]
            d = {k: ops[k][a:b] for k in ("Ca", "Cb", "Za", "Zb", "CIa", "CIb", "ZIa", "ZIb",
                                          "qI", "wI", "q") if k in ops}
            if "qI_scale" in ops:
                d["qI_scale"] = ops["qI_scale"][a:b]
            out[j] = d
        return out

    def run(self, local: Dict[int, Dict[str, torch.Tensor]], shared: Dict[str, torch.Tensor]):
        w, dist, H = self.w, self.dist, self.halo
        kv_keys = ("Ca", "Cb", "Za", "Zb", "CIa", "CIb", "ZIa", "ZIb")
        # 1. halos: every chunk's last H rows of the KV-side operands, gathered
        tails = {}
        for key in kv_keys:
            mine = torch.cat([local[j][key][-H:] if local[j][key].shape[0] >= H else
                              local[j][key] for j in self.mine])
            got = _gather_equal(mine, dist, self.group)
            for r, t in enumerate(got):
                ja, jb = owned(self.world, r)
                la = self.ch[ja][1] - self.ch[ja][0]
                na = min(la, H)
                tails[(key, ja)] = t[:na]
                tails[(key, jb)] = t[na:]

        def with_halo(key, j):
            """Rows [a - H', b) of operand `key` for chunk j (H' <= H)."""
            a, _ = self.ch[j]
            if a == 0 or j == 0:
                return local[j][key], 0
            prev = [tails[(key, i)] for i in range(j - 1, -1, -1)]
            rows, need = [], H
            for t in prev:                          # the chunk before may be short
                rows.insert(0, t[-need:] if t.shape[0] >= need else t)
                need -= rows[0].shape[0]
                if need <= 0:
                    break
            h = torch.cat(rows) if rows else local[j][key][:0]
            return torch.cat([h, local[j][key]]), h.shape[0]

        # 2. compression of the owned chunks (the first entry of a halo run is
        # a partial block and is dropped)
        ent_parts, ki_parts = {}, {}
        for j in self.mine:
            a, b = self.ch[j]
            rows = {k: with_halo(k, j) for k in kv_keys}
            for kind, names, bias in (("kv", ("Ca", "Cb", "Za", "Zb"), ("Ba", "Bb")),
                                      ("ki", ("CIa", "CIb", "ZIa", "ZIb"), ("BIa", "BIb"))):
                xs = [rows[nm][0] for nm in names]
                hl = rows[names[0]][1]
                skip = hl % w.m
                xs = [x[skip:] for x in xs]
                res = self.be.compress(kind, xs, shared[bias[0]], shared[bias[1]], w)
                drop = (hl - skip) // w.m
                res = tuple(r[drop:] if r is not None else None for r in res)
                (ent_parts if kind == "kv" else ki_parts)[j] = res
        # 3. one all-gather of the entries and the indexer keys, reassembled in
        # sequence order
        full = {}
        for name, parts in (("ent", ent_parts), ("ki", ki_parts)):
            cols = len(parts[self.mine[0]])
            gathered = []
            for ci in range(cols):
                if parts[self.mine[0]][ci] is None:
                    gathered.append(None)
                    continue
                mine = torch.cat([parts[j][ci] for j in self.mine])
                got = _gather_equal(mine, dist, self.group)
                seq = [None] * (2 * self.world)
                for r, t in enumerate(got):
                    ja, jb = owned(self.world, r)
                    na = (self.ch[ja][1] - self.ch[ja][0]) // w.m
                    seq[ja], seq[jb] = t[:na], t[na:]
                gathered.append(torch.cat(seq))
            full[name] = tuple(gathered)
        # 4. this rank's queries: indexer, top-k, attention with its window rows
        res = {}
        for j in self.mine:
            a, b = self.ch[j]
            if b <= a:
                continue
            pos = torch.arange(a, b, dtype=torch.int64, device=local[j]["q"].device)
            kwin, hl = with_halo("Ca", j)
            sc = self.be.indexer(local[j], full["ki"], pos, w)
            idx = self.be.topk(sc, pos, w)
            out, lse = self.be.attend(local[j]["q"], full["ent"], idx, kwin, a - hl, pos,
                                      shared["sink"], w)
            res[j] = (pos, out, lse, idx)
        return res


class AbiBackend:
    """The per-rank steps through the C ABI (device tensors of this rank)."""

    def __init__(self, device="cuda"):
        from . import abi
        self.abi = abi
        self.device = device

    def compress(self, kind, xs, Ba, Bb, w):
        from .abi import Entries
        Ca, Cb, Za, Zb = xs
        n = Ca.shape[0]
        E = n // w.m
        width = w.c if kind == "kv" else w.cI
        dev = Ca.device
        if kind == "ki" and w.idx_dtype == "e4m3":
            out = Entries(torch.empty(E, width, device=dev, dtype=torch.float8_e4m3fn), width,
                          scale=torch.empty(E, device=dev, dtype=torch.float32),
                          scale_group=width)
        else:
            dt = w.dtype if kind == "kv" else w.idx_dtype
            out = Entries(torch.empty(E, width, device=dev,
                                      dtype=torch.float32 if dt == "f32" else torch.bfloat16),
                          width)
        self.abi.csa_compress_kv(Ca.contiguous(), Cb.contiguous(), Za.contiguous(),
                                 Zb.contiguous(), Ba, Bb, w.m, True, out)
        return (out.body, out.scale)

    def indexer(self, loc, ki, pos, w):
        from .abi import Entries
        body, scale = ki
        E = body.shape[0]
        kI = Entries(body.contiguous(), w.cI, scale=scale.contiguous() if scale is not None
                     else None, scale_group=w.cI if scale is not None else 0)
        qs = loc.get("qI_scale")
        sc = torch.empty(1, pos.numel(), max(E, 1), device=pos.device, dtype=torch.float32)
        self.abi.csa_indexer_scores(loc["qI"].contiguous()[None],
                                    qs.contiguous()[None] if qs is not None else None,
                                    loc["wI"].contiguous()[None], kI, pos[None], w.m, sc, E)
        return sc[0]

    def topk(self, sc, pos, w):
        E = sc.shape[1]
        idx = torch.empty(pos.numel(), w.k, device=pos.device, dtype=torch.int32)
        nws = self.abi.csa_topk_workspace_size(pos.numel(), E, w.k)
        ws = torch.empty(nws, device=pos.device, dtype=torch.uint8) if nws else None
        self.abi.csa_topk(sc, pos, w.m, w.k, idx, E, workspace=ws)
        return idx

    def attend(self, q, ent, idx, kwin, win_pos0, pos, sink, w):
        from .abi import Entries
        body = ent[0]
        E = body.shape[0]
        n_q = q.shape[0]
        out = torch.empty_like(q)[None]
        lse = torch.empty(1, n_q, w.h, device=q.device, dtype=torch.float32)
        p0 = torch.tensor([win_pos0], device=q.device, dtype=torch.int64)
        nws = self.abi.csa_mqa_workspace_size(1, n_q, w.h, w.c, w.k + w.n_win)
        ws = torch.empty(nws, device=q.device, dtype=torch.uint8) if nws else None
        self.abi.csa_sparse_mqa(q.contiguous()[None], Entries(body.contiguous(), w.c), E, w.m,
                                idx, w.k, kwin.contiguous()[None], p0, w.n_win, pos[None], sink,
                                1.0 / math.sqrt(w.c), out, lse, workspace=ws)
        return out[0], lse[0]
