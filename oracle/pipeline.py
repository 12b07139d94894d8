"""Whole-step oracle runs (CSA prefill, HCA prefill, batched decode).

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline of the benchmark).

Chains the float64 steps of ``csa_oracle.c`` in the order of the method
(compression -> indexer -> top-k -> shared-KV attention with window and sink;
HCA: compression -> dense attention) and stores each intermediate in the
precision the path stores it in:

* compressed entries: the float64 value is rounded to float32 (the precision
  they are computed in) and then to the storage dtype (bfloat16, RNE), or
  quantised to e4m3 with per-row scales by the oracle's own quantiser;
* index scores: float32 (the selection reads float32 scores);
* selections: int32.

``rows`` restricts the quadratic steps (indexer, top-k, attention) to a
subset of query positions so that the large workloads stay affordable; the
linear compression step always runs in full.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import attend, compress, dequantize, f64, indexer, norm_rope, quantize_e4m3, topk


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to float32 and then to the storage dtype."""
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _indexer_operands(ops, rows, w):
    if w.idx_dtype == "e4m3":
        qI = dequantize(ops["qI"][rows], ops["qI_scale"][rows].reshape(-1, w.hI, 1), w.cI)
        qI = qI.reshape(len(rows), w.hI, w.cI)
    else:
        qI = f64(ops["qI"][rows])
    return qI, f64(ops["wI"][rows])


def csa_prefill(ops: Dict[str, torch.Tensor], w, rows: Optional[Sequence[int]] = None) -> dict:
    """One CSA prefill of a single sequence; queries at positions ``rows``."""
    n = w.n
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    entries = store(compress(ops["Ca"], ops["Cb"], ops["Za"], ops["Zb"], ops["Ba"], ops["Bb"],
                             w.m, True), w.dtype)
    kI64 = compress(ops["CIa"], ops["CIb"], ops["ZIa"], ops["ZIb"], ops["BIa"], ops["BIb"],
                    w.m, True)
    res = {"entries": entries}
    if w.idx_dtype == "e4m3":
        codes, scales = quantize_e4m3(kI64, w.cI)
        res["kI_codes"], res["kI_scale"] = codes, scales[:, 0]
        kI = dequantize(codes, scales, w.cI)
    else:
        kI = store(kI64, w.idx_dtype)
    res["kI"] = kI
    qI, wI = _indexer_operands(ops, rows, w)
    pos = rows.reshape(1, -1)
    sc = indexer(qI[None], wI[None], kI[None], pos, w.m)[0]
    sc32 = sc.astype(np.float32).astype(np.float64)
    res["scores"] = sc32
    sel = topk(sc32, rows, w.m, w.k)
    res["idx"] = sel
    out, lse = attend(f64(ops["q"][rows])[None], entries[None], sel, w.k, w.m,
                      f64(ops["Ca"])[None], [0], w.n_win, pos, ops["sink"],
                      1.0 / math.sqrt(w.c))
    res["out"], res["lse"], res["rows"] = out[0], lse[0], rows
    return res


def hca_prefill(ops: Dict[str, torch.Tensor], w, rows: Optional[Sequence[int]] = None) -> dict:
    """One HCA prefill (m' = w.m, no overlap); queries at positions ``rows``."""
    n = w.n
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    entries = store(compress(ops["C"], None, ops["Z"], None, ops["B"], None, w.m, False),
                    w.dtype)
    pos = rows.reshape(1, -1)
    out, lse = attend(f64(ops["q"][rows])[None], entries[None], None, 0, w.m,
                      f64(ops["C"])[None], [0], w.n_win, pos, ops["sink"],
                      1.0 / math.sqrt(w.c))
    return {"entries": entries, "out": out[0], "lse": lse[0], "rows": rows}


def split_entries(nope, scale, rope, group: int) -> np.ndarray:
    """Stored value of split-layout entries: fp8 body times its group scale,
    then the bf16 RoPE dims (Module F)."""
    body = dequantize(nope, scale, group)
    return np.concatenate([body, f64(rope)], axis=-1)


def decode(ops: Dict[str, torch.Tensor], w) -> dict:
    """One batched decode step (CSA with top-k, and HCA dense)."""
    B = w.batch
    qI = dequantize(ops["qI"], ops["qI_scale"].reshape(B, 1, w.hI, 1), w.cI)
    kI = dequantize(ops["kI"], ops["kI_scale"].reshape(B, -1, 1), w.cI)
    pos = ops["q_pos"].numpy()
    sc = indexer(qI, f64(ops["wI"]), kI, pos, w.m)
    E = kI.shape[1]
    sc32 = sc.reshape(B, E).astype(np.float32).astype(np.float64)
    sel = topk(sc32, pos.reshape(B), w.m, w.k)
    ent = split_entries(ops["kv_nope"], ops["kv_scale"], ops["kv_rope"], w.scale_group)
    scale = 1.0 / math.sqrt(w.c)
    out, lse = attend(ops["q"], ent, sel, w.k, w.m, ops["kwin"], ops["win_pos0"], w.n_win,
                      pos, ops["sink"], scale)
    hent = split_entries(ops["hca_nope"], ops["hca_scale"], ops["hca_rope"], w.scale_group)
    hout, hlse = attend(ops["q"], hent, None, 0, w.m_hca, ops["kwin"], ops["win_pos0"],
                        w.n_win, pos, ops["sink"], scale)
    return {"scores": sc32, "idx": sel, "out": out, "lse": lse, "hca_out": hout,
            "hca_lse": hlse}


def csa_prefill_rope(ops: Dict[str, torch.Tensor], w, rows: Optional[Sequence[int]] = None,
                     rope_dims: int = 64, gamma_q=None, gamma_kv=None, eps: float = 1e-6,
                     base: float = 10000.0, shift: int = 0) -> dict:
    """CSA prefill with the Q/KV RMSNorm and partial RoPE of Module D before
    the core attention, and its output rotated back by the query position:
    queries at their positions t, compressed entry i at the position of its
    last token m i + m - 1, window rows at their own positions; every
    normalised and rotated tensor is stored in the path's dtype. ``shift``
    adds a constant to every RoPE position (a test of relative positions)."""
    n = w.n
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    base_res = csa_prefill(ops, w, rows)                 # compression, indexer, top-k
    E = base_res["entries"].shape[0]
    ent = store(norm_rope(base_res["entries"], np.arange(E) * w.m + w.m - 1 + shift,
                          rope_dims, gamma_kv, True, eps, base), w.dtype)
    win = store(norm_rope(f64(ops["Ca"]), np.arange(n) + shift, rope_dims, gamma_kv, True,
                          eps, base), w.dtype)
    q = store(norm_rope(f64(ops["q"][rows]), rows + shift, rope_dims, gamma_q, True, eps,
                        base).reshape(len(rows), w.h, w.c), w.dtype)
    pos = rows.reshape(1, -1)
    out, lse = attend(q[None], ent[None], base_res["idx"], w.k, w.m, win[None], [0], w.n_win,
                      pos, ops["sink"], 1.0 / math.sqrt(w.c))
    o = norm_rope(out[0], -(rows + shift), rope_dims, None, False, eps, base)
    return {"entries": ent, "idx": base_res["idx"], "out": o, "lse": lse[0], "rows": rows,
            "q": q, "win": win}
