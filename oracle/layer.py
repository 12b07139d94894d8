"""Whole-layer oracle of the small CSA workloads: from the hidden state H.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).

The path's operands are projections of H ("DeepSeek-V4: Towards Highly
Efficient Million-Token Context Intelligence", Module B steps 1-3: Eq. 9-10
for the KV compressor, Eq. 13-15 for the indexer queries, head weights and
the indexer-key compressor, Eq. 18 for the attention queries):

    C^a = H W^{aKV},  C^b = H W^{bKV},  Z^a = H W^{aZ},  Z^b = H W^{bZ}
    (and the same with the indexer-key compressor's weights, width c_I)
    c^Q = H W^{DQ},   q^I = c^Q W^{IUQ},  w^I = H W^w,  q = c^Q W^{UQ}

computed here in float64 (numpy matmul), each rounded to float32 and then to
the workload's storage dtype, after which the oracle's chain of steps
(``pipeline.csa_prefill``) runs on them. Because C^a..Z^b share H and q, q^I
share c^Q, these operands carry the correlations a real layer has, which the
directly drawn operands of the other workloads do not.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import pipeline


def project(draws: Dict[str, np.ndarray], w) -> Dict[str, np.ndarray]:
    """float64 projections of H (shapes as the path takes them)."""
    d = {k: np.asarray(v, dtype=np.float64) for k, v in draws.items()}
    H = d["H"]
    n = H.shape[0]
    out = {}
    for a, b in (("Ca", "W_aKV"), ("Cb", "W_bKV"), ("Za", "W_aZ"), ("Zb", "W_bZ"),
                 ("CIa", "W_aKI"), ("CIb", "W_bKI"), ("ZIa", "W_aZI"), ("ZIb", "W_bZI")):
        out[a] = H @ d[b]
    cQ = H @ d["W_DQ"]
    out["qI"] = (cQ @ d["W_IUQ"]).reshape(n, w.hI, w.cI)
    out["wI"] = H @ d["W_w"]
    out["q"] = (cQ @ d["W_UQ"]).reshape(n, w.h, w.c)
    return out


def _store(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def layer_operands(draws: Dict[str, np.ndarray], w) -> Dict[str, torch.Tensor]:
    """The path's operands from H, in storage dtypes (the keys of
    ``workloads.csa_operands``): projections in the workload's dtype (the
    indexer's in its indexer dtype, bf16 or f32); biases, head weights and
    the sink in float32."""
    if w.idx_dtype not in ("f32", "bf16"):
        raise ValueError("whole-layer operands are defined for f32 / bf16 indexers")
    P = project(draws, w)
    ops = {}
    for k in ("Ca", "Cb", "Za", "Zb", "q"):
        ops[k] = _store(P[k], w.dtype)
    for k in ("CIa", "CIb", "ZIa", "ZIb", "qI"):
        ops[k] = _store(P[k], w.idx_dtype)
    ops["wI"] = _store(P["wI"], "f32")
    for k in ("Ba", "Bb", "BIa", "BIb", "sink"):
        ops[k] = torch.from_numpy(np.ascontiguousarray(draws[k], dtype=np.float32))
    return ops


def csa_layer(draws: Dict[str, np.ndarray], w, rows: Optional[Sequence[int]] = None) -> dict:
    """The whole CSA layer from H: projections, then the oracle's chain."""
    ops = layer_operands(draws, w)
    res = pipeline.csa_prefill(ops, w, rows)
    res["ops"] = ops
    return res
