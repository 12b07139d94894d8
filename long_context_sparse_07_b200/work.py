"""Algorithmic work of each kernel of the path (for roofline fractions).

Counts follow the method, not the implementation: causal visibility
V_t = floor((t + 1) / m), min(k, V_t) selected entries, min(n_win, t + 1)
window rows, no padded tiles, each operand read once and each result written
once. FLOPs count a multiply-add as two.
"""
from __future__ import annotations

from typing import Dict

DT_BYTES = {"f32": 4, "bf16": 2, "e4m3": 1}


def _vis_sum(n: int, m: int, lo: int = 0) -> int:
    """sum over t in [lo, n) of floor((t + 1) / m)."""
    return sum((t + 1) // m for t in range(lo, n))


def _key_visits(n: int, m: int, k: int, n_win: int, dense: bool, lo: int = 0) -> int:
    tot = 0
    for t in range(lo, n):
        V = (t + 1) // m
        tot += (V if dense else min(k, V)) + min(n_win, t + 1)
    return tot


def csa_prefill(w, fp4_keys: bool = False, q_lo: int = 0) -> Dict[str, Dict[str, float]]:
    """Work of one CSA prefill step; with q_lo > 0, of the queries at
    positions q_lo .. n - 1 only (the entries still cover the sequence)."""
    n, c, m, E = w.n, w.c, w.m, w.E
    nq = n - q_lo
    b = DT_BYTES[w.dtype]
    bi = DT_BYTES[w.idx_dtype]
    ki_bytes = 1 if w.idx_dtype == "e4m3" else b
    pairs = _vis_sum(n, m, q_lo)
    keys = _key_visits(n, m, w.k, w.n_win, False, q_lo)
    out = {}
    out["compress_kv"] = {"bytes": 4 * n * c * b + E * c * b + 2 * m * c * 4, "flops": 0}
    # bytes of the stored indexer keys: codes + scales (FP4: half a byte per
    # channel + one exponent byte per 32 channels)
    key_row = (w.cI // 2 + w.cI // 32) if fp4_keys else \
        (w.cI * ki_bytes + (4 if w.idx_dtype == "e4m3" else 0))
    out["compress_index"] = {"bytes": 4 * n * w.cI * (4 if w.idx_dtype == "f32" else 2)
                             + E * key_row, "flops": 0}
    out["indexer"] = {"flops": 2 * pairs * w.hI * w.cI,
                      "bytes": nq * w.hI * w.cI * bi + nq * w.hI * 4 + E * key_row + pairs * 4}
    out["topk"] = {"bytes": pairs * 4 + nq * w.k * 4 + nq * 8, "flops": 0}
    # the indexer and the top-k in one call: the score rows are neither
    # written nor read back
    out["indexer_topk"] = {"flops": out["indexer"]["flops"],
                           "bytes": out["indexer"]["bytes"] - pairs * 4 + nq * w.k * 4}
    out["attend"] = {"flops": 4 * keys * w.h * c,
                     "bytes": 2 * nq * w.h * c * b + E * c * b + n * c * b + nq * w.k * 4
                     + nq * w.h * 4}
    return out


def hca_prefill(w) -> Dict[str, Dict[str, float]]:
    n, c, m, E = w.n, w.c, w.m, w.E
    b = DT_BYTES[w.dtype]
    keys = _key_visits(n, m, 0, w.n_win, True)
    return {
        "compress_kv": {"bytes": 2 * n * c * b + E * c * b + m * c * 4, "flops": 0},
        "attend": {"flops": 4 * keys * w.h * c,
                   "bytes": 2 * n * w.h * c * b + E * c * b + n * c * b + n * w.h * 4},
    }


def decode(w, E: int, E_hca: int, fp4_keys: bool = False) -> Dict[str, Dict[str, float]]:
    B, c = w.batch, w.c
    entry = (c - w.rope_dims) + 4 * ((c - w.rope_dims) // w.scale_group) + 2 * w.rope_dims
    kbytes = B * E * ((w.cI // 2 + w.cI // 32) if fp4_keys else (w.cI + 4))
    return {
        "indexer": {"flops": 2 * B * E * w.hI * w.cI,
                    "bytes": kbytes + B * w.hI * (w.cI + 8) + B * E * 4},
        "topk": {"bytes": B * E * 4 + B * w.k * 4, "flops": 0},
        "attend": {"flops": 4 * B * (w.k + w.n_win) * w.h * c,
                   "bytes": B * (w.k * (entry + 4) + w.n_win * c * 2 + 2 * w.h * c * 2)},
        "attend_hca": {"flops": 4 * B * (E_hca + w.n_win) * w.h * c,
                       "bytes": B * (E_hca * entry + w.n_win * c * 2 + 2 * w.h * c * 2)},
    }
