"""Seeded synthetic operands for the CSA / HCA path.

This module only draws numbers. It computes no step of the method: no
projection, no compression, no score, no selection, no attention and no
quantisation rule. Every tensor is drawn from numpy's PCG64 generator, keyed by
``(seed, tensor id, row chunk)``, so any subset of rows can be drawn again
with identical bits, on any machine, without drawing the rest.

Projections are dense GEMMs that sit before the path (DeepSeek-V4 technical
report restatements, "Compressed Sparse Attention", Eq. 9-10, 13-15 and 18).
They are not drawn as ``H @ W``: their outputs are drawn directly from the
normal law that ``H ~ N(0, 1)`` and ``W ~ N(0, sigma_w^2)`` give them, i.e.
``N(0, fan_in * sigma_w^2)``. The standard deviations of each workload follow
from its description (hidden size, low-rank query width, weight law).

Storage casts: float32 -> bfloat16 is round-to-nearest-even (torch). The 8-bit
operands that arrive already quantised (indexer queries, the decode cache) are
drawn as e4m3 codes of ``N(0, 64^2)`` values clipped to +-448, each row with a
positive float32 scale ``std/64 * (1 + u/4)``, ``u ~ U(0, 1)``; this is an
input encoding, not the path's own quantisation rule.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, Optional

import numpy as np
import torch

ROW_CHUNK = 4096          # rows drawn per generator stream
E4M3_MAX = 448.0
CODE_STD = 64.0           # spread of drawn e4m3 codes

# Stable stream ids, one per named operand. Never renumber: stored fixtures
# and cached inputs depend on them.
_TENSOR_IDS = {
    "Ca": 1, "Cb": 2, "Za": 3, "Zb": 4, "Ba": 5, "Bb": 6,
    "CIa": 7, "CIb": 8, "ZIa": 9, "ZIb": 10, "BIa": 11, "BIb": 12,
    "qI": 13, "qI_scale": 14, "wI": 15, "q": 16, "sink": 17,
    "C": 18, "Z": 19, "B": 20,
    "kv_nope": 21, "kv_scale": 22, "kv_rope": 23, "kI": 24, "kI_scale": 25,
    "kwin": 26, "hca_nope": 27, "hca_scale": 28, "hca_rope": 29,
    "scores": 30, "idx_u": 31, "entries": 32, "kwin_step": 33,
    "kI_fp4": 34, "kI_exp": 35,
    "H": 40, "W_aKV": 41, "W_bKV": 42, "W_aZ": 43, "W_bZ": 44, "W_aKI": 45, "W_bKI": 46,
    "W_aZI": 47, "W_bZI": 48, "W_DQ": 49, "W_IUQ": 50, "W_w": 51, "W_UQ": 52,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload. Sizes follow the pages' notation.

    n: tokens (prefill) or context length (decode); c: compressed head dim;
    m: compression ratio (m' for HCA); hI, cI: indexer heads and head dim;
    k: top-k; n_win: sliding-window length; h: query heads sharing one KV
    head; dtype: KV / query / output storage; idx_dtype: indexer operands.
    """
    name: str
    kind: str                 # "csa", "hca" or "decode"
    n: int
    c: int
    m: int
    hI: int
    cI: int
    k: int
    n_win: int
    h: int
    dtype: str                # "f32" or "bf16"
    idx_dtype: str            # "f32", "bf16" or "e4m3"
    seed: int
    std_proj: float           # KV-side projections C, Z (and indexer C^I, Z^I)
    std_bias: float           # position biases B^a, B^b (B for HCA)
    std_q: float              # queries q and indexer queries q^I
    std_w: float              # indexer head weights w^I
    batch: int = 1
    m_hca: int = 128          # HCA ratio for the decode workload
    rope_dims: int = 0        # decode cache: trailing dims stored as bf16
    scale_group: int = 0      # decode cache: channels per fp8 scale

    @property
    def E(self) -> int:
        return self.n // self.m


def _std(fan_in: int, var_w: float, var_in: float = 1.0) -> float:
    return math.sqrt(fan_in * var_w * var_in)


# Standard deviations of projected operands, derived from each description:
#   CSA fp32:  d=128, W ~ N(0, 1/fan_in)  -> projections N(0, 1)
#   CSA bf16:  d=2048, W ~ N(0, 0.02^2)   -> C, Z, w^I: sqrt(2048*4e-4);
#              q^I, q from a rank-256 latent: sqrt(256 * 0.8192 * 4e-4)
#   HCA / large CSA: d=4096, latent width 1024 (Flash configuration)
_S2 = _std(2048, 4e-4)
_S2Q = _std(256, 4e-4, _S2 ** 2)
_S4 = _std(4096, 4e-4)
_S4Q = _std(1024, 4e-4, _S4 ** 2)

WORKLOADS: Dict[str, Workload] = {
    "csa_fp32_n256": Workload(
        "csa_fp32_n256", "csa", n=256, c=64, m=4, hI=4, cI=32, k=8, n_win=16,
        h=4, dtype="f32", idx_dtype="f32", seed=0, std_proj=1.0,
        std_bias=math.sqrt(1.0 / 128), std_q=1.0, std_w=1.0),
    "csa_bf16_n4096": Workload(
        "csa_bf16_n4096", "csa", n=4096, c=512, m=4, hI=16, cI=128, k=256,
        n_win=128, h=32, dtype="bf16", idx_dtype="bf16", seed=1,
        std_proj=_S2, std_bias=0.02, std_q=_S2Q, std_w=_S2),
    "hca_bf16_n65536": Workload(
        "hca_bf16_n65536", "hca", n=65536, c=512, m=128, hI=0, cI=0, k=0,
        n_win=128, h=64, dtype="bf16", idx_dtype="bf16", seed=2,
        std_proj=_S4, std_bias=0.02, std_q=_S4Q, std_w=0.0),
    "csa_fp8idx_n131072": Workload(
        "csa_fp8idx_n131072", "csa", n=131072, c=512, m=4, hI=64, cI=128,
        k=1024, n_win=128, h=64, dtype="bf16", idx_dtype="e4m3", seed=3,
        std_proj=_S4, std_bias=0.02, std_q=_S4Q, std_w=_S4),
    "decode_b8_ctx1m": Workload(
        "decode_b8_ctx1m", "decode", n=1 << 20, c=512, m=4, hI=64, cI=128,
        k=1024, n_win=128, h=64, dtype="bf16", idx_dtype="e4m3", seed=4,
        std_proj=1.0, std_bias=0.0, std_q=1.0, std_w=1.0, batch=8,
        m_hca=128, rope_dims=64, scale_group=64),
}


@dataclasses.dataclass(frozen=True)
class Layer:
    """Hidden size d and query latent width d_c of a workload's layer, and the
    law of its weights: std_w (None: 1/sqrt(fan_in)) and of its biases."""
    d: int
    dc: int
    std_w: Optional[float]
    std_bias: float


# The whole-layer form of the two small CSA workloads: the operands of the
# path are projections of a hidden state H ~ N(0, 1) (the 256-token fp32 case:
# d = 128, weights N(0, 1/fan_in), no low-rank query stated, so the latent is
# full width d_c = d; the 4096-token bf16 case: d = 2048, low-rank query of
# rank 256, weights and biases N(0, 0.02^2)).
LAYERS: Dict[str, Layer] = {
    "csa_fp32_n256": Layer(d=128, dc=128, std_w=None, std_bias=math.sqrt(1.0 / 128)),
    "csa_bf16_n4096": Layer(d=2048, dc=256, std_w=0.02, std_bias=0.02),
}


def layer_draws(w: Workload, layer: Optional[Layer] = None) -> Dict[str, np.ndarray]:
    """Hidden state and weights of one CSA layer (float32 draws, no arithmetic
    of the method): H [n, d]; KV compressor W_aKV, W_bKV, W_aZ, W_bZ [d, c]
    and biases Ba, Bb [m, c]; indexer-key compressor W_aKI, W_bKI, W_aZI,
    W_bZI [d, cI] and BIa, BIb [m, cI]; query latent W_DQ [d, dc]; indexer
    query W_IUQ [dc, hI * cI] and head weights W_w [d, hI]; attention query
    W_UQ [dc, h * c]; sink [h]."""
    L = LAYERS[w.name.split("@")[0]] if layer is None else layer
    s, d, dc = w.seed, L.d, L.dc

    def wstd(fan_in):
        return L.std_w if L.std_w is not None else math.sqrt(1.0 / fan_in)

    out = {"H": normal(s, "H", w.n, d, 1.0)}
    for nm in ("W_aKV", "W_bKV", "W_aZ", "W_bZ"):
        out[nm] = normal(s, nm, d, w.c, wstd(d))
    for nm in ("W_aKI", "W_bKI", "W_aZI", "W_bZI"):
        out[nm] = normal(s, nm, d, w.cI, wstd(d))
    out["W_DQ"] = normal(s, "W_DQ", d, dc, wstd(d))
    out["W_IUQ"] = normal(s, "W_IUQ", dc, w.hI * w.cI, wstd(dc))
    out["W_w"] = normal(s, "W_w", d, w.hI, wstd(d))
    out["W_UQ"] = normal(s, "W_UQ", dc, w.h * w.c, wstd(dc))
    for nm in ("Ba", "Bb"):
        out[nm] = normal(s, nm, w.m, w.c, L.std_bias)
    for nm in ("BIa", "BIb"):
        out[nm] = normal(s, nm, w.m, w.cI, L.std_bias)
    out["sink"] = normal(s, "sink", 1, w.h, 1.0).reshape(w.h)
    return out


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some sizes changed (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


# ----------------------------------------------------------------------------
# generator streams


def _gen(seed: int, tid: int, chunk: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(tid, chunk))
    return np.random.Generator(np.random.PCG64(ss))


_POOL: Optional[ThreadPoolExecutor] = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))
    return _POOL


def _rows(seed: int, name: str, rows: int, cols: int, draw, lo: int = 0,
          hi: Optional[int] = None, dtype=np.float32, out=None):
    """Rows [lo, hi) of a [rows, cols] array drawn chunk by chunk. Chunks are
    independent streams, so they are drawn on a thread pool (numpy's
    generators release the GIL); the values do not depend on the pool.
    With ``out`` (a torch tensor [hi - lo, cols]) each drawn chunk is cast
    into it (RNE, element by element) instead of returning float32 rows."""
    hi = rows if hi is None else hi
    tid = _TENSOR_IDS[name]
    if out is None:
        out = np.empty((hi - lo, cols), dtype=dtype)
    c0 = lo // ROW_CHUNK
    c1 = (hi + ROW_CHUNK - 1) // ROW_CHUNK

    def one(ch):
        r0 = ch * ROW_CHUNK
        r1 = min(rows, r0 + ROW_CHUNK)
        block = draw(_gen(seed, tid, ch), (r1 - r0, cols))
        a = max(lo, r0)
        b = min(hi, r1)
        if isinstance(out, torch.Tensor):
            out[a - lo:b - lo] = torch.from_numpy(block[a - r0:b - r0]).to(out.dtype)
        else:
            out[a - lo:b - lo] = block[a - r0:b - r0]

    if c1 - c0 > 1:
        list(_pool().map(one, range(c0, c1)))
    else:
        for ch in range(c0, c1):
            one(ch)
    return out


def normal(seed, name, rows, cols, std, lo=0, hi=None) -> np.ndarray:
    def draw(g, shape):
        return (g.standard_normal(shape, dtype=np.float32) * np.float32(std))
    return _rows(seed, name, rows, cols, draw, lo, hi)


def normal_as(seed, name, rows, cols, std, dtype: str, lo=0, hi=None) -> torch.Tensor:
    """``to_storage(normal(...), dtype)`` with the cast done chunk by chunk
    (same bits, without the whole float32 array in host memory)."""
    hi = rows if hi is None else hi
    out = torch.empty((hi - lo, cols), dtype={"f32": torch.float32, "bf16": torch.bfloat16}[dtype])

    def draw(g, shape):
        return (g.standard_normal(shape, dtype=np.float32) * np.float32(std))
    _rows(seed, name, rows, cols, draw, lo, hi, out=out)
    return out


def uniform(seed, name, rows, cols, lo=0, hi=None) -> np.ndarray:
    def draw(g, shape):
        return g.random(shape, dtype=np.float32)
    return _rows(seed, name, rows, cols, draw, lo, hi)


def bytes_in(seed, name, rows, cols, lo_val, hi_val, lo=0, hi=None) -> torch.Tensor:
    """Drawn uint8 values, uniform in [lo_val, hi_val]."""
    def draw(g, shape):
        return g.integers(lo_val, hi_val + 1, size=shape, dtype=np.uint8)
    return torch.from_numpy(_rows(seed, name, rows, cols, draw, lo, hi, dtype=np.uint8))


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Cast drawn float32 values to a storage dtype ("f32" or "bf16")."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "f32":
        return t.clone()
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    raise ValueError(dtype)


def e4m3_codes(seed, name, rows, cols, lo=0, hi=None) -> torch.Tensor:
    """Drawn e4m3 codes (clipped N(0, 64^2) values cast by torch, RNE)."""
    x = normal(seed, name, rows, cols, CODE_STD, lo, hi)
    np.clip(x, -E4M3_MAX, E4M3_MAX, out=x)
    return torch.from_numpy(x).to(torch.float8_e4m3fn)


def e4m3_scales(seed, name, rows, cols, std, lo=0, hi=None) -> torch.Tensor:
    u = uniform(seed, name, rows, cols, lo, hi)
    return torch.from_numpy((np.float32(std / CODE_STD) * (1 + u / 4)).astype(np.float32))


# ----------------------------------------------------------------------------
# operand sets


def csa_operands(w: Workload, lo: int = 0, hi: Optional[int] = None,
                 parts: Iterable[str] = ("kv", "indexer", "query")) -> Dict[str, torch.Tensor]:
    """Operands of one CSA prefill over tokens [lo, hi) of the sequence.

    kv: Ca, Cb, Za, Zb [n, c] and Ba, Bb [m, c] (float32) -- compression of the
        KV entries; Ca doubles as the raw sliding-window KV.
    indexer: CIa, CIb, ZIa, ZIb [n, cI], BIa, BIb [m, cI] -- the indexer-key
        compressor; qI [n, hI, cI] (+ qI_scale [n, hI] for e4m3), wI [n, hI].
    query: q [n, h, c] and sink [h].
    """
    n, s = w.n, w.seed
    hi = n if hi is None else hi
    out: Dict[str, torch.Tensor] = {}
    parts = set(parts)
    if "kv" in parts:
        for nm in ("Ca", "Cb", "Za", "Zb"):
            out[nm] = to_storage(normal(s, nm, n, w.c, w.std_proj, lo, hi), w.dtype)
        for nm in ("Ba", "Bb"):
            out[nm] = to_storage(normal(s, nm, w.m, w.c, w.std_bias), "f32")
    if "indexer" in parts and w.hI:
        ik = "f32" if w.idx_dtype == "f32" else "bf16"
        for nm in ("CIa", "CIb", "ZIa", "ZIb"):
            out[nm] = to_storage(normal(s, nm, n, w.cI, w.std_proj, lo, hi), ik)
        for nm in ("BIa", "BIb"):
            out[nm] = to_storage(normal(s, nm, w.m, w.cI, w.std_bias), "f32")
        if w.idx_dtype == "e4m3":
            out["qI"] = e4m3_codes(s, "qI", n, w.hI * w.cI, lo, hi).view(hi - lo, w.hI, w.cI)
            out["qI_scale"] = e4m3_scales(s, "qI_scale", n, w.hI, w.std_q, lo, hi)
        else:
            out["qI"] = to_storage(normal(s, "qI", n, w.hI * w.cI, w.std_q, lo, hi),
                                   w.idx_dtype).view(hi - lo, w.hI, w.cI)
        out["wI"] = to_storage(normal(s, "wI", n, w.hI, w.std_w, lo, hi), "f32")
    if "query" in parts:
        out["q"] = normal_as(s, "q", n, w.h * w.c, w.std_q, w.dtype, lo,
                             hi).view(hi - lo, w.h, w.c)
        out["sink"] = to_storage(normal(s, "sink", 1, w.h, 1.0), "f32").view(w.h)
    return out


def hca_operands(w: Workload, lo: int = 0, hi: Optional[int] = None,
                 parts: Iterable[str] = ("kv", "query")) -> Dict[str, torch.Tensor]:
    """Operands of one HCA prefill: C, Z [n, c], B [m', c]; q [n, h, c], sink [h].
    C doubles as the raw sliding-window KV."""
    n, s = w.n, w.seed
    hi = n if hi is None else hi
    out: Dict[str, torch.Tensor] = {}
    parts = set(parts)
    if "kv" in parts:
        out["C"] = to_storage(normal(s, "C", n, w.c, w.std_proj, lo, hi), w.dtype)
        out["Z"] = to_storage(normal(s, "Z", n, w.c, w.std_proj, lo, hi), w.dtype)
        out["B"] = to_storage(normal(s, "B", w.m, w.c, w.std_bias), "f32")
    if "query" in parts:
        out["q"] = normal_as(s, "q", n, w.h * w.c, w.std_q, w.dtype, lo,
                             hi).view(hi - lo, w.h, w.c)
        out["sink"] = to_storage(normal(s, "sink", 1, w.h, 1.0), "f32").view(w.h)
    return out


def decode_operands(w: Workload, E: Optional[int] = None,
                    E_hca: Optional[int] = None, fp4_keys: bool = False) -> Dict[str, torch.Tensor]:
    """Operands of one batched decode step.

    Every sequence b holds a context of ``n`` tokens and one query at position
    n - 1. CSA cache: kv_nope [B, E, c - rope] e4m3, kv_scale [B, E, groups]
    fp32, kv_rope [B, E, rope] bf16; kI [B, E, cI] e4m3, kI_scale [B, E].
    HCA cache: hca_nope / hca_scale / hca_rope with E_hca entries. Queries:
    qI [B, 1, hI, cI] e4m3, qI_scale [B, 1, hI], wI [B, 1, hI], q [B, 1, h, c]
    bf16, kwin [B, n_win, c] bf16 holding positions n - n_win .. n - 1, sink
    [h]; q_pos [B, 1] and win_pos0 [B] (int64). With fp4_keys the indexer
    keys are FP4 instead: kI [B, E, cI / 2] uniform packed e2m1 code bytes,
    kI_exp [B, E, cI / 32] block exponents uniform in 118..126 (a span of 8).
    """
    B, s = w.batch, w.seed
    E = w.n // w.m if E is None else E
    E_hca = w.n // w.m_hca if E_hca is None else E_hca
    nope = w.c - w.rope_dims
    G = nope // w.scale_group
    out: Dict[str, torch.Tensor] = {}
    for pre, En in (("kv", E), ("hca", E_hca)):
        out[pre + "_nope"] = e4m3_codes(s, pre + "_nope", B * En, nope).view(B, En, nope)
        out[pre + "_scale"] = e4m3_scales(s, pre + "_scale", B * En, G,
                                          w.std_proj).view(B, En, G)
        out[pre + "_rope"] = to_storage(normal(s, pre + "_rope", B * En, w.rope_dims,
                                               w.std_proj), "bf16").view(B, En, w.rope_dims)
    if fp4_keys:
        out["kI"] = bytes_in(s, "kI_fp4", B * E, w.cI // 2, 0, 255).view(B, E, w.cI // 2)
        out["kI_exp"] = bytes_in(s, "kI_exp", B * E, w.cI // 32, 118, 126).view(B, E, w.cI // 32)
    else:
        out["kI"] = e4m3_codes(s, "kI", B * E, w.cI).view(B, E, w.cI)
        out["kI_scale"] = e4m3_scales(s, "kI_scale", B * E, 1, w.std_proj).view(B, E)
    out["qI"] = e4m3_codes(s, "qI", B, w.hI * w.cI).view(B, 1, w.hI, w.cI)
    out["qI_scale"] = e4m3_scales(s, "qI_scale", B, w.hI, w.std_q).view(B, 1, w.hI)
    out["wI"] = to_storage(normal(s, "wI", B, w.hI, w.std_w), "f32").view(B, 1, w.hI)
    out["q"] = to_storage(normal(s, "q", B, w.h * w.c, w.std_q), "bf16").view(B, 1, w.h, w.c)
    out["kwin"] = to_storage(normal(s, "kwin", B * w.n_win, w.c, w.std_proj),
                             "bf16").view(B, w.n_win, w.c)
    out["sink"] = to_storage(normal(s, "sink", 1, w.h, 1.0), "f32").view(w.h)
    out["q_pos"] = torch.full((B, 1), w.n - 1, dtype=torch.int64)
    out["win_pos0"] = torch.full((B,), w.n - w.n_win, dtype=torch.int64)
    return out


# ----------------------------------------------------------------------------
# operands for single-step parity cases


def score_rows(seed: int, rows: int, E: int, tie_frac: float = 0.25) -> torch.Tensor:
    """float32 score rows [rows, E] for the top-k step.

    A fraction of each row is snapped to a coarse grid so that exact ties
    occur (the tie rule is part of what is checked); some values are zero,
    some negative, and a few are -0.0.
    """
    x = normal(seed, "scores", rows, E, 1.0)
    u = uniform(seed, "idx_u", rows, E)
    snap = u < tie_frac
    x[snap] = np.round(x[snap] * 4) / 4
    x[(u > 0.97)] = 0.0
    x[(u > 0.985)] = -0.0
    return torch.from_numpy(x)


def stratified_idx(seed: int, rows: int, k: int, visible: np.ndarray) -> torch.Tensor:
    """Selection lists [rows, k] int32: for each row, min(k, V) distinct
    ascending indices below V (one per stratum of V/k), then -1 padding."""
    visible = np.asarray(visible, dtype=np.int64)
    u = uniform(seed, "idx_u", rows, max(k, 1))[:, :k].astype(np.float64)
    j = np.arange(k, dtype=np.int64)[None, :]
    V = visible[:, None]
    lo = (j * V) // max(k, 1)                 # stratum j is [lo, hi): disjoint,
    hi = ((j + 1) * V) // max(k, 1)           # non-empty when V >= k
    pick = lo + np.floor(u * (hi - lo)).astype(np.int64)
    out = np.where(V > k, pick, np.where(j < V, j, -1))
    return torch.from_numpy(out.astype(np.int32))
