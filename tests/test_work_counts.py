"""The algorithmic counts behind the roofline fractions (work.py) against the
visits the oracle actually makes on small workloads: index scores it writes
(visible entries), selections it returns (min(k, V_t)) and window rows."""
import numpy as np

from oracle import pipeline
from long_context_sparse_07_b200 import work, workloads as W


def test_csa_counts_match_the_oracle_visits():
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=96)
    res = pipeline.csa_prefill(W.csa_operands(w), w)
    pairs = int(np.isfinite(res["scores"]).sum())          # written = visible
    sel = int((res["idx"] >= 0).sum())
    win = sum(min(w.n_win, t + 1) for t in range(w.n))
    cnt = work.csa_prefill(w)
    assert cnt["indexer"]["flops"] == 2 * pairs * w.hI * w.cI
    assert cnt["attend"]["flops"] == 4 * (sel + win) * w.h * w.c
    assert cnt["topk"]["bytes"] == pairs * 4 + w.n * w.k * 4 + w.n * 8


def test_hca_counts_match_the_oracle_visits():
    w = W.scaled(W.WORKLOADS["hca_bf16_n65536"], n=64, c=16, m=8, n_win=5, h=2, dtype="f32")
    E = w.n // w.m
    vis = sum(min(E, (t + 1) // w.m) for t in range(w.n))
    win = sum(min(w.n_win, t + 1) for t in range(w.n))
    assert work.hca_prefill(w)["attend"]["flops"] == 4 * (vis + win) * w.h * w.c


def test_decode_entry_bytes_follow_the_split_layout():
    # 448 e4m3 body bytes, 7 float32 group scales, 64 bf16 RoPE dims = 604 B
    w = W.WORKLOADS["decode_b8_ctx1m"]
    cnt = work.decode(w, 262144, 8192)
    per_seq = cnt["attend_hca"]["bytes"] / w.batch
    assert per_seq == 8192 * 604 + w.n_win * w.c * 2 + 2 * w.h * w.c * 2
