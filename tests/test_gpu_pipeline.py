"""End-to-end parity of the five workloads: the whole hot path on the GPU
(through the C ABI) against the oracle's own chain of steps, each side starting
from the same generated operands.

Selections: where the oracle's k-th and (k+1)-th scores are separated by more
than the score tolerance the selected set is unique and must match exactly;
elsewhere the GPU's set must be a valid top-k within that tolerance (every
chosen entry scores at least the oracle's k-th score minus the tolerance). The
share of such near-tie rows is bounded. First, the oracle's top-k over the
GPU's own float32 scores must be the GPU's selection exactly. Attention
outputs are compared with the oracle's on every row whose selection matches
the oracle's, and on every sampled row with the oracle's attention over the
GPU's own selection.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline
from long_context_sparse_07_b200 import abi, path, workloads as W
from helpers import assert_close_out, sample_rows, score_scale, to_np, SCORE_REL

pytestmark = pytest.mark.gpu


def check_selection(gpu_idx, ref_idx, ref_scores, V, k, tol, max_tie_share=0.05):
    """Returns the rows whose selection equals the oracle's."""
    same = np.zeros(len(V), dtype=bool)
    for r in range(len(V)):
        g, o = gpu_idx[r], ref_idx[r]
        if np.array_equal(g, o):
            same[r] = True
            continue
        assert V[r] > k, "row %d: short row must select everything" % r
        sel = g[g >= 0]
        assert len(sel) == k and len(np.unique(sel)) == k and sel.max() < V[r], r
        row = ref_scores[r, :V[r]]
        kth = np.sort(row)[::-1][k - 1]
        assert (row[sel] >= kth - 2 * tol[r]).all(), "row %d: invalid selection" % r
    assert (~same).mean() <= max_tie_share, "near-tie rows %.3f" % (~same).mean()
    return same


def run_csa(w, rows, seed_rows_note=""):
    ops = W.csa_operands(w)
    p = path.CsaPrefill(w, ops)
    p.step()
    abi.csa_get_error()
    ref = pipeline.csa_prefill(ops, w, rows)
    # compressed KV entries (full)
    assert_close_out(to_np(p.entries.body), ref["entries"], w.dtype, "entries")
    # indexer keys
    if w.idx_dtype == "e4m3":
        kI = oracle.dequantize(p.kI.body.cpu(), p.kI.scale.cpu().view(-1, 1), w.cI)
    else:
        kI = to_np(p.kI.body)
    np.testing.assert_allclose(kI, ref["kI"], rtol=0.13, atol=1e-2)
    # scores on the sampled rows
    qv, wv = pipeline._indexer_operands(ops, rows, w)
    S = score_scale(qv, wv, np.abs(ref["kI"]).max())
    sc = p.scores[0][torch.as_tensor(rows, device="cuda")].cpu().double().numpy()
    V = np.array([oracle.visible(t, w.m, w.E) for t in rows])
    close = []
    for r in range(len(rows)):
        d = np.abs(sc[r, :V[r]] - ref["scores"][r, :V[r]])
        assert (d <= 5e-3 * S[r] + 1e-30).all()
        close.append((d <= SCORE_REL * S[r]).mean() if V[r] else 1.0)
    assert np.mean(close) > 0.99
    gidx = p.idx[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    # selection, first level: the oracle's top-k over the GPU's own float32
    # score rows is the GPU's selection exactly (same values, same tie rule)
    np.testing.assert_array_equal(gidx, oracle.topk(sc, rows, w.m, w.k))
    # second level: against the oracle's float64 scores, differences are near ties
    same = check_selection(gidx, ref["idx"], ref["scores"], V, w.k, 5e-3 * S)
    out = p.out[0][torch.as_tensor(rows, device="cuda")]
    assert_close_out(to_np(out)[same], ref["out"][same], w.dtype, "out")
    lse = p.lse[0][torch.as_tensor(rows, device="cuda")].cpu().double().numpy()
    np.testing.assert_allclose(lse[same], ref["lse"][same], rtol=1e-3, atol=1e-3)
    # every sampled row against the oracle's attention over the GPU's own
    # selection, so that a tolerated near tie cannot hide an output error
    o2, l2 = oracle.attend(oracle.f64(ops["q"][rows])[None], ref["entries"][None], gidx, w.k,
                           w.m, oracle.f64(ops["Ca"])[None], [0], w.n_win,
                           np.asarray(rows).reshape(1, -1), ops["sink"], 1.0 / math.sqrt(w.c))
    assert_close_out(to_np(out), o2[0], w.dtype, "out (GPU selection)")
    np.testing.assert_allclose(lse, l2[0], rtol=1e-3, atol=1e-3)


def test_csa_fp32_n256_all_rows():
    w = W.WORKLOADS["csa_fp32_n256"]
    run_csa(w, np.arange(w.n))


def test_csa_bf16_n4096_sampled():
    w = W.WORKLOADS["csa_bf16_n4096"]
    run_csa(w, sample_rows(w.n, w.m, 256, 4))


def test_csa_fp8idx_n131072_sampled():
    w = W.WORKLOADS["csa_fp8idx_n131072"]
    run_csa(w, sample_rows(w.n, w.m, 48, 5))


def test_hca_bf16_n65536_sampled():
    w = W.WORKLOADS["hca_bf16_n65536"]
    ops = W.hca_operands(w)
    p = path.HcaPrefill(w, ops)
    p.step()
    abi.csa_get_error()
    rows = sample_rows(w.n, w.m, 160, 6)
    ref = pipeline.hca_prefill(ops, w, rows)
    assert_close_out(to_np(p.entries.body), ref["entries"], w.dtype, "entries")
    sel = torch.as_tensor(rows, device="cuda")
    assert_close_out(to_np(p.out[0][sel]), ref["out"], w.dtype, "out")
    np.testing.assert_allclose(p.lse[0][sel].cpu().double().numpy(), ref["lse"], rtol=1e-3,
                               atol=1e-3)


def test_decode_b8_ctx1m():
    w = W.WORKLOADS["decode_b8_ctx1m"]
    ops = W.decode_operands(w)
    p = path.Decode(w, ops)
    p.step()
    abi.csa_get_error()
    ref = pipeline.decode(ops, w)
    B = w.batch
    qv = oracle.dequantize(ops["qI"], ops["qI_scale"].reshape(B, 1, w.hI, 1), w.cI)
    kmax = np.abs(oracle.dequantize(ops["kI"], ops["kI_scale"].reshape(B, -1, 1), w.cI)).max()
    S = score_scale(qv[:, 0], oracle.f64(ops["wI"])[:, 0], kmax)
    sc = p.scores.view(B, -1).cpu().double().numpy()
    for b in range(B):
        assert (np.abs(sc[b] - ref["scores"][b]) <= SCORE_REL * S[b]).all()
    V = np.full(B, p.E)
    gidx = p.idx.cpu().numpy()
    np.testing.assert_array_equal(gidx, oracle.topk(sc, ops["q_pos"].numpy().reshape(B), w.m,
                                                    w.k))
    same = check_selection(gidx, ref["idx"], ref["scores"], V, w.k,
                           SCORE_REL * S, max_tie_share=0.5)
    assert_close_out(to_np(p.out)[same], ref["out"][same], "bf16", "csa out")
    ent = pipeline.split_entries(ops["kv_nope"], ops["kv_scale"], ops["kv_rope"], w.scale_group)
    o2, _ = oracle.attend(ops["q"], ent, gidx, w.k, w.m, ops["kwin"], ops["win_pos0"], w.n_win,
                          ops["q_pos"].numpy(), ops["sink"], 1.0 / math.sqrt(w.c))
    assert_close_out(to_np(p.out), o2, "bf16", "csa out (GPU selection)")
    assert_close_out(to_np(p.hout), ref["hca_out"], "bf16", "hca out")
    np.testing.assert_allclose(p.hlse.cpu().double().numpy(), ref["hca_lse"], rtol=1e-3)
