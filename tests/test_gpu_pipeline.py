"""End-to-end parity of the five workloads: the whole hot path on the GPU
(through the C ABI) against the oracle's own chain of steps, each side starting
from the same generated operands.

Scores: the oracle's indexer over the GPU's own indexer keys must match every
visible GPU score to SCORE_REL of the row scale (only the accumulation order
differs); against the oracle's own keys (which may sit one storage code away)
a looser bound holds. Selections, first level: the oracle's top-k over the
GPU's own float32 scores must be the GPU's selection exactly. Second level:
against the oracle's float64 scores, every entry the two sides disagree on
must sit at the selection boundary, within twice the row's measured score
error of the k-th score (or 1e-6 of it); the gaps are printed. Attention
outputs are compared with the oracle's on every row whose selection matches
the oracle's chain, and on every sampled row with the oracle's attention over
the GPU's own selection.
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


def check_selection(gpu_idx, ref_idx, ref_scores, gpu_scores, V, k, what):
    """Second-level selection check against the oracle's float64 scores.

    Returns the rows whose selection equals the oracle's. On a row that
    differs, every entry the two sides disagree on must sit at the selection
    boundary: its float64 score lies within `band` of the oracle's k-th
    score, band = max(1e-6 |kth|, 2 err), err = the row's largest
    |GPU score - float64 score| over its visible entries (the GPU selects
    exactly on its own scores, checked at the first level, so a swap needs a
    gap no larger than twice the score error). The relative gap of each
    differing row is printed."""
    same = np.zeros(len(V), dtype=bool)
    for r in range(len(V)):
        g, o = gpu_idx[r], ref_idx[r]
        if np.array_equal(g, o):
            same[r] = True
            continue
        assert V[r] > k, "%s row %d: short row must select everything" % (what, r)
        sel = g[g >= 0]
        assert len(sel) == k and len(np.unique(sel)) == k and sel.max() < V[r], r
        row = ref_scores[r, :V[r]]
        kth = np.sort(row)[::-1][k - 1]
        err = np.abs(gpu_scores[r, :V[r]] - row).max()
        diff = np.setxor1d(sel, o[o >= 0])
        gap = np.abs(row[diff] - kth).max()
        band = max(1e-6 * abs(kth), 2 * err)
        print("%s row %d: %d entries swapped at the boundary; max |score - kth| = %.3g "
              "(%.3g of |kth|), row score error %.3g (%.3g of |kth|)"
              % (what, r, len(diff) // 2, gap, gap / abs(kth), err, err / abs(kth)))
        assert gap <= band, "%s row %d: swap beyond the score error" % (what, r)
    print("%s: %d of %d rows select exactly the oracle's set" % (what, same.sum(), len(V)))
    return same


def run_csa(w, rows, ops=None, ref=None):
    """GPU path on `ops` (default: the workload's drawn operands) against the
    oracle's chain `ref` (default: the chain over the same operands)."""
    ops = W.csa_operands(w) if ops is None else ops
    p = path.CsaPrefill(w, ops)
    p.step()
    abi.csa_get_error()
    ref = pipeline.csa_prefill(ops, w, rows) if ref is None else ref
    # compressed KV entries (full)
    assert_close_out(to_np(p.entries.body), ref["entries"], w.dtype, "entries")
    # indexer keys: the GPU's float32 compressor output may round to the
    # neighbouring bf16 value or e4m3 code of the oracle's (one e4m3 code is
    # up to 2^-3 relative, hence the loose relative bound here)
    if w.idx_dtype == "e4m3":
        kI = oracle.dequantize(p.kI.body.cpu(), p.kI.scale.cpu().view(-1, 1), w.cI)
    else:
        kI = to_np(p.kI.body)
    np.testing.assert_allclose(kI, ref["kI"], rtol=0.13, atol=1e-2)
    qv, wv = pipeline._indexer_operands(ops, rows, w)
    sel_rows = torch.as_tensor(rows, device="cuda")
    sc = p.scores[0][sel_rows].cpu().double().numpy()
    V = np.array([oracle.visible(t, w.m, w.E) for t in rows])
    pos = np.asarray(rows).reshape(1, -1)
    # scores on exactly the GPU's inputs: the oracle's indexer over the GPU's
    # own keys; only the float32 accumulation order differs, so every visible
    # score is held to SCORE_REL * S_t
    own = oracle.indexer(qv[None], wv[None], kI[None], pos, w.m)[0]
    S = score_scale(qv, wv, np.abs(kI).max())
    worst = 0.0
    for r in range(len(rows)):
        if not V[r]:
            continue
        d = np.abs(sc[r, :V[r]] - own[r, :V[r]])
        worst = max(worst, d.max() / S[r])
        assert (d <= SCORE_REL * S[r] + 1e-30).all(), "row %d: score error %.3g S_t" % (
            r, d.max() / S[r])
    print("%s: largest score error over the GPU's own keys %.3g S_t" % (w.name, worst))
    # scores against the oracle's whole chain (its own keys): a key one
    # storage code away moves a score by at most sum_h |w| |qI_h . dk|, which
    # stays under 5e-3 S_t for these operand laws
    Sref = score_scale(qv, wv, np.abs(ref["kI"]).max())
    for r in range(len(rows)):
        d = np.abs(sc[r, :V[r]] - ref["scores"][r, :V[r]])
        assert (d <= 5e-3 * Sref[r] + 1e-30).all()
    gidx = p.idx[sel_rows].cpu().numpy()
    # selection, first level: the oracle's top-k over the GPU's own float32
    # score rows is the GPU's selection exactly (same values, same tie rule)
    np.testing.assert_array_equal(gidx, oracle.topk(sc, rows, w.m, w.k))
    # the indexer and the top-k in one call select exactly the same, on
    # every row (both select on the same float32 scores)
    qs = p.d.get("qI_scale")
    nws = abi.csa_indexer_topk_workspace_size(1, w.n, w.E, w.hI, w.cI, w.k, p.d["qI"])
    fws = torch.empty(nws, device="cuda", dtype=torch.uint8) if nws else None
    fidx = torch.full_like(p.idx, -7)
    abi.csa_indexer_topk(p.d["qI"][None], qs[None] if qs is not None else None, p.d["wI"][None],
                         p.kI, p.q_pos[None], w.m, w.k, fidx, w.E, workspace=fws)
    abi.csa_get_error()
    del fws
    nbad = int((fidx != p.idx).any(1).sum())
    assert nbad == 0, "%d rows of csa_indexer_topk differ from the two calls" % nbad
    # second level, on the GPU's keys: the oracle's float64 selection over the
    # same keys differs only at the boundary, within the score error
    own_idx = oracle.topk(own.astype(np.float32).astype(np.float64), rows, w.m, w.k)
    check_selection(gidx, own_idx, own, sc, V, w.k, w.name + " (GPU keys)")
    # against the oracle's whole chain: rows with the same selection compare
    # outputs directly
    same = np.array([np.array_equal(gidx[r], ref["idx"][r]) for r in range(len(rows))])
    print("%s: %d of %d rows select the oracle chain's set" % (w.name, same.sum(), len(rows)))
    out = p.out[0][sel_rows]
    assert_close_out(to_np(out)[same], ref["out"][same], w.dtype, "out")
    lse = p.lse[0][sel_rows].cpu().double().numpy()
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
    run_csa(w, sample_rows(w.n, w.m, 512, 5))


def harness_projections(draws, w):
    """The projections before the path (Eq. 9-10, 13-15, 18), computed on the
    test harness's side with float64 torch matmuls on the GPU, rounded to
    float32 and then to the storage dtype: the same definition the oracle's
    layer computes with numpy, done independently."""
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev, torch.float64)
         for k, v in draws.items()}
    H = t["H"]
    n = H.shape[0]

    def store(x, dt):
        x = x.to(torch.float32)
        return (x.to(torch.bfloat16) if dt == "bf16" else x).cpu()

    ops = {}
    for a, b in (("Ca", "W_aKV"), ("Cb", "W_bKV"), ("Za", "W_aZ"), ("Zb", "W_bZ")):
        ops[a] = store(H @ t[b], w.dtype)
    for a, b in (("CIa", "W_aKI"), ("CIb", "W_bKI"), ("ZIa", "W_aZI"), ("ZIb", "W_bZI")):
        ops[a] = store(H @ t[b], w.idx_dtype)
    cQ = H @ t["W_DQ"]
    ops["qI"] = store(cQ @ t["W_IUQ"], w.idx_dtype).view(n, w.hI, w.cI)
    ops["wI"] = store(H @ t["W_w"], "f32")
    ops["q"] = store(cQ @ t["W_UQ"], w.dtype).view(n, w.h, w.c)
    for k in ("Ba", "Bb", "BIa", "BIb", "sink"):
        ops[k] = torch.from_numpy(np.ascontiguousarray(draws[k], dtype=np.float32))
    return ops


@pytest.mark.parametrize("name,count", [("csa_fp32_n256", None), ("csa_bf16_n4096", 256)])
def test_whole_layer_from_hidden_state(name, count):
    """The path on operands projected from one hidden state H (correlated as
    in a real layer) against the oracle's whole layer from the same H."""
    from oracle import layer
    w = W.WORKLOADS[name]
    draws = W.layer_draws(w)
    ops = harness_projections(draws, w)
    rows = np.arange(w.n) if count is None else sample_rows(w.n, w.m, count, 8)
    ref = layer.csa_layer(draws, w, rows)
    moved = sum(int((ops[k].double() != ref["ops"][k].double()).sum()) for k in ops)
    total = sum(v.numel() for v in ops.values())
    print("%s: %d of %d projected inputs round differently on the two sides" % (
        name, moved, total))
    assert moved <= total * 1e-6
    run_csa(w, rows, ops=ops, ref=ref)


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
    same = check_selection(gidx, ref["idx"], ref["scores"], sc, V, w.k, "decode")
    assert_close_out(to_np(p.out)[same], ref["out"][same], "bf16", "csa out")
    ent = pipeline.split_entries(ops["kv_nope"], ops["kv_scale"], ops["kv_rope"], w.scale_group)
    o2, _ = oracle.attend(ops["q"], ent, gidx, w.k, w.m, ops["kwin"], ops["win_pos0"], w.n_win,
                          ops["q_pos"].numpy(), ops["sink"], 1.0 / math.sqrt(w.c))
    assert_close_out(to_np(p.out), o2, "bf16", "csa out (GPU selection)")
    assert_close_out(to_np(p.hout), ref["hca_out"], "bf16", "hca out")
    np.testing.assert_allclose(p.hlse.cpu().double().numpy(), ref["hca_lse"], rtol=1e-3)
