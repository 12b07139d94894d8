"""csa_indexer_topk (the indexer scores of Eq. 16 and the top-k of Eq. 17 in
one call, without the score rows) against the oracle.

The call selects exactly on float32 scores; the oracle scores in float64. On
rows longer than k, every entry whose float64 score lies clearly above the
row's k-th largest must be selected and every entry clearly below must not
(clearly: further than the float32 accumulation error SCORE_REL * S_t from
it); the selection has exactly k distinct visible entries in ascending
order. Rows of at most k visible entries select all of them. Where the
scores are exact on both sides (all equal), the oracle's selection, ties to
the lower index, must come out exactly. The call must also give exactly what
csa_indexer_scores followed by csa_topk give on the same device (both select
on the same float32 values): that covers every row of every case, including
the rows that take the full recomputation.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_07_b200 import abi, workloads as W
from long_context_sparse_07_b200.abi import Entries
from helpers import score_scale, SCORE_REL

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean_error_word():
    abi.csa_get_error()
    yield
    abi.csa_get_error()


def _operands(B, n_q, E, hI, cI, dtype, seed):
    """Device operands and their float64 values (qv [B, n_q, hI, cI],
    kv [B, E, cI], wv [B, n_q, hI])."""
    if dtype == "e4m3":
        qI = W.e4m3_codes(seed, "qI", B * n_q, hI * cI).view(B, n_q, hI, cI)
        qs = W.e4m3_scales(seed, "qI_scale", B * n_q, hI, 0.8).view(B, n_q, hI)
        kI = W.e4m3_codes(seed, "kI", B * E, cI).view(B * E, cI)
        ks = W.e4m3_scales(seed, "kI_scale", B * E, 1, 1.0).view(B * E)
    else:
        qI = W.to_storage(W.normal(seed, "qI", B * n_q, hI * cI, 0.5), dtype).view(B, n_q, hI, cI)
        kI = W.to_storage(W.normal(seed, "kI", B * E, cI, 1.0), dtype).view(B * E, cI)
        qs = ks = None
    wI = W.to_storage(W.normal(seed, "wI", B * n_q, hI, 1.0), "f32").view(B, n_q, hI)
    return qI, qs, kI, ks, wI


def _values(qI, qs, kI, ks, wI, B, E, cI):
    if qs is not None:
        qv = oracle.dequantize(qI, qs.reshape(*qs.shape, 1), cI)
        kv = oracle.dequantize(kI, ks.reshape(-1, 1), cI).reshape(B, E, cI)
    else:
        qv = oracle.f64(qI)
        kv = oracle.f64(kI).reshape(B, E, cI)
    return qv, kv, oracle.f64(wI)


def _run(qI, qs, kI, ks, wI, pos, m, k, E):
    """(fused idx, idx of csa_indexer_scores + csa_topk), both [B * n_q, k]."""
    B, n_q, hI, cI = qI.shape
    dq = lambda t: t.to(DEV) if t is not None else None
    qI_d, qs_d, wI_d = dq(qI), dq(qs), dq(wI)
    kent = Entries(kI.to(DEV), cI, scale=dq(ks), scale_group=cI if ks is not None else 0)
    q_pos = torch.as_tensor(pos, dtype=torch.int64).view(B, n_q).to(DEV)
    nws = abi.csa_indexer_topk_workspace_size(B, n_q, E, hI, cI, k, qI)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8) if nws else None
    fused = torch.full((B * n_q, k), -7, device=DEV, dtype=torch.int32)
    abi.csa_indexer_topk(qI_d, qs_d, wI_d, kent, q_pos, m, k, fused, E, workspace=ws)
    abi.csa_get_error()
    del ws
    scores = torch.empty(B, n_q, max(E, 1), device=DEV, dtype=torch.float32)
    abi.csa_indexer_scores(qI_d, qs_d, wI_d, kent, q_pos, m, scores, E)
    two = torch.full((B * n_q, k), -7, device=DEV, dtype=torch.int32)
    nt = abi.csa_topk_workspace_size(B * n_q, E, k)
    tws = torch.empty(nt, device=DEV, dtype=torch.uint8) if nt else None
    abi.csa_topk(scores.view(B * n_q, -1), q_pos.view(-1), m, k, two, E, workspace=tws)
    abi.csa_get_error()
    return fused.cpu().numpy(), two.cpu().numpy()


def _check_rows(got, qv, kv, wv, pos, m, k, rows, what):
    """Selection properties against the oracle's float64 scores on the given
    flat rows (b * n_q + t)."""
    B, n_q = qv.shape[:2]
    E = kv.shape[1]
    S = score_scale(qv, wv, np.abs(kv).max())
    pos = np.asarray(pos).reshape(B, n_q)
    for r in rows:
        b, t = divmod(int(r), n_q)
        ref = oracle.indexer(qv[b:b + 1, t:t + 1], wv[b:b + 1, t:t + 1], kv[b:b + 1],
                             pos[b:b + 1, t:t + 1], m)[0, 0]
        V = oracle.visible(int(pos[b, t]), m, E)
        g = got[r]
        if V <= k:
            exp = np.concatenate([np.arange(V), -np.ones(k - V)])
            np.testing.assert_array_equal(g, exp, err_msg="%s row %d" % (what, r))
            continue
        sel = g[g >= 0]
        assert len(sel) == k, "%s row %d: %d selected" % (what, r, len(sel))
        assert (np.diff(sel) > 0).all() and sel.min() >= 0 and sel.max() < V, (what, r)
        row = ref[:V]
        kth = np.partition(row, V - k)[V - k]
        tol = 2 * SCORE_REL * S[b, t]
        must = np.nonzero(row > kth + tol)[0]
        never = np.nonzero(row < kth - tol)[0]
        assert np.isin(must, sel).all(), "%s row %d: a clear winner is missing" % (what, r)
        assert not np.isin(never, sel).any(), "%s row %d: a clear loser is selected" % (what, r)


def _case(B, n_q, E, hI, cI, k, m, dtype, seed, pos, check_rows, fused):
    launches = abi.csa_indexer_topk_launches(B, n_q, E, hI, cI, k, abi.CSA_E4M3 if
                                             dtype == "e4m3" else abi.CSA_BF16 if
                                             dtype == "bf16" else abi.CSA_F32)
    assert (launches == 6) == fused, "candidate path %s expected, %d launches" % (fused, launches)
    qI, qs, kI, ks, wI = _operands(B, n_q, E, hI, cI, dtype, seed)
    got, two = _run(qI, qs, kI, ks, wI, pos, m, k, E)
    bad = np.nonzero((got != two).any(1))[0]
    assert len(bad) == 0, "rows %s: fused %s, two calls %s" % (bad[:4], got[bad[0]][:12],
                                                              two[bad[0]][:12])
    qv, kv, wv = _values(qI, qs, kI, ks, wI, B, E, cI)
    _check_rows(got, qv, kv, wv, pos, m, k, check_rows, "%s E=%d" % (dtype, E))


def _spread(n_q, E, m, seed):
    """Causal prefill positions reaching every length 0 .. E entries, with
    the first block, block edges and the last position among them."""
    pos = np.linspace(0, m * E - 1, n_q).astype(np.int64)
    pos[:m + 1] = np.arange(m + 1)
    pos[-1] = m * E - 1
    return np.sort(pos)


def _some(n_q, step):
    return np.unique(np.concatenate([np.arange(0, n_q, step), [1, 2, n_q // 2, n_q - 1]]))


def test_fused_prefill_e4m3_h64():
    # 16-token blocks owning whole rows: the candidate path
    n_q, E, m, k = 6144, 16384, 4, 1024
    _case(1, n_q, E, 64, 128, k, m, "e4m3", 31, _spread(n_q, E, m, 1), _some(n_q, 151), True)


def test_fused_prefill_bf16_h64():
    n_q, E, m, k = 1600, 8192, 4, 512
    _case(1, n_q, E, 64, 128, k, m, "bf16", 32, _spread(n_q, E, m, 2), _some(n_q, 61), True)


def test_fused_prefill_e4m3_h16_ragged():
    # a ragged last token block (4803 = 300 * 16 + 3)
    n_q, E, m, k = 4803, 20480, 4, 256
    _case(1, n_q, E, 16, 128, k, m, "e4m3", 33, _spread(n_q, E, m, 3), _some(n_q, 131), True)


def test_fused_prefill_e4m3_h32():
    n_q, E, m, k = 4800, 16384, 4, 512
    _case(1, n_q, E, 32, 128, k, m, "e4m3", 40, _spread(n_q, E, m, 8), _some(n_q, 149), True)


def test_fused_decode_takes_the_two_calls():
    # one query per batch: few token blocks split each row over many blocks,
    # and the call runs the two plain kernels
    B, E, m, k = 4, 65536, 4, 1024
    pos = np.array([m * E - 1, m * 50000 + 3, m * E - 1, m * 4000])
    _case(B, 1, E, 64, 128, k, m, "e4m3", 34, pos, np.arange(B), False)


def test_fused_few_queries_take_the_two_calls():
    n_q, E, m, k = 203, 20480, 4, 256
    _case(1, n_q, E, 16, 128, k, m, "e4m3", 35, _spread(n_q, E, m, 9), np.arange(0, n_q, 7),
          False)


def test_fused_short_rows_and_f32_take_the_two_calls():
    # E < 16 k (no candidate path) and a float32 indexer (no tensor-core path)
    n_q, E, m, k = 700, 1024, 4, 256
    _case(1, n_q, E, 16, 128, k, m, "bf16", 36, _spread(n_q, E, m, 4), np.arange(0, n_q, 37),
          False)
    n_q, E = 300, 20000
    _case(1, n_q, E, 4, 32, 64, m, "f32", 37, _spread(n_q, E, m, 5), np.arange(0, n_q, 29),
          False)


def _e4m3(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)


def test_fused_all_equal_scores_prefer_low_indices():
    # every key is zero: every score is exactly 0 on both sides. Rows longer
    # than their candidate room are recomputed in full, shorter ones are cut
    # among the tied keys; both must keep the lowest indices
    B, n_q, E, hI, cI, m, k = 1, 4800, 16384, 64, 128, 4, 1024
    assert abi.csa_indexer_topk_launches(B, n_q, E, hI, cI, k, abi.CSA_E4M3) == 6
    qI, qs, _, _, wI = _operands(B, n_q, E, hI, cI, "e4m3", 38)
    kI = _e4m3(np.zeros((E, cI)))
    ks = torch.ones(E, dtype=torch.float32)
    pos = _spread(n_q, E, m, 6)
    got, two = _run(qI, qs, kI, ks, wI, pos, m, k, E)
    np.testing.assert_array_equal(got, two)
    rows = _some(n_q, 173)
    qv, kv, wv = _values(qI[:, rows], qs[:, rows], kI, ks, wI[:, rows], B, E, cI)
    sc = oracle.indexer(qv, wv, kv, pos[rows].reshape(1, -1), m)[0]
    assert (sc[np.isfinite(sc)] == 0).all()
    np.testing.assert_array_equal(got[rows], oracle.topk(sc, pos[rows], m, k))


def test_fused_misleading_sample_is_recomputed():
    # the sampled keys (every S-th, S = 32 here) all score far above every
    # other key, so the bound from the sample leaves fewer than k candidates:
    # every long row takes the full recomputation, which must still select
    # the row's true top-k
    B, n_q, E, hI, cI, m, k = 1, 4800, 16384, 64, 128, 4, 1024
    assert abi.csa_indexer_topk_launches(B, n_q, E, hI, cI, k, abi.CSA_E4M3) == 6
    g = np.random.default_rng(39)
    kv = g.uniform(-0.25, 0.25, size=(E, cI))
    kv[::32] = 2.0
    kI = _e4m3(kv)
    ks = torch.ones(E, dtype=torch.float32)
    qI = _e4m3(g.uniform(0.5, 1.0, size=(B, n_q, hI, cI)))
    qs = torch.ones(B, n_q, hI, dtype=torch.float32)
    wI = torch.as_tensor(g.uniform(0.5, 1.0, size=(B, n_q, hI)).astype(np.float32))
    pos = _spread(n_q, E, m, 7)
    got, two = _run(qI, qs, kI, ks, wI, pos, m, k, E)
    np.testing.assert_array_equal(got, two)
    qv, kv64, wv = _values(qI, qs, kI, ks, wI, B, E, cI)
    _check_rows(got, qv, kv64, wv, pos, m, k, _some(n_q, 397), "planted sample")


def test_fused_few_distinct_scores():
    # every key is one of 6 vectors, so a query's scores take at most 6
    # values: the threshold value is shared by thousands of candidates (the
    # select's path for a crowded threshold bin, cut among equal scores by
    # index)
    B, n_q, E, hI, cI, m, k = 1, 4800, 16384, 64, 128, 4, 1024
    assert abi.csa_indexer_topk_launches(B, n_q, E, hI, cI, k, abi.CSA_E4M3) == 6
    g = np.random.default_rng(41)
    base = g.normal(0.0, 1.0, size=(6, cI))
    kI = _e4m3(base[g.integers(0, 6, size=E)])
    ks = torch.ones(E, dtype=torch.float32)
    qI, qs, _, _, wI = _operands(B, n_q, E, hI, cI, "e4m3", 42)
    pos = _spread(n_q, E, m, 10)
    got, two = _run(qI, qs, kI, ks, wI, pos, m, k, E)
    np.testing.assert_array_equal(got, two)
    qv, kv, wv = _values(qI, qs, kI, ks, wI, B, E, cI)
    _check_rows(got, qv, kv, wv, pos, m, k, _some(n_q, 397), "six key vectors")
