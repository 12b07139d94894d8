"""Edge cases of the C-ABI calls on the GPU: empty inputs, the largest k, the
widest indexer, and attention sinks at +-inf, each against the oracle or the
documented behaviour (an empty call is a successful no-op)."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_07_b200 import abi, workloads as W
from long_context_sparse_07_b200.abi import Entries
from helpers import assert_close_out, score_scale, to_np, SCORE_REL

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean_error_word():
    abi.csa_get_error()
    yield


def test_empty_inputs_are_no_ops():
    # zero tokens, zero score rows and zero queries: each call returns CSA_OK
    # and leaves its outputs untouched. The sizes are passed to the C calls
    # directly (valid buffers, zero counts).
    L = abi.load()
    c, m = 512, 4
    big = torch.randn(8, c, device=DEV).to(torch.bfloat16)
    bias = torch.zeros(m, c, device=DEV)
    out = torch.full((4, c), 7.0, device=DEV).to(torch.bfloat16)
    p = lambda t: t.data_ptr()
    st = L.csa_compress_kv(p(big), p(big), p(big), p(big), p(bias), p(bias), 0, c, m, 1,
                           abi.dtype_code(big), Entries(out, c).struct(), None)
    assert st == 0
    sc = torch.zeros(4, 64, device=DEV)
    idx = torch.full((4, 8), -7, device=DEV, dtype=torch.int32)
    pos = torch.zeros(4, dtype=torch.int64, device=DEV)
    st = L.csa_topk(p(sc), 0, 64, 64, p(pos), 1, 8, p(idx), None, 0, None)
    assert st == 0
    q = torch.randn(1, 4, 16, c, device=DEV).to(torch.bfloat16)
    o = torch.full((1, 4, 16, c), 7.0, device=DEV).to(torch.bfloat16)
    sink = torch.zeros(16, device=DEV)
    wp = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = L.hca_dense_mqa(p(q), abi.dtype_code(q), Entries(big, c).struct(), 8, m, p(big), 8,
                         p(wp), 4, p(pos), p(sink), 1, 0, 16, 0.1, p(o), None, None, 0, None)
    assert st == 0
    torch.cuda.synchronize()
    assert (out == 7.0).all() and (idx == -7).all() and (o == 7.0).all()
    abi.csa_get_error()


def test_attend_sinks_at_plus_and_minus_infinity_tensor_core_path():
    # h = 16 bf16 (tensor-core kernel): head 0 sink +inf (output 0, lse +inf),
    # head 1 sink -inf (plain softmax), the rest finite
    B, n, E, m, h, c, k, n_win, seed = 1, 96, 24, 4, 16, 512, 8, 16, 71
    pos = np.arange(n).reshape(1, n)
    q = W.to_storage(W.normal(seed, "q", n, h * c, 1.0), "bf16").view(B, n, h, c)
    kvt = W.to_storage(W.normal(seed, "entries", E, c, 1.0), "bf16")
    kwin = W.to_storage(W.normal(seed, "kwin_step", n, c, 1.0), "bf16").view(B, n, c)
    sink = W.to_storage(W.normal(seed, "sink", 1, h, 1.0), "f32").view(h)
    sink[0], sink[1] = float("inf"), -float("inf")
    vis = np.array([oracle.visible(t, m, E) for t in range(n)])
    idx = W.stratified_idx(seed, n, k, vis)
    out = torch.empty(B, n, h, c, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, n, h, device=DEV)
    scale = 1.0 / math.sqrt(c)
    wp = torch.zeros(B, dtype=torch.int64, device=DEV)
    nws = abi.csa_mqa_workspace_size(B, n, h, c, k + n_win)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8) if nws else None
    abi.csa_sparse_mqa(q.to(DEV), Entries(kvt.to(DEV), c), E, m, idx.to(DEV), k, kwin.to(DEV), wp,
                       n_win, torch.as_tensor(pos).to(DEV), sink.to(DEV), scale, out, lse,
                       workspace=ws)
    abi.csa_get_error()
    ref, lref = oracle.attend(q, oracle.f64(kvt).reshape(B, E, c), idx.numpy(), k, m, kwin,
                              np.zeros(B, dtype=np.int64), n_win, pos, sink, scale)
    got = to_np(out)
    assert (got[:, :, 0] == 0).all()
    assert np.isposinf(lse[:, :, 0].cpu().numpy()).all()
    assert_close_out(got, ref, "bf16", "out")
    lg = lse.cpu().double().numpy()
    fin = np.isfinite(lref)
    np.testing.assert_allclose(lg[fin], lref[fin], rtol=0, atol=2.0 ** -8)


@pytest.mark.parametrize("rows,E,k", [(48, 8192, 4096), (40, 1500, 4096), (8, 70000, 4096)])
def test_topk_largest_k(rows, E, k):
    sc = W.score_rows(81, rows, E)
    pos = np.linspace(0, E - 1, rows).astype(np.int64)
    idx = torch.full((rows, k), -7, device=DEV, dtype=torch.int32)
    nws = abi.csa_topk_workspace_size(rows, E, k)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8) if nws else None
    abi.csa_topk(sc.to(DEV), torch.as_tensor(pos).to(DEV), 1, k, idx, E, workspace=ws)
    abi.csa_get_error()
    ref = oracle.topk(sc.double().numpy(), pos, 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_indexer_widest_heads():
    # h_I = 128 (the largest the call takes) with c_I = 64, bf16
    B, n_q, E, hI, cI, m, seed = 1, 200, 50, 128, 64, 4, 91
    qI = W.to_storage(W.normal(seed, "qI", n_q, hI * cI, 0.5), "bf16").view(B, n_q, hI, cI)
    kI = W.to_storage(W.normal(seed, "kI", E, cI, 1.0), "bf16").view(E, cI)
    wI = W.to_storage(W.normal(seed, "wI", n_q, hI, 1.0), "f32").view(B, n_q, hI)
    pos = torch.arange(n_q, dtype=torch.int64).view(B, n_q)
    scores = torch.full((B, n_q, E), float("nan"), device=DEV)
    abi.csa_indexer_scores(qI.to(DEV), None, wI.to(DEV), Entries(kI.to(DEV), cI), pos.to(DEV), m,
                           scores, E)
    abi.csa_get_error()
    qv, kv = oracle.f64(qI), oracle.f64(kI).reshape(B, E, cI)
    ref = oracle.indexer(qv, oracle.f64(wI), kv, pos.numpy(), m)
    S = score_scale(qv, oracle.f64(wI), np.abs(kv).max())
    got = scores.cpu().double().numpy()
    for t in range(n_q):
        V = oracle.visible(t, m, E)
        d = np.abs(got[0, t, :V] - ref[0, t, :V])
        assert (d <= SCORE_REL * S[0, t] + 1e-30).all(), (t, d.max())
        assert np.isnan(got[0, t, V:]).all()
