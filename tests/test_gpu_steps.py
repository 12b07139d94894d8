"""Per-step parity: each C-ABI call against the float64 oracle on identical inputs.

Inputs come from the seeded generators only; the oracle never sees a value
the CUDA path produced. Sizes span several tiles with ragged tails; the large
cases compare sampled query rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_07_b200 import abi, workloads as W
from long_context_sparse_07_b200.abi import Entries
from helpers import (assert_close_out, sample_rows, score_scale, to_np, SCORE_REL,
                     F32_MAX_ABS)

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def _clean_error_word():
    abi.csa_get_error()
    yield


# ---------------------------------------------------------------- compression


@pytest.mark.parametrize("name,n,c,m,overlap,dtype", [
    ("csa_f32", 256, 64, 4, True, "f32"),
    ("csa_f32_m1", 100, 32, 1, True, "f32"),
    ("csa_bf16", 4096, 512, 4, True, "bf16"),
    ("csa_bf16_ragged", 4 * 37, 128, 4, True, "bf16"),
    ("hca_bf16", 128 * 19, 512, 128, False, "bf16"),
    ("hca_f32_m16", 16 * 9, 64, 16, False, "f32"),
])
def test_compress_plain(name, n, c, m, overlap, dtype):
    s = 100 + len(name)
    Ca = W.to_storage(W.normal(s, "Ca", n, c, 1.0), dtype)
    Cb = W.to_storage(W.normal(s, "Cb", n, c, 1.0), dtype)
    Za = W.to_storage(W.normal(s, "Za", n, c, 1.5), dtype)
    Zb = W.to_storage(W.normal(s, "Zb", n, c, 1.5), dtype)
    Ba = W.to_storage(W.normal(s, "Ba", m, c, 0.3), "f32")
    Bb = W.to_storage(W.normal(s, "Bb", m, c, 0.3), "f32")
    E = n // m
    out = torch.empty(E, c, device=DEV, dtype=DT[dtype])
    g = lambda t: t.to(DEV) if t is not None else None
    if overlap:
        abi.csa_compress_kv(g(Ca), g(Cb), g(Za), g(Zb), g(Ba), g(Bb), m, True, Entries(out, c))
        ref = oracle.compress(Ca, Cb, Za, Zb, Ba, Bb, m, True)
    else:
        abi.csa_compress_kv(g(Ca), None, g(Za), None, g(Ba), None, m, False, Entries(out, c))
        ref = oracle.compress(Ca, None, Za, None, Ba, None, m, False)
    abi.csa_get_error()
    assert_close_out(to_np(out), ref, dtype, name)
    if dtype == "bf16":
        # storage rounding is the main difference: at most one bf16 ulp, plus
        # the float32 accumulation error (absolute: results near zero cancel)
        refb = torch.from_numpy(ref).float().to(torch.bfloat16).float().numpy()
        ulp = np.abs(refb) * 2.0 ** -7 + 4e-6
        assert (np.abs(to_np(out) - refb) <= ulp).all()


@pytest.mark.parametrize("n,cI,rope,group,dtype", [
    (4096, 128, 0, 128, "bf16"),      # indexer keys: one scale per key
    (512, 512, 64, 64, "bf16"),       # decode cache layout: 7 groups + bf16 rope
    (256, 128, 0, 128, "f32"),
])
def test_compress_fp8_output(n, cI, rope, group, dtype):
    m, s = 4, 7
    Ca = W.to_storage(W.normal(s, "CIa", n, cI, 1.0), dtype)
    Cb = W.to_storage(W.normal(s, "CIb", n, cI, 1.0), dtype)
    Za = W.to_storage(W.normal(s, "ZIa", n, cI, 1.0), dtype)
    Zb = W.to_storage(W.normal(s, "ZIb", n, cI, 1.0), dtype)
    Ba = W.to_storage(W.normal(s, "BIa", m, cI, 0.1), "f32")
    Bb = W.to_storage(W.normal(s, "BIb", m, cI, 0.1), "f32")
    E = n // m
    body = torch.empty(E, cI - rope, device=DEV, dtype=torch.float8_e4m3fn)
    scale = torch.empty(E, (cI - rope) // group, device=DEV, dtype=torch.float32)
    rp = torch.empty(E, rope, device=DEV, dtype=torch.bfloat16) if rope else None
    out = Entries(body, cI, scale=scale, rope=rp, rope_dims=rope, scale_group=group)
    abi.csa_compress_kv(Ca.to(DEV), Cb.to(DEV), Za.to(DEV), Zb.to(DEV), Ba.to(DEV), Bb.to(DEV),
                        m, True, out)
    abi.csa_get_error()
    ref = oracle.compress(Ca, Cb, Za, Zb, Ba, Bb, m, True)
    codes_ref, scale_ref = oracle.quantize_e4m3(ref[:, :cI - rope], group)
    np.testing.assert_allclose(scale.cpu().numpy(), scale_ref, rtol=2e-6)
    codes = body.cpu().view(torch.uint8).numpy()
    diff = codes != codes_ref
    # a code may differ only by one step, only where the float32 value sits
    # at a rounding boundary; such cases must be rare
    assert diff.mean() < 2e-3
    deq = oracle.dequantize(codes, scale.cpu().numpy(), group)
    deq_ref = oracle.dequantize(codes_ref, scale_ref, group)
    step = np.abs(deq_ref) * 2.0 ** -3 + np.repeat(scale_ref, group, axis=1) * 2.0 ** -9
    assert (np.abs(deq - deq_ref) <= step * 1.01).all()
    if rope:
        assert_close_out(to_np(rp), ref[:, cI - rope:], "bf16", "rope part")


# -------------------------------------------------------------------- indexer


def _indexer_case(B, n_q, E, hI, cI, m, dtype, seed, pos):
    if dtype == "e4m3":
        qI = W.e4m3_codes(seed, "qI", B * n_q, hI * cI).view(B, n_q, hI, cI)
        qs = W.e4m3_scales(seed, "qI_scale", B * n_q, hI, 0.8).view(B, n_q, hI)
        kI = W.e4m3_codes(seed, "kI", B * E, cI).view(B * E, cI)
        ks = W.e4m3_scales(seed, "kI_scale", B * E, 1, 1.0).view(B * E)
        qv = oracle.dequantize(qI, qs.reshape(B, n_q, hI, 1), cI)
        kv = oracle.dequantize(kI, ks.reshape(B * E, 1), cI).reshape(B, E, cI)
        kent = Entries(kI.to(DEV), cI, scale=ks.to(DEV), scale_group=cI)
    else:
        qI = W.to_storage(W.normal(seed, "qI", B * n_q, hI * cI, 0.5), dtype).view(B, n_q, hI, cI)
        kI = W.to_storage(W.normal(seed, "kI", B * E, cI, 1.0), dtype).view(B * E, cI)
        qs = None
        qv = oracle.f64(qI)
        kv = oracle.f64(kI).reshape(B, E, cI)
        kent = Entries(kI.to(DEV), cI)
    wI = W.to_storage(W.normal(seed, "wI", B * n_q, hI, 1.0), "f32").view(B, n_q, hI)
    q_pos = torch.as_tensor(pos, dtype=torch.int64).view(B, n_q)
    scores = torch.full((B, n_q, E), float("nan"), device=DEV)
    abi.csa_indexer_scores(qI.to(DEV), qs.to(DEV) if qs is not None else None, wI.to(DEV), kent,
                           q_pos.to(DEV), m, scores, E)
    abi.csa_get_error()
    ref = oracle.indexer(qv, oracle.f64(wI), kv, q_pos.numpy(), m)
    S = score_scale(qv, oracle.f64(wI), np.abs(kv).max())
    got = scores.cpu().double().numpy()
    for b in range(B):
        for t in range(n_q):
            V = oracle.visible(int(q_pos[b, t]), m, E)
            d = np.abs(got[b, t, :V] - ref[b, t, :V])
            assert (d <= SCORE_REL * S[b, t] + 1e-30).all(), (b, t, d.max(), S[b, t])
            assert np.isnan(got[b, t, V:]).all(), "entries past V_t must not be written"


@pytest.mark.parametrize("n,E,hI,cI,dtype", [
    (256, 64, 4, 32, "f32"),
    (4096, 1024, 16, 128, "bf16"),
    (1000, 250, 64, 128, "e4m3"),
    (300, 75, 16, 64, "bf16"),
])
def test_indexer_prefill(n, E, hI, cI, dtype):
    _indexer_case(1, n, E, hI, cI, 4, dtype, 11, np.arange(n))


def test_indexer_decode_batches():
    B, E = 3, 20000
    pos = np.array([4 * E - 1, 4 * 15000 + 2, 4 * E - 1])     # last batch sees all
    _indexer_case(B, 1, E, 64, 128, 4, "e4m3", 12, pos)


# ---------------------------------------------------------------------- top-k


def _topk_case(rows, E, k, m, pos, seed):
    sc = W.score_rows(seed, rows, E)
    q_pos = torch.as_tensor(pos, dtype=torch.int64)
    idx = torch.full((rows, k), -7, device=DEV, dtype=torch.int32)
    nws = abi.csa_topk_workspace_size(rows, E, k)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8) if nws else None
    abi.csa_topk(sc.to(DEV), q_pos.to(DEV), m, k, idx, E, workspace=ws)
    abi.csa_get_error()
    ref = oracle.topk(sc.double().numpy(), q_pos.numpy(), m, k)
    got = idx.cpu().numpy()
    bad = np.nonzero((got != ref).any(1))[0]
    assert len(bad) == 0, "rows %s differ, first: gpu %s oracle %s" % (
        bad[:5], got[bad[0]][:16], ref[bad[0]][:16])


@pytest.mark.parametrize("rows,E,k,m", [
    (4096, 1024, 256, 4),      # causal prefill rows (V_t grows with t)
    (300, 64, 8, 4),
    (257, 300, 1, 1),
    (64, 5000, 4096, 1),       # k larger than most rows
])
def test_topk_causal(rows, E, k, m):
    _topk_case(rows, E, k, m, np.arange(rows) * max(1, (E * m) // rows), 21)


def test_topk_long_rows_resident_and_streamed():
    # rows of 32768 (staged in shared memory) and 262144 (re-read from L2)
    _topk_case(6, 32768, 1024, 4, [4 * 32768 - 1, 40000, 4 * 30000, 4000, 4 * 32768 - 1, 5], 22)
    _topk_case(3, 262144, 1024, 4, [4 * 262144 - 1] * 3, 23)


def test_topk_block_rows_streamed_and_ties():
    # one block per row past the shared-memory stage (rows re-read from L2)
    _topk_case(4, 50000, 1000, 1, [49999, 41000, 900, 45000], 25)
    # ties straddling the k-th value in every radix digit: five distinct scores
    rows, E, k = 3, 20000, 777
    rng = np.random.default_rng(26)
    sc = torch.as_tensor(rng.integers(0, 5, size=(rows, E)).astype(np.float32) * 0.5 - 1.0)
    q_pos = torch.tensor([E - 1, 15000, E - 1], dtype=torch.int64)
    idx = torch.empty(rows, k, device=DEV, dtype=torch.int32)
    abi.csa_topk(sc.to(DEV), q_pos.to(DEV), 1, k, idx, E)
    abi.csa_get_error()
    ref = oracle.topk(sc.double().numpy(), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_mid_rows_clustered_sorted_and_sparse():
    # rows of 2K..64K entries take a sampled lower bound and per-warp candidate
    # regions; rows whose top entries crowd one part of the row (sorted rows,
    # one hot cluster) overflow a region and are selected from the row itself
    rows, E, k = 6, 40000, 1024
    rng = np.random.default_rng(27)
    sc = rng.standard_normal((rows, E)).astype(np.float32)
    sc[0] = np.arange(E, dtype=np.float32)                 # ascending: top-k at the end
    sc[1] = -np.arange(E, dtype=np.float32)                # descending: top-k at the start
    sc[2, 20000:22000] += 50.0                             # one hot cluster of 2000
    sc[3] = np.where(rng.random(E) < 0.03, 10.0, -10.0)    # 3 % hot entries, all tied
    sc[4, ::7] = 3.0                                       # a tied grid near the bound
    q_pos = torch.tensor([E - 1, E - 1, E - 1, E - 1, E - 1, 30000], dtype=torch.int64)
    idx = torch.empty(rows, k, device=DEV, dtype=torch.int32)
    abi.csa_topk(torch.as_tensor(sc).to(DEV), q_pos.to(DEV), 1, k, idx, E)
    abi.csa_get_error()
    ref = oracle.topk(sc.astype(np.float64), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_long_rows_split_over_blocks():
    # rows of 65536 .. 262144 entries: one cluster of blocks per row, each
    # block a share of the row; the threshold key's ties across block borders,
    # short rows (V <= k) mixed in, and a row with massive ties
    rows, E, k = 5, 100000, 700
    assert abi.csa_topk_workspace_size(rows, E, k) == 0
    pos = [E - 1, 70000, 500, E - 1, 80000]
    _topk_case(rows, E, k, 1, pos, 24)
    sc = torch.zeros(2, E)
    sc[1, ::3] = 1.0
    q_pos = torch.tensor([E - 1, E - 1], dtype=torch.int64)
    idx = torch.empty(2, k, device=DEV, dtype=torch.int32)
    ws = torch.empty(abi.csa_topk_workspace_size(2, E, k), device=DEV, dtype=torch.uint8)
    abi.csa_topk(sc.to(DEV), q_pos.to(DEV), 1, k, idx, E, workspace=ws)
    abi.csa_get_error()
    ref = oracle.topk(sc.double().numpy(), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_cluster_rows_unaligned_and_tied():
    # decode-width rows (262144 entries) whose starts are not 16-byte aligned
    # (row stride E + 1: the shares are read element by element), the largest
    # k, and rows whose k-th value is tied across every block of the row
    rows, E, k = 6, 262144, 4096
    rng = np.random.default_rng(28)
    full = rng.standard_normal((rows, E + 1)).astype(np.float32)
    full[1, :E] = np.where(rng.random(E) < 0.02, 2.0, -1.0)     # ~5200 tied at the top
    full[2, :E] = 0.0
    full[2, 100:E:50] = -0.0                                    # -0 and +0 are one value
    full[3, :E] = np.round(full[3, :E] * 4) / 4                 # many ties in every digit
    q_pos = torch.tensor([E - 1, E - 1, E - 1, 4000, 200000, E - 2], dtype=torch.int64)
    sc = torch.as_tensor(full)
    idx = torch.full((rows, k), -7, device=DEV, dtype=torch.int32)
    abi.csa_topk(sc.to(DEV), q_pos.to(DEV), 1, k, idx, E)      # row stride E + 1
    abi.csa_get_error()
    ref = oracle.topk(full[:, :E].astype(np.float64), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_cluster_rows_mixed_lengths_and_orders():
    # 40 rows of a 131072-wide table: lengths from k + 1 up to the full row,
    # normal, exponential, sorted and grid-valued rows (the candidate path and
    # the all-keys path both taken), k = 1000
    rows, E, k = 40, 131072, 1000
    rng = np.random.default_rng(30)
    sc = rng.standard_normal((rows, E)).astype(np.float32)
    sc[1::5] = rng.exponential(1.0, size=(len(range(1, rows, 5)), E))
    sc[2] = np.arange(E, dtype=np.float32)                 # ascending
    sc[3] = -np.arange(E, dtype=np.float32)                # descending
    sc[4::5] = np.round(sc[4::5] * 8) / 8                  # many ties near every digit
    V = np.concatenate([[k + 1, k + 2, 2 * k, 32 * k + 7, E, E - 1, 65537, 100001],
                        rng.integers(k + 1, E + 1, size=rows - 8)])
    q_pos = torch.as_tensor(V - 1, dtype=torch.int64)
    idx = torch.full((rows, k), -7, device=DEV, dtype=torch.int32)
    abi.csa_topk(torch.as_tensor(sc).to(DEV), q_pos.to(DEV), 1, k, idx, E)
    abi.csa_get_error()
    ref = oracle.topk(sc.astype(np.float64), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_rows_past_cluster_reach():
    # rows longer than 262144 entries: the four-launch chunked path with a
    # caller workspace
    rows, E, k = 3, 300000, 1024
    assert abi.csa_topk_workspace_size(rows, E, k) > 0
    _topk_case(rows, E, k, 1, [E - 1, 290000, 262145], 29)


def test_topk_all_equal_scores_prefers_low_indices():
    rows, E, k = 4, 2000, 100
    sc = torch.zeros(rows, E)
    sc[1] = -0.0
    sc[2, 1500:] = 1.0
    q_pos = torch.tensor([E - 1, E - 1, E - 1, 50], dtype=torch.int64)
    idx = torch.empty(rows, k, device=DEV, dtype=torch.int32)
    abi.csa_topk(sc.to(DEV), q_pos.to(DEV), 1, k, idx, E)
    ref = oracle.topk(sc.double().numpy(), q_pos.numpy(), 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    assert idx[0].tolist() == list(range(k))


# ------------------------------------------------------------------ attention


def _attend_case(B, n, E, m, h, c, k, n_win, dtype, seed, rows=None, kv_layout="plain",
                 dense=False, bad_index=False):
    pos = np.tile(np.arange(n), (B, 1)) if rows is None else np.tile(rows, (B, 1))
    n_q = pos.shape[1]
    q = W.to_storage(W.normal(seed, "q", B * n_q, h * c, 1.0), dtype).view(B, n_q, h, c)
    if kv_layout == "fp8":
        G = 64
        body = W.e4m3_codes(seed, "kv_nope", B * E, c - 64)
        scl = W.e4m3_scales(seed, "kv_scale", B * E, (c - 64) // G, 1.0)
        rope = W.to_storage(W.normal(seed, "kv_rope", B * E, 64, 1.0), "bf16")
        ent64 = np.concatenate([oracle.dequantize(body, scl, G), oracle.f64(rope)], -1)
        ent = Entries(body.to(DEV), c, scale=scl.to(DEV), rope=rope.to(DEV), rope_dims=64,
                      scale_group=G)
    else:
        kvt = W.to_storage(W.normal(seed, "entries", B * E, c, 1.0), dtype)
        ent64 = oracle.f64(kvt)
        ent = Entries(kvt.to(DEV), c)
    ent64 = ent64.reshape(B, E, c)
    win_rows = n
    kwin = W.to_storage(W.normal(seed, "kwin_step", B * win_rows, c, 1.0), dtype).view(
        B, win_rows, c)
    win_pos0 = np.zeros(B, dtype=np.int64)
    sink = W.to_storage(W.normal(seed, "sink", 1, h, 1.0), "f32").view(h)
    sink[0] = -float("inf")
    vis = np.array([oracle.visible(t, m, E) for t in pos.reshape(-1)])
    idx = None
    if not dense:
        idx = W.stratified_idx(seed, B * n_q, k, vis)
        if bad_index:
            idx[-1, 0] = int(vis[-1]) + 3          # an invisible entry
    out = torch.empty(B, n_q, h, c, device=DEV, dtype=DT[dtype])
    lse = torch.empty(B, n_q, h, device=DEV)
    scale = 1.0 / math.sqrt(c)
    qp = torch.as_tensor(pos, dtype=torch.int64).to(DEV)
    wp = torch.as_tensor(win_pos0).to(DEV)
    nws = abi.csa_mqa_workspace_size(B, n_q, h, c, (E if dense else k) + n_win)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8) if nws else None
    if dense:
        abi.hca_dense_mqa(q.to(DEV), ent, E, m, kwin.to(DEV), wp, n_win, qp, sink.to(DEV),
                          scale, out, lse, workspace=ws)
    else:
        abi.csa_sparse_mqa(q.to(DEV), ent, E, m, idx.to(DEV), k, kwin.to(DEV), wp, n_win, qp,
                           sink.to(DEV), scale, out, lse, workspace=ws)
    if bad_index:
        with pytest.raises(abi.CsaError) as ei:
            abi.csa_get_error()
        assert ei.value.status == -5
        idx[-1, 0] = -1                             # the kernel skipped it
    else:
        abi.csa_get_error()
    ref, lref = oracle.attend(q, ent64, idx.numpy() if idx is not None else None, k, m, kwin,
                              win_pos0, n_win, pos, sink, scale)
    assert_close_out(to_np(out), ref, dtype, "out")
    lg = lse.cpu().double().numpy()
    fin = np.isfinite(lref)
    # bf16 path: probabilities are rounded to bf16 (relative error <= 2^-9)
    # before both the weighted sum and the normaliser, so lse = M + log(sum)
    # carries up to ~2^-9 of absolute error; the f32 path keeps 1e-4.
    tol = 1e-4 if dtype == "f32" else 2.0 ** -8
    np.testing.assert_allclose(lg[fin], lref[fin], rtol=0, atol=tol)
    assert (lg[~fin] == lref[~fin]).all()


def test_attend_sparse_f32_small():
    _attend_case(1, 256, 64, 4, 4, 64, 8, 16, "f32", 31)


def test_attend_sparse_bf16_prefill_sampled():
    rows = sample_rows(4096, 4, 160, 1)
    _attend_case(1, 4096, 1024, 4, 32, 512, 256, 128, "bf16", 32, rows=rows)


def test_attend_sparse_bf16_h64_k1024_sampled():
    rows = sample_rows(8192, 4, 96, 2)
    _attend_case(1, 8192, 2048, 4, 64, 512, 1024, 128, "bf16", 33, rows=rows)


def test_attend_sparse_decode_fp8_layout():
    L = 4 * 6000
    _attend_case(2, L, 6000, 4, 64, 512, 1024, 128, "bf16", 34, rows=np.array([L - 1]),
                 kv_layout="fp8")


def test_attend_dense_hca_sampled():
    rows = sample_rows(128 * 40, 128, 96, 3)
    _attend_case(1, 128 * 40, 40, 128, 64, 512, 0, 128, "bf16", 35, rows=rows, dense=True)


def test_attend_split_keys_dense_bf16_few_queries():
    # few queries, many keys: each query's key tiles are split over blocks and
    # joined by the combine step (scratch from csa_mqa_workspace_size)
    rows = np.array([0, 15, 16 * 700 - 1, 16 * 1500, 16 * 3000 - 1, 16 * 2999 + 5])
    _attend_case(1, 16 * 3000, 3000, 16, 32, 512, 0, 128, "bf16", 40, rows=rows, dense=True)


def test_attend_split_keys_sparse_bf16_h16():
    rows = np.array([3, 4000, 4 * 2000 - 1])
    _attend_case(1, 4 * 2000, 2000, 4, 16, 512, 1024, 128, "bf16", 41, rows=rows)


def test_attend_split_keys_decode_fp8_h64_hca():
    L = 128 * 300
    _attend_case(2, L, 300, 128, 64, 512, 0, 128, "bf16", 42, rows=np.array([L - 1]),
                 kv_layout="fp8", dense=True)


def test_attend_dense_f32_small():
    _attend_case(1, 200, 12, 16, 4, 64, 0, 16, "f32", 36, dense=True)


def test_attend_window_only_and_no_window():
    _attend_case(1, 300, 75, 4, 8, 64, 0, 32, "f32", 37)          # k = 0: window only
    _attend_case(1, 300, 75, 4, 8, 64, 8, 0, "f32", 38)           # no window


def test_attend_bad_index_is_reported_and_skipped():
    _attend_case(1, 64, 16, 4, 4, 64, 4, 8, "f32", 39, bad_index=True)
