"""FP4 (e2m1) indexer keys on the GPU against the oracle.

* Compression to the fp4 layout: the GPU compresses in float32, the oracle in
  float64, so a value may round to a neighbouring code, or its block take the
  neighbouring exponent, where the two sides straddle a boundary; every value
  is held to one code step of its block scale and nearly all must be equal.
* Indexer scores with fp4 keys and e4m3 queries: every product is exact on
  the GPU (the keys are rebuilt exactly as e4m3 values), so only the float32
  accumulation order differs from the oracle's float64 scores over the
  oracle's own decoding of the same codes: SCORE_REL * S_t.
* The indexer and the top-k in one call with fp4 keys select exactly what the
  two calls select, and agree with the oracle's scores at the boundary.
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


def fp4_keys(seed, rows, cI, lo=118, hi=126):
    """Random packed e2m1 codes and block exponents (a span of at most 8)."""
    g = np.random.default_rng(seed)
    packed = g.integers(0, 256, size=(rows, cI // 2), dtype=np.uint8)
    exps = g.integers(lo, hi + 1, size=(rows, cI // 32), dtype=np.uint8)
    return torch.from_numpy(packed), torch.from_numpy(exps)


def e4m3_queries(seed, B, n_q, hI, cI):
    qI = W.e4m3_codes(seed, "qI", B * n_q, hI * cI).view(B, n_q, hI, cI)
    qs = W.e4m3_scales(seed, "qI_scale", B * n_q, hI, 0.8).view(B, n_q, hI)
    wI = W.to_storage(W.normal(seed, "wI", B * n_q, hI, 1.0), "f32").view(B, n_q, hI)
    return qI, qs, wI


def test_compress_fp4_output():
    n, c, m = 4096, 128, 4
    g = np.random.default_rng(5)
    Ca, Cb, Za, Zb = (torch.from_numpy(g.normal(0, 1, size=(n, c)).astype(np.float32))
                      .to(torch.bfloat16) for _ in range(4))
    Ca[7 * m:8 * m, 32:64] = 0                    # an entry block of zeros (its Cb half too)
    Cb[6 * m:7 * m, 32:64] = 0
    Ca[100 * m:101 * m] *= 1e-4                   # rows far below their neighbours
    Ba, Bb = (torch.from_numpy(g.normal(0, 0.5, size=(m, c)).astype(np.float32))
              for _ in range(2))
    E = n // m
    body = torch.empty(E, c // 2, device=DEV, dtype=torch.uint8)
    exps = torch.empty(E, c // 32, device=DEV, dtype=torch.uint8)
    out = Entries(body, c, scale=exps, scale_group=32, fp4=True)
    abi.csa_compress_kv(*(t.to(DEV) for t in (Ca, Cb, Za, Zb, Ba, Bb)), m, True, out)
    abi.csa_get_error()
    ref = oracle.compress(Ca, Cb, Za, Zb, Ba, Bb, m)
    rp, re = oracle.quantize_e2m1(ref)
    ge = exps.cpu().numpy().astype(np.int64)
    assert (ge.max(1) - ge.min(1) <= 8).all(), "block exponents of a row span more than 8"
    assert (np.abs(ge - re.astype(np.int64)) <= 1).all()
    gv = oracle.dequantize_e2m1(body.cpu(), exps.cpu())
    rv = oracle.dequantize_e2m1(rp, re)
    scale = 2.0 ** (np.maximum(ge, re).repeat(32, axis=1) - 127)
    assert (np.abs(gv - rv) <= 2 * scale).all()
    assert (gv == rv).mean() > 0.99, (gv == rv).mean()
    # values agree with the oracle's float64 compression within the grid
    assert (np.abs(gv - ref) <= 2 * scale).all()


def _indexer_case(B, n_q, E, hI, cI, m, pos, seed):
    qI, qs, wI = e4m3_queries(seed, B, n_q, hI, cI)
    packed, exps = fp4_keys(seed + 1, B * E, cI)
    kent = Entries(packed.to(DEV), cI, scale=exps.to(DEV), scale_group=32, fp4=True)
    q_pos = torch.as_tensor(pos, dtype=torch.int64).view(B, n_q)
    scores = torch.full((B, n_q, E), float("nan"), device=DEV)
    abi.csa_indexer_scores(qI.to(DEV), qs.to(DEV), wI.to(DEV), kent, q_pos.to(DEV), m, scores, E)
    abi.csa_get_error()
    qv = oracle.dequantize(qI, qs.reshape(B, n_q, hI, 1), cI)
    kv = oracle.dequantize_e2m1(packed, exps).reshape(B, E, cI)
    ref = oracle.indexer(qv, oracle.f64(wI), kv, q_pos.numpy(), m)
    S = score_scale(qv, oracle.f64(wI), np.abs(kv).max())
    got = scores.cpu().double().numpy()
    for b in range(B):
        for t in range(n_q):
            V = oracle.visible(int(q_pos[b, t]), m, E)
            d = np.abs(got[b, t, :V] - ref[b, t, :V])
            assert (d <= SCORE_REL * S[b, t] + 1e-30).all(), (b, t, d.max(), S[b, t])
            assert np.isnan(got[b, t, V:]).all(), "entries past V_t must not be written"


@pytest.mark.parametrize("n,E,hI,cI", [
    (1000, 250, 64, 128),       # tensor-core path, 16-token blocks
    (640, 3000, 16, 128),       # h16
    (512, 2000, 32, 128),       # h32, two token groups per block
    (300, 75, 16, 64),          # c_I = 64: the CUDA-core path
])
def test_indexer_fp4_keys_prefill(n, E, hI, cI):
    _indexer_case(1, n, E, hI, cI, 4, np.arange(n) * max(1, (4 * E) // n), 61)


def test_indexer_fp4_keys_decode_batches():
    B, E = 3, 20000
    pos = np.array([4 * E - 1, 4 * 15000 + 2, 4 * E - 1])
    _indexer_case(B, 1, E, 64, 128, 4, pos, 62)


def test_indexer_topk_fp4_keys():
    # the candidate path (whole rows per block) and the two plain calls
    # select the same entries; the oracle's scores confirm the boundary
    B, n_q, E, hI, cI, m, k = 1, 4800, 16384, 64, 128, 4, 1024
    assert abi.csa_indexer_topk_launches(B, n_q, E, hI, cI, k, abi.CSA_E4M3) == 6
    qI, qs, wI = e4m3_queries(63, B, n_q, hI, cI)
    packed, exps = fp4_keys(64, E, cI)
    kent = Entries(packed.to(DEV), cI, scale=exps.to(DEV), scale_group=32, fp4=True)
    pos = np.sort(np.linspace(0, m * E - 1, n_q).astype(np.int64))
    q_pos = torch.as_tensor(pos).view(B, n_q).to(DEV)
    nws = abi.csa_indexer_topk_workspace_size(B, n_q, E, hI, cI, k, qI)
    ws = torch.empty(nws, device=DEV, dtype=torch.uint8)
    got = torch.full((n_q, k), -7, device=DEV, dtype=torch.int32)
    abi.csa_indexer_topk(qI.to(DEV), qs.to(DEV), wI.to(DEV), kent, q_pos, m, k, got, E,
                         workspace=ws)
    abi.csa_get_error()
    del ws
    scores = torch.empty(B, n_q, E, device=DEV)
    abi.csa_indexer_scores(qI.to(DEV), qs.to(DEV), wI.to(DEV), kent, q_pos, m, scores, E)
    two = torch.empty_like(got)
    abi.csa_topk(scores.view(n_q, E), q_pos.view(-1), m, k, two, E)
    abi.csa_get_error()
    np.testing.assert_array_equal(got.cpu().numpy(), two.cpu().numpy())
    # boundary check on sampled rows against the oracle's float64 scores
    qv = oracle.dequantize(qI, qs.reshape(B, n_q, hI, 1), cI)
    kv = oracle.dequantize_e2m1(packed, exps).reshape(B, E, cI)
    S = score_scale(qv, oracle.f64(wI), np.abs(kv).max())
    g = got.cpu().numpy()
    for r in list(range(0, n_q, 397)) + [n_q - 1]:
        ref = oracle.indexer(qv[:, r:r + 1], oracle.f64(wI)[:, r:r + 1], kv, pos[r:r + 1][None],
                             m)[0, 0]
        V = oracle.visible(int(pos[r]), m, E)
        if V <= k:
            assert (g[r, :V] == np.arange(V)).all() and (g[r, V:] == -1).all()
            continue
        sel = g[r]
        row = ref[:V]
        kth = np.partition(row, V - k)[V - k]
        tol = 2 * SCORE_REL * S[0, r]
        assert np.isin(np.nonzero(row > kth + tol)[0], sel).all(), r
        assert not np.isin(np.nonzero(row < kth - tol)[0], sel).any(), r
