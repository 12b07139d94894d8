"""Pins of the float64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a closed form
(mean pooling, one-hot selection, weights summing to one), a library routine
(numpy matmul, scipy softmax, torch scaled-dot-product attention and
logsumexp, torch's float8 cast, Python's sort), an invariant (additivity over
heads, order invariance, causality) or a fixture under ``tests/golden``. Each
is chosen so that a plausible slip in the oracle (a shifted window, a swapped
operand, a dropped term, a wrong sign, a missing max-subtraction, an
off-by-one in visibility) fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import pipeline
from conftest import golden_rows
from long_context_sparse_07_b200 import workloads as W


def rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------- compression


@pytest.mark.parametrize("m", [1, 2, 4])
def test_compress_equal_logits_is_mean_of_2m_rows(m):
    # Softmax over the 2m positions with equal logits gives weight 1/(2m):
    # entry i is the plain mean of Ca rows m*i.. and Cb rows m*(i-1)..
    # (entry 0: the mean of its m Ca rows only).
    g = rng(m)
    n, c = 16 * m, 8
    Ca, Cb = g.standard_normal((n, c)), g.standard_normal((n, c))
    Z = np.zeros((n, c))
    B = np.zeros((m, c))
    out = oracle.compress(Ca, Cb, Z, Z, B, B, m, True)
    E = n // m
    want = np.empty((E, c))
    want[0] = Ca[:m].mean(0)
    for i in range(1, E):
        want[i] = np.concatenate([Ca[m * i:m * i + m], Cb[m * (i - 1):m * i]]).mean(0)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)


def test_compress_onehot_follows_golden_windows():
    # A logit of +60 on one row of one window makes the softmax one-hot, so
    # the entry returns that row: this reads back, per channel, exactly which
    # Ca / Cb rows feed entry i (fixture from the overlapping-window text).
    m, c = 4, 2 * 4
    rows = [list(map(int, r)) for r in golden_rows("overlap_windows_m4.txt")]
    n = m * (len(rows))
    g = rng(7)
    Ca, Cb = g.standard_normal((n, c)), g.standard_normal((n, c))
    B = np.zeros((m, c))
    for i, a0, a1, b0, b1 in rows:
        for r in range(m):
            # channel r: one-hot on Ca row a0 + r; channel m + r: on Cb row b0 + r
            Za = np.full((n, c), -60.0)
            Zb = np.full((n, c), -60.0)
            Za[a0 + r, r] = 60.0
            if b0 >= 0:
                Zb[b0 + r, m + r] = 60.0
            else:
                Za[a0 + r, m + r] = 60.0          # entry 0 has no b-window
            out = oracle.compress(Ca, Cb, Za, Zb, B, B, m, True)
            assert a1 - a0 + 1 == m
            assert abs(out[i, r] - Ca[a0 + r, r]) < 1e-12
            want = Cb[b0 + r, m + r] if b0 >= 0 else Ca[a0 + r, m + r]
            assert abs(out[i, m + r] - want) < 1e-12


def test_compress_weights_sum_to_one():
    # With every KV value equal to 1 the entry equals the sum of its softmax
    # weights, which must be exactly one for any logits and biases.
    g = rng(3)
    n, c, m = 64, 16, 4
    ones = np.ones((n, c))
    Za, Zb = 3 * g.standard_normal((n, c)), 3 * g.standard_normal((n, c))
    Ba, Bb = g.standard_normal((m, c)), g.standard_normal((m, c))
    out = oracle.compress(ones, ones, Za, Zb, Ba, Bb, m, True)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=2e-15)


def test_compress_bias_only_matches_scipy_softmax():
    # With Z = 0 the weights are softmax([Ba; Bb]) per channel (scipy), the
    # same for every entry i >= 1; entry 0 uses softmax(Ba).
    g = rng(4)
    n, c, m = 32, 6, 4
    Ca, Cb = g.standard_normal((n, c)), g.standard_normal((n, c))
    Ba, Bb = g.standard_normal((m, c)), g.standard_normal((m, c))
    Z = np.zeros((n, c))
    out = oracle.compress(Ca, Cb, Z, Z, Ba, Bb, m, True)
    wab = scipy.special.softmax(np.concatenate([Ba, Bb]), axis=0)
    wa0 = scipy.special.softmax(Ba, axis=0)
    np.testing.assert_allclose(out[0], (wa0 * Ca[:m]).sum(0), atol=1e-14)
    for i in range(1, n // m):
        win = np.concatenate([Ca[m * i:m * i + m], Cb[m * (i - 1):m * i]])
        np.testing.assert_allclose(out[i], (wab * win).sum(0), atol=1e-14)


def test_compress_large_logits_stay_finite_and_shift_invariant():
    g = rng(5)
    n, c, m = 16, 4, 4
    Ca, Cb = g.standard_normal((n, c)), g.standard_normal((n, c))
    Za, Zb = g.standard_normal((n, c)), g.standard_normal((n, c))
    B = g.standard_normal((m, c))
    base = oracle.compress(Ca, Cb, Za, Zb, B, B, m, True)
    big = oracle.compress(Ca, Cb, Za + 1000.0, Zb + 1000.0, B, B, m, True)
    assert np.isfinite(big).all()
    np.testing.assert_allclose(big, base, atol=1e-12)


def test_hca_equal_logits_is_block_mean():
    # Eq. 20-23 without overlap, m' = 128: plain mean of each 128-row block.
    g = rng(6)
    n, c, m = 512, 8, 128
    C = g.standard_normal((n, c))
    out = oracle.compress(C, None, np.zeros((n, c)), None, np.zeros((m, c)), None, m, False)
    np.testing.assert_allclose(out, C.reshape(n // m, m, c).mean(1), atol=1e-14)


def test_hca_ignores_second_window():
    g = rng(8)
    n, c, m = 64, 4, 16
    C, Z = g.standard_normal((n, c)), g.standard_normal((n, c))
    B = g.standard_normal((m, c))
    a = oracle.compress(C, g.standard_normal((n, c)), Z, g.standard_normal((n, c)), B,
                        g.standard_normal((m, c)), m, False)
    b = oracle.compress(C, None, Z, None, B, None, m, False)
    np.testing.assert_array_equal(a, b)
    w = scipy.special.softmax(Z.reshape(n // m, m, c) + B[None], axis=1)
    np.testing.assert_allclose(b, (w * C.reshape(n // m, m, c)).sum(1), atol=1e-14)


# ------------------------------------------------------------------- e4m3


def test_e4m3_values_match_torch_decode_for_every_code():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(i) for i in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_rounding_matches_torch_cast():
    g = rng(9)
    x = np.concatenate([g.standard_normal(4000) * 100, g.standard_normal(2000) * 0.01,
                        np.array([448, 449, 464, 465, 1e6, -1e6, 0.0, -0.0, 2.0 ** -10,
                                  3 * 2.0 ** -10, 1.0625, 1.1875])])
    want = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float32).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_code(v) for v in x.astype(np.float32).astype(np.float64)],
                   dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


def test_quantize_maps_row_amax_to_448_and_bounds_error():
    g = rng(10)
    x = g.standard_normal((50, 128)) * 3
    codes, scales = oracle.quantize_e4m3(x, 128)
    deq = oracle.dequantize(codes, scales, 128)
    amax_col = np.abs(x).argmax(1)
    assert all(abs(oracle.e4m3_value(codes[r, amax_col[r]])) == 448.0 for r in range(50))
    # scale = float32(amax) / 448 in float32 arithmetic (numpy float32 division)
    amax32 = np.abs(x).astype(np.float32).max(1, keepdims=True)
    np.testing.assert_array_equal(scales, amax32 / np.float32(448))
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the normal range
    big = np.abs(x) > scales * 2.0 ** -6
    assert (np.abs(deq - x)[big] <= np.abs(x)[big] * 2.0 ** -4 + 1e-12).all()


# ------------------------------------------------------------------ indexer


def test_visibility_matches_golden_table():
    for t, v in golden_rows("visibility_m4.txt"):
        assert oracle.visible(int(t), 4, 1 << 20) == int(v)


def test_indexer_single_head_is_relu_of_matmul():
    g = rng(11)
    n, E, cI, m = 40, 10, 16, 4
    q = g.standard_normal((1, n, 1, cI))
    k = g.standard_normal((1, E, cI))
    w = np.ones((1, n, 1))
    pos = np.arange(n)[None]
    s = oracle.indexer(q, w, k, pos, m)[0]
    ref = np.maximum(q[0, :, 0, :] @ k[0].T, 0.0)
    for t in range(n):
        V = (t + 1) // m
        np.testing.assert_allclose(s[t, :V], ref[t, :V], atol=1e-12)
        assert np.isneginf(s[t, V:]).all()


def test_indexer_is_additive_over_heads_and_odd_in_w():
    g = rng(12)
    B, n, E, hI, cI, m = 2, 24, 6, 6, 8, 4
    q = g.standard_normal((B, n, hI, cI))
    k = g.standard_normal((B, E, cI))
    w = g.standard_normal((B, n, hI))
    pos = np.tile(np.arange(n), (B, 1))
    full = oracle.indexer(q, w, k, pos, m)
    a = oracle.indexer(q[:, :, :3], w[:, :, :3], k, pos, m)
    b = oracle.indexer(q[:, :, 3:], w[:, :, 3:], k, pos, m)
    fin = np.isfinite(full)
    np.testing.assert_allclose(full[fin], (a + b)[fin], atol=1e-12)
    neg = oracle.indexer(q, -w, k, pos, m)
    np.testing.assert_allclose(neg[fin], -full[fin], atol=1e-12)
    # batches use their own keys: swapping key sets swaps scores
    sw = oracle.indexer(q[::-1].copy(), w[::-1].copy(), k[::-1].copy(), pos, m)
    np.testing.assert_array_equal(sw, full[::-1])


def test_indexer_relu_drops_negative_dot_products():
    q = np.array([[[[1.0, 0.0]], [[1.0, 0.0]], [[1.0, 0.0]], [[1.0, 0.0]]]])  # [1,4,1,2]
    k = np.array([[[-2.0, 5.0]]])                                           # q.k = -2
    w = np.ones((1, 4, 1))
    s = oracle.indexer(q, w, k, np.arange(4)[None], 4)
    assert s[0, 3, 0] == 0.0 and np.isneginf(s[0, 2, 0])


# -------------------------------------------------------------------- top-k


def _brute_topk(row, V, k):
    order = sorted(range(V), key=lambda s: (-(row[s] + 0.0), s))[:k]
    return sorted(order) + [-1] * (k - min(k, V))


@pytest.mark.parametrize("k", [1, 5, 16, 40])
def test_topk_matches_brute_force_sort(k):
    rows, E, m = 33, 32, 1
    sc = W.score_rows(5, rows, E).double().numpy()
    pos = np.arange(rows) - 1          # V = pos + 1 = 0 .. 32 (m = 1)
    got = oracle.topk(sc, pos, m, k)
    for r in range(rows):
        V = max(0, min(E, (pos[r] + 1) // m))
        assert got[r].tolist() == _brute_topk(sc[r], V, k)


def test_topk_ties_prefer_lower_index_and_signed_zeros_tie():
    sc = np.array([[1.0, 2.0, 2.0, 0.0, -0.0, 2.0, 0.0, -1.0]])
    got = oracle.topk(sc, [7], 1, 4)
    assert got[0].tolist() == [0, 1, 2, 5]
    got = oracle.topk(sc, [7], 1, 6)
    assert got[0].tolist() == [0, 1, 2, 3, 4, 5]


def test_topk_pads_short_rows():
    sc = np.array([[3.0, 1.0, 2.0, 9.0]])
    assert oracle.topk(sc, [2], 1, 5)[0].tolist() == [0, 1, 2, -1, -1]
    assert oracle.topk(sc, [0], 4, 3)[0].tolist() == [-1, -1, -1]


# ---------------------------------------------------------------- attention


def _sdpa(q, keys, mask):
    """torch reference: softmax(q k^T / sqrt(c)) k with a boolean mask."""
    qt = torch.from_numpy(q)[None]               # [1, h, L, c]
    kt = torch.from_numpy(keys)[None, None]      # [1, 1, S, c]
    kt = kt.expand(1, q.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, kt, attn_mask=torch.from_numpy(mask)[None, None])[0].numpy()


def test_attention_dense_no_window_no_sink_is_textbook_softmax():
    g = rng(13)
    n, E, h, c, m = 20, 5, 3, 8, 4
    ent = g.standard_normal((1, E, c))
    q = g.standard_normal((1, n, h, c))
    out, _ = oracle.attend(q, ent, None, 0, m, None, [0], 0, np.arange(n)[None],
                           np.full(h, -np.inf), 1 / math.sqrt(c))
    for t in range(m - 1, n):        # rows with at least one visible entry
        V = (t + 1) // m
        mask = np.zeros((1, E), dtype=bool)
        mask[0, :V] = True
        ref = _sdpa(q[0, t][:, None, :], ent[0], mask)[:, 0, :]
        np.testing.assert_allclose(out[0, t], ref, atol=1e-12)
    assert (out[0, :m - 1] == 0).all()


def test_attention_window_only_is_sliding_window_attention():
    g = rng(14)
    n, h, c, W_ = 24, 2, 8, 5
    kwin = g.standard_normal((1, n, c))
    q = g.standard_normal((1, n, h, c))
    idx = -np.ones((n, 3), dtype=np.int32)          # nothing selected
    out, _ = oracle.attend(q, np.zeros((1, 1, c)), idx, 3, 4, kwin, [0], W_,
                           np.arange(n)[None], np.full(h, -np.inf), 1 / math.sqrt(c))
    i = np.arange(n)
    band = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W_)
    qt = torch.from_numpy(q[0].transpose(1, 0, 2))          # [h, n, c]
    kt = torch.from_numpy(kwin[0])[None].expand(h, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, kt, attn_mask=torch.from_numpy(band)).numpy().transpose(1, 0, 2)
    np.testing.assert_allclose(out[0], ref, atol=1e-12)


def test_attention_sink_rescales_by_logsumexp():
    # With a finite sink the weights are the sink-free ones times
    # 1 / (1 + exp(z' - lse)), and lse gains the sink term (torch.logsumexp).
    g = rng(15)
    E, h, c, m, k = 12, 4, 16, 1, 5
    ent = g.standard_normal((1, E, c))
    q = g.standard_normal((1, 1, h, c))
    idx = np.array([[1, 3, 4, 7, 11]], dtype=np.int32)
    pos = [[11]]
    sink = g.standard_normal(h)
    scale = 1 / math.sqrt(c)
    o0, l0 = oracle.attend(q, ent, idx, k, m, None, [0], 0, pos, np.full(h, -np.inf), scale)
    o1, l1 = oracle.attend(q, ent, idx, k, m, None, [0], 0, pos, sink, scale)
    logits = torch.from_numpy(scale * q[0, 0] @ ent[0, idx[0]].T)        # [h, k]
    lse0 = torch.logsumexp(logits, dim=1).numpy()
    lse1 = torch.logsumexp(torch.cat([logits, torch.from_numpy(sink)[:, None]], 1), 1).numpy()
    np.testing.assert_allclose(l0[0, 0], lse0, atol=1e-12)
    np.testing.assert_allclose(l1[0, 0], lse1, atol=1e-12)
    factor = 1.0 / (1.0 + np.exp(sink - lse0))
    np.testing.assert_allclose(o1[0, 0], o0[0, 0] * factor[:, None], atol=1e-12)
    o2, l2 = oracle.attend(q, ent, idx, k, m, None, [0], 0, pos, np.full(h, np.inf), scale)
    assert (o2 == 0).all() and np.isposinf(l2).all()


def test_attention_selection_order_is_irrelevant_and_full_selection_is_dense():
    g = rng(16)
    n, E, h, c, m, Wn = 32, 8, 2, 8, 4, 3
    ent = g.standard_normal((1, E, c))
    kwin = g.standard_normal((1, n, c))
    q = g.standard_normal((1, n, h, c))
    sink = g.standard_normal(h)
    pos = np.arange(n)[None]
    k = E
    idx = np.array([list(range((t + 1) // m)) + [-1] * (k - (t + 1) // m) for t in range(n)],
                   dtype=np.int32)
    a, la = oracle.attend(q, ent, idx, k, m, kwin, [0], Wn, pos, sink, 0.3)
    perm = np.array([g.permutation(r) for r in idx], dtype=np.int32)
    b, lb = oracle.attend(q, ent, perm, k, m, kwin, [0], Wn, pos, sink, 0.3)
    d, ld = oracle.attend(q, ent, None, 0, m, kwin, [0], Wn, pos, sink, 0.3)
    np.testing.assert_allclose(a, b, atol=1e-13)
    np.testing.assert_allclose(a, d, atol=1e-13)
    np.testing.assert_allclose(la, ld, atol=1e-13)


def test_attention_rejects_invisible_selection():
    ent = np.zeros((1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attend(np.zeros((1, 1, 1, 2)), ent, np.array([[1]], np.int32), 1, 4, None,
                      [0], 0, [[3]], np.zeros(1), 1.0)      # V = 1: entry 1 is future


# ------------------------------------------------------------------ pipeline


def test_pipeline_is_causal():
    # Changing every operand of tokens after t leaves outputs up to t exactly
    # unchanged: no entry holding a future token is visible, and the window
    # never reaches past t.
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=64)
    ops = W.csa_operands(w)
    base = pipeline.csa_prefill(ops, w)
    t = 37
    g = rng(17)
    ops2 = {k: v.clone() for k, v in ops.items()}
    for key in ("Ca", "Cb", "Za", "Zb", "CIa", "CIb", "ZIa", "ZIb", "qI", "wI", "q"):
        x = ops2[key]
        x[t + 1:] = torch.from_numpy(g.standard_normal(tuple(x[t + 1:].shape))).to(x.dtype)
    pert = pipeline.csa_prefill(ops2, w)
    np.testing.assert_array_equal(base["out"][:t + 1], pert["out"][:t + 1])
    np.testing.assert_array_equal(base["idx"][:t + 1], pert["idx"][:t + 1])
    assert not np.array_equal(base["out"][t + 1:], pert["out"][t + 1:])


def test_pipeline_topk_at_least_visible_equals_dense_attention():
    # k >= every V_t: the selection keeps every visible entry and CSA equals
    # the dense (HCA-style) attention over the same entries.
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=48, k=16)
    ops = W.csa_operands(w)
    res = pipeline.csa_prefill(ops, w)
    d, ld = oracle.attend(oracle.f64(ops["q"])[None], res["entries"][None], None, 0, w.m,
                          oracle.f64(ops["Ca"])[None], [0], w.n_win,
                          np.arange(w.n)[None], ops["sink"], 1 / math.sqrt(w.c))
    np.testing.assert_allclose(res["out"], d[0], atol=1e-13)


def test_golden_configuration_matches_flash_workload_shapes():
    cfg = {k: int(v) for k, v in golden_rows("configurations.txt")}
    w = W.WORKLOADS["csa_fp8idx_n131072"]
    assert (w.m, w.hI, w.cI, w.h, w.c, w.n_win) == (
        cfg["m"], cfg["indexer_heads"], cfg["indexer_head_dim"], cfg["query_heads"],
        cfg["head_dim"], cfg["n_win"])
    assert W.WORKLOADS["hca_bf16_n65536"].m == cfg["hca_ratio"]
    assert W.WORKLOADS["decode_b8_ctx1m"].rope_dims == cfg["rope_dims"]
