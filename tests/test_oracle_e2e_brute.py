"""End-to-end pins of the oracle's CSA and HCA prefills against a brute force.

The brute force below restates the whole chain in plain Python (scalar loops,
``math``): overlapping compression (CSA Eq. 9-12, the first entry taking its
m own rows only), the indexer (Eq. 16) over visible entries, the top-k of
Eq. 17 (ties to the lower index), and shared-KV attention over the selected
entries, the sliding window (self included) and the sink (Eq. 18-19, Module
D). It stores intermediates at the same points and in the same precision as
the path (entries and index scores rounded to float32) and shares nothing with
``oracle/`` but the inputs. Tiny sequences, m in {1, 2, 4} and k in {1, V, more
than V} cover the cases where a composition slip (visibility off by one, the
window start, the sink in the max, an index-order mistake) would show. The
HCA brute force does the same with non-overlapping blocks (Eq. 20-23) and
every visible entry (Eq. 24-26); the decode one reads the fp8 caches (codes
decoded by torch, times their group scales, then the bf16 RoPE dims; Module F)
and the window buffer by position.
"""
import math

import numpy as np
import pytest

from oracle import pipeline
from long_context_sparse_07_b200 import workloads as W


def f32(x):
    return float(np.float32(x))


def softmax_pool(logits, rows):
    mx = max(logits)
    ws = [math.exp(l - mx) for l in logits]
    tot = sum(ws)
    return sum(w * r for w, r in zip(ws, rows)) / tot


def compress_bf(Ca, Cb, Za, Zb, Ba, Bb, m):
    n, c = len(Ca), len(Ca[0])
    E = n // m
    out = []
    for i in range(E):
        row = []
        for j in range(c):
            logits = [Za[m * i + r][j] + Ba[r][j] for r in range(m)]
            vals = [Ca[m * i + r][j] for r in range(m)]
            if i > 0:
                logits += [Zb[m * (i - 1) + r][j] + Bb[r][j] for r in range(m)]
                vals += [Cb[m * (i - 1) + r][j] for r in range(m)]
            row.append(f32(softmax_pool(logits, vals)))
        out.append(row)
    return out


def visible(t, m, E):
    return min(E, (t + 1) // m)


def brute_csa(ops, w):
    L = {k: v.double().numpy().tolist() for k, v in ops.items()}
    m, k, W_ = w.m, w.k, w.n_win
    ent = compress_bf(L["Ca"], L["Cb"], L["Za"], L["Zb"], L["Ba"], L["Bb"], m)
    kI = compress_bf(L["CIa"], L["CIb"], L["ZIa"], L["ZIb"], L["BIa"], L["BIb"], m)
    E = len(ent)
    scale = 1.0 / math.sqrt(w.c)
    outs, lses, sels = [], [], []
    for t in range(w.n):
        V = visible(t, m, E)
        scores = []
        for s in range(V):
            acc = 0.0
            for hh in range(w.hI):
                dot = sum(L["qI"][t][hh][x] * kI[s][x] for x in range(w.cI))
                acc += L["wI"][t][hh] * max(0.0, dot)
            scores.append(f32(acc))
        order = sorted(range(V), key=lambda s: (-scores[s], s))
        sel = sorted(order[:min(k, V)])
        sels.append(sel + [-1] * (k - len(sel)))
        keys = [ent[s] for s in sel] + [L["Ca"][p] for p in range(max(0, t - W_ + 1), t + 1)]
        o_t, l_t = [], []
        for hh in range(w.h):
            q = L["q"][t][hh]
            z = [scale * sum(q[x] * key[x] for x in range(w.c)) for key in keys]
            zs = L["sink"][hh]
            M = max(z + [zs])
            e = [math.exp(v - M) for v in z]
            den = sum(e) + math.exp(zs - M)
            o_t.append([sum(e[j] * keys[j][x] for j in range(len(keys))) / den for x in range(w.c)])
            l_t.append(M + math.log(den))
        outs.append(o_t)
        lses.append(l_t)
    return np.array(ent), np.array(sels), np.array(outs), np.array(lses)


@pytest.mark.parametrize("m,k", [(1, 1), (2, 3), (4, 2), (4, 16), (2, 40)])
def test_csa_prefill_matches_brute_force(m, k):
    # n = 24 tokens: with m = 4, V_t runs 0..6 so k = 2 < V, k = 16 > V; with
    # m = 2 and k = 40 every query takes all visible entries
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=24, c=8, m=m, hI=2, cI=4, k=k, n_win=3,
                 h=2, seed=11 + m + k)
    ops = W.csa_operands(w)
    ent, sel, out, lse = brute_csa(ops, w)
    res = pipeline.csa_prefill(ops, w)
    np.testing.assert_allclose(res["entries"], ent, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(res["idx"], sel)
    np.testing.assert_allclose(res["out"], out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-12, atol=1e-12)


def brute_hca(ops, w):
    L = {k: v.double().numpy().tolist() for k, v in ops.items()}
    m, W_ = w.m, w.n_win
    n, c = len(L["C"]), len(L["C"][0])
    ent = []
    for i in range(n // m):                     # no overlap: block i alone (Eq. 20-23)
        ent.append([f32(softmax_pool([L["Z"][m * i + r][j] + L["B"][r][j] for r in range(m)],
                                     [L["C"][m * i + r][j] for r in range(m)]))
                    for j in range(c)])
    E = len(ent)
    scale = 1.0 / math.sqrt(w.c)
    outs, lses = [], []
    for t in range(w.n):
        keys = ent[:visible(t, m, E)] + [L["C"][p] for p in range(max(0, t - W_ + 1), t + 1)]
        o_t, l_t = [], []
        for hh in range(w.h):
            q = L["q"][t][hh]
            z = [scale * sum(q[x] * key[x] for x in range(w.c)) for key in keys]
            zs = L["sink"][hh]
            M = max(z + [zs])
            e = [math.exp(v - M) for v in z]
            den = sum(e) + math.exp(zs - M)
            o_t.append([sum(e[j] * keys[j][x] for j in range(len(keys))) / den for x in range(w.c)])
            l_t.append(M + math.log(den))
        outs.append(o_t)
        lses.append(l_t)
    return np.array(ent), np.array(outs), np.array(lses)


@pytest.mark.parametrize("m", [1, 3, 8])
def test_hca_prefill_matches_brute_force(m):
    w = W.scaled(W.WORKLOADS["hca_bf16_n65536"], n=24, c=8, m=m, n_win=4, h=2, dtype="f32",
                 seed=31 + m)
    ops = W.hca_operands(w)
    ent, out, lse = brute_hca(ops, w)
    res = pipeline.hca_prefill(ops, w)
    np.testing.assert_allclose(res["entries"], ent, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["out"], out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-12, atol=1e-12)


def e4m3(codes):
    """e4m3 codes (uint8 tensor) to float64 values by torch's own decoder."""
    import torch
    return codes.contiguous().view(torch.float8_e4m3fn).to(torch.float64).numpy().tolist()


def attend_bf(q, keys, zs, scale):
    z = [scale * sum(qx * kx for qx, kx in zip(q, key)) for key in keys]
    M = max(z + [zs])
    e = [math.exp(v - M) for v in z]
    den = sum(e) + math.exp(zs - M)
    c = len(q)
    return [sum(e[j] * keys[j][x] for j in range(len(keys))) / den for x in range(c)], \
        M + math.log(den)


def brute_decode(ops, w):
    scale = 1.0 / math.sqrt(w.c)
    G = w.scale_group
    sink = ops["sink"].double().tolist()
    res = {"idx": [], "out": [], "lse": [], "hca_out": [], "hca_lse": [], "scores": []}
    for b in range(w.batch):
        t = int(ops["q_pos"][b, 0])
        qI_c, kI_c = e4m3(ops["qI"][b, 0]), e4m3(ops["kI"][b])
        qs, ks = ops["qI_scale"][b, 0].double().tolist(), ops["kI_scale"][b].double().tolist()
        wI = ops["wI"][b, 0].double().tolist()
        E = len(kI_c)
        V = visible(t, w.m, E)
        sc = []
        for s in range(V):
            acc = 0.0
            for hh in range(w.hI):
                dot = sum(qI_c[hh][x] * qs[hh] * kI_c[s][x] * ks[s] for x in range(w.cI))
                acc += wI[hh] * max(0.0, dot)
            sc.append(f32(acc))
        order = sorted(range(V), key=lambda s: (-sc[s], s))
        sel = sorted(order[:min(w.k, V)])
        res["scores"].append(sc)
        res["idx"].append(sel + [-1] * (w.k - len(sel)))

        def entry(pre, s):
            body = e4m3(ops[pre + "_nope"][b, s])
            scl = ops[pre + "_scale"][b, s].double().tolist()
            return [body[x] * scl[x // G] for x in range(len(body))] + \
                ops[pre + "_rope"][b, s].double().tolist()

        p0 = int(ops["win_pos0"][b])
        win = [ops["kwin"][b, p - p0].double().tolist() for p in range(max(0, t - w.n_win + 1), t + 1)]
        q = ops["q"][b, 0].double().tolist()
        keys = [entry("kv", s) for s in sel] + win
        Eh = ops["hca_nope"].shape[1]
        hkeys = [entry("hca", s) for s in range(visible(t, w.m_hca, Eh))] + win
        o, l, ho, hl = [], [], [], []
        for hh in range(w.h):
            oo, ll = attend_bf(q[hh], keys, sink[hh], scale)
            o.append(oo)
            l.append(ll)
            oo, ll = attend_bf(q[hh], hkeys, sink[hh], scale)
            ho.append(oo)
            hl.append(ll)
        res["out"].append([o])
        res["lse"].append([l])
        res["hca_out"].append([ho])
        res["hca_lse"].append([hl])
    return res


def test_decode_matches_brute_force():
    # two sequences of 64 tokens: 16 CSA entries (k = 4 of them), 8 HCA
    # entries (m' = 8), a 4-row window, fp8 split-layout caches
    w = W.scaled(W.WORKLOADS["decode_b8_ctx1m"], n=64, batch=2, hI=2, cI=32, k=4, n_win=4,
                 h=2, m_hca=8, seed=41)
    ops = W.decode_operands(w)
    bf = brute_decode(ops, w)
    res = pipeline.decode(ops, w)
    for b in range(w.batch):
        V = len(bf["scores"][b])
        # both round a float64 sum to float32; the sums may differ in their
        # last bits (summation order), so allow one float32 step
        np.testing.assert_allclose(res["scores"][b, :V], bf["scores"][b], rtol=2 ** -23, atol=0)
    np.testing.assert_array_equal(res["idx"], np.array(bf["idx"]))
    for key in ("out", "lse", "hca_out", "hca_lse"):
        np.testing.assert_allclose(np.asarray(res[key]), np.array(bf[key]), rtol=1e-12,
                                   atol=1e-12, err_msg=key)
