"""Pins of the whole-layer oracle (``oracle/layer.py``): the path's operands
as projections of the hidden state H (Module B steps 1-3: Eq. 9-10, 13-15,
18), then the chain of steps.

* With H and the query latent both identity matrices, every projection is the
  weight itself, read back exactly: this fixes which weight feeds which
  operand and the [token, head, dim] order of the query reshapes.
* On a tiny layer, projections written as plain Python loops followed by the
  plain-Python chain of ``test_oracle_e2e_brute`` give the oracle's entries,
  selections, outputs and log-sum-exps.
* The projected operands carry the correlation that a shared H gives them:
  with W^{bKV} = W^{aKV}, C^b equals C^a row for row.
"""
import math

import numpy as np
import pytest
import torch

from oracle import layer
from long_context_sparse_07_b200 import workloads as W
from test_oracle_e2e_brute import brute_csa


def tiny(n=24, d=6, dc=5, m=2, k=3, seed=5):
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=n, c=8, m=m, hI=2, cI=4, k=k, n_win=3, h=2,
                 seed=seed, name="tiny_layer")
    L = W.Layer(d=d, dc=dc, std_w=None, std_bias=0.3)
    return w, W.layer_draws(w, L)


def test_identity_hidden_state_reads_back_the_weights():
    w, dr = tiny(n=6, d=6, dc=6)
    dr["H"] = np.eye(6, dtype=np.float32)
    dr["W_DQ"] = np.eye(6, dtype=np.float32)
    ops = layer.layer_operands(dr, w)
    for a, b in (("Ca", "W_aKV"), ("Cb", "W_bKV"), ("Za", "W_aZ"), ("Zb", "W_bZ"),
                 ("CIa", "W_aKI"), ("CIb", "W_bKI"), ("ZIa", "W_aZI"), ("ZIb", "W_bZI"),
                 ("wI", "W_w")):
        assert np.array_equal(ops[a].numpy(), dr[b]), a
    # q[t, head, dim] = W_UQ[t, head * c + dim]; the same for q^I
    assert np.array_equal(ops["q"].numpy(), dr["W_UQ"].reshape(6, w.h, w.c))
    assert np.array_equal(ops["qI"].numpy(), dr["W_IUQ"].reshape(6, w.hI, w.cI))
    assert np.array_equal(ops["q"][2, 1].numpy(), dr["W_UQ"][2, w.c:2 * w.c])


def matmul_loops(A, B):
    return [[sum(A[i][p] * B[p][j] for p in range(len(B))) for j in range(len(B[0]))]
            for i in range(len(A))]


@pytest.mark.parametrize("m,k", [(2, 3), (4, 1), (1, 40)])
def test_tiny_layer_matches_loops_and_brute_chain(m, k):
    w, dr = tiny(m=m, k=k, seed=7 + m + k)
    L = {kk: np.asarray(v, dtype=np.float64).tolist() for kk, v in dr.items()}
    H = L["H"]
    P = {}
    for a, b in (("Ca", "W_aKV"), ("Cb", "W_bKV"), ("Za", "W_aZ"), ("Zb", "W_bZ"),
                 ("CIa", "W_aKI"), ("CIb", "W_bKI"), ("ZIa", "W_aZI"), ("ZIb", "W_bZI"),
                 ("wI", "W_w")):
        P[a] = matmul_loops(H, L[b])
    cQ = matmul_loops(H, L["W_DQ"])
    P["q"] = matmul_loops(cQ, L["W_UQ"])
    P["qI"] = matmul_loops(cQ, L["W_IUQ"])
    ops_bf = {kk: torch.tensor(v, dtype=torch.float64).to(torch.float32) for kk, v in P.items()}
    ops_bf["q"] = ops_bf["q"].view(w.n, w.h, w.c)
    ops_bf["qI"] = ops_bf["qI"].view(w.n, w.hI, w.cI)
    for kk in ("Ba", "Bb", "BIa", "BIb", "sink"):
        ops_bf[kk] = torch.from_numpy(np.asarray(dr[kk], dtype=np.float32))
    ops = layer.layer_operands(dr, w)
    for kk, v in ops_bf.items():
        # float64 sums in another order, then one rounding to float32: equal
        # except where a sum lands within a few float64 ulps of a rounding
        # boundary
        np.testing.assert_allclose(ops[kk].numpy(), v.numpy(), rtol=2e-7, atol=0)
    ent, sel, out, lse = brute_csa(ops_bf, w)
    res = layer.csa_layer(dr, w)
    np.testing.assert_allclose(res["entries"], ent, rtol=1e-6, atol=1e-7)
    np.testing.assert_array_equal(res["idx"], sel)
    np.testing.assert_allclose(res["out"], out, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-6, atol=1e-6)


def test_shared_hidden_state_correlates_the_operands():
    w, dr = tiny()
    dr["W_bKV"] = dr["W_aKV"].copy()
    ops = layer.layer_operands(dr, w)
    assert torch.equal(ops["Ca"], ops["Cb"])
    # and the drawn H is N(0, 1): the projections have the variance d * std_w^2
    w2 = W.WORKLOADS["csa_bf16_n4096"]
    L2 = W.LAYERS["csa_bf16_n4096"]
    ops2 = layer.layer_operands(W.layer_draws(W.scaled(w2, n=512), L2), W.scaled(w2, n=512))
    sd = float(ops2["Ca"].float().std())
    assert abs(sd - math.sqrt(L2.d) * L2.std_w) < 0.05 * math.sqrt(L2.d) * L2.std_w
