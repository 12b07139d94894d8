"""GPU parity of the Q/KV RMSNorm + partial RoPE step and the output rotation
(Module D), through the C ABI, against the oracle (float64 on the same input
bits, result compared in the storage dtype's tolerance)."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import pipeline
from long_context_sparse_07_b200 import abi, path, workloads as W
from helpers import assert_close_out, sample_rows, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def assert_elementwise(gpu, ref, dtype, what):
    """An elementwise step: every value within its storage rounding of the
    float64 result (bf16: half an ulp, 2^-9 relative, plus the float32
    arithmetic; f32: a few float32 ulps)."""
    rel = 2.0 ** -8 if dtype == "bf16" else 1e-5
    err = np.abs(gpu - ref)
    bound = rel * np.abs(ref) + 1e-6
    assert np.isfinite(gpu).all(), what
    assert (err <= bound).all(), "%s: worst error %.3g of the bound" % (
        what, (err / bound).max())


@pytest.mark.parametrize("dtype,c,heads,R,normalise", [
    ("bf16", 512, 64, 64, True),     # queries of the large workloads
    ("bf16", 512, 1, 64, True),      # compressed entries / window rows
    ("f32", 64, 4, 64, True),        # the small fp32 workload: every dim turns
    ("f32", 512, 8, 0, True),        # RMSNorm alone
    ("bf16", 512, 64, 64, False),    # rotation alone (the output's rotation back)
])
def test_norm_rope_matches_oracle(dtype, c, heads, R, normalise):
    rows = 300
    g = np.random.default_rng(31)
    x = W.to_storage(g.standard_normal((rows, heads * c)).astype(np.float32) * 3.0, dtype)
    x = x.view(rows, heads, c)
    gam = torch.from_numpy((0.5 + g.random(c)).astype(np.float32))
    pos = torch.as_tensor(np.concatenate([[0, 1, 2, 127, 128], g.integers(0, 1 << 20, rows - 5)]),
                          dtype=torch.int64)
    for mul, add in ((1, 0), (-1, 0), (4, 3)):
        ref = oracle.norm_rope(x, pos.numpy() * mul + add, R, gamma=gam if normalise else None,
                               normalise=normalise)
        xg = x.to(DEV).clone()
        abi.csa_norm_rope(xg, R, pos=pos.to(DEV), pos_mul=mul, pos_add=add,
                          gamma=gam.to(DEV) if normalise else None, normalise=normalise)
        abi.csa_get_error()
        assert_elementwise(to_np(xg), ref, dtype, "norm_rope %s mul %d" % (dtype, mul))
    # positions from the row number (entries: m * row + m - 1)
    ref = oracle.norm_rope(x, np.arange(rows) * 4 + 3, R, gamma=gam if normalise else None,
                           normalise=normalise)
    xg = x.to(DEV).clone()
    abi.csa_norm_rope(xg, R, pos=None, pos_mul=4, pos_add=3,
                      gamma=gam.to(DEV) if normalise else None, normalise=normalise)
    assert_elementwise(to_np(xg), ref, dtype, "norm_rope by row number")


@pytest.mark.parametrize("name,count", [("csa_fp32_n256", None), ("csa_bf16_n4096", 192)])
def test_csa_prefill_with_norm_rope_and_rotation_back(name, count):
    """The whole CSA step with Module D's normalisation and partial RoPE: the
    entries at their blocks' last tokens, the window rows and the queries at
    their positions, the output turned back by the query position."""
    w = W.WORKLOADS[name]
    R = 64
    ops = W.csa_operands(w)
    p = path.CsaPrefill(w, ops, rope_dims=R)
    p.step()
    abi.csa_get_error()
    rows = np.arange(w.n) if count is None else sample_rows(w.n, w.m, count, 9)
    ref = pipeline.csa_prefill_rope(ops, w, rows, rope_dims=R)
    # the rotated entries, window rows and queries themselves
    assert_close_out(to_np(p.entries.body), ref["entries"], w.dtype, "rotated entries")
    assert_close_out(to_np(p.kwin), ref["win"], w.dtype, "rotated window rows")
    sel = torch.as_tensor(rows, device=DEV)
    assert_close_out(to_np(p.d["q"][sel]), ref["q"], w.dtype, "rotated queries")
    # outputs on the GPU's own selection (a near tie cannot hide an error)
    gidx = p.idx[sel].cpu().numpy()
    o, _ = oracle.attend(ref["q"][None], ref["entries"][None], gidx, w.k, w.m, ref["win"][None],
                         [0], w.n_win, rows.reshape(1, -1), ops["sink"], 1.0 / math.sqrt(w.c))
    o = oracle.norm_rope(o[0], -rows, R, normalise=False)
    assert_close_out(to_np(p.out[0][sel]), o, w.dtype, "output turned back")
