"""The no-allocation variant of the sparse attention call.

Some callers cannot allocate device memory on their hot path (a host
framework that owns all device memory through pre-reserved pools, or a decode
loop that cannot afford an allocation's device-wide synchronisation).
csa_sparse_mqa_noalloc serves them from a fixed device array inside the
library instead of a caller workspace. These tests call it through the C ABI
and compare it with csa_sparse_mqa given a workspace, on two calls in a row
with different inputs (so a stale scratch from the first call cannot leak
into the second), and check that a shape needing more scratch than the array
holds is refused. This file is collected last on purpose.
"""
import math

import numpy as np
import pytest
import torch

from long_context_sparse_07_b200 import abi, workloads as W
from long_context_sparse_07_b200.abi import Entries
from helpers import assert_close_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(seed, B=4, E=5000, k=1024, n_win=128, h=64, c=512):
    """A decode-shaped case (few queries, many keys): the call splits each
    query's keys and needs scratch."""
    L = 4 * E
    body = W.e4m3_codes(seed, "kv_nope", B * E, c - 64)
    scl = W.e4m3_scales(seed, "kv_scale", B * E, (c - 64) // 64, 1.0)
    rope = W.to_storage(W.normal(seed, "kv_rope", B * E, 64, 1.0), "bf16")
    kv = Entries(body.to(DEV), c, scale=scl.to(DEV), rope=rope.to(DEV), rope_dims=64,
                 scale_group=64)
    q = W.to_storage(W.normal(seed, "q", B, h * c, 1.0), "bf16").view(B, 1, h, c).to(DEV)
    kwin = W.to_storage(W.normal(seed, "kwin", B * n_win, c, 1.0), "bf16").view(
        B, n_win, c).to(DEV)
    idx = W.stratified_idx(seed, B, k, np.full(B, E)).to(DEV)
    sink = W.to_storage(W.normal(seed, "sink", 1, h, 1.0), "f32").view(h).to(DEV)
    q_pos = torch.full((B, 1), L - 1, dtype=torch.int64, device=DEV)
    win_pos0 = torch.full((B,), L - n_win, dtype=torch.int64, device=DEV)
    return dict(q=q, kv=kv, E=E, m=4, idx=idx, k=k, kwin=kwin, win_pos0=win_pos0, n_win=n_win,
                q_pos=q_pos, sink=sink, scale=1.0 / math.sqrt(c))


def _with_workspace(cs):
    B, n_q, h, c = cs["q"].shape
    n = abi.csa_mqa_workspace_size(B, n_q, h, c, cs["k"] + cs["n_win"])
    assert 0 < n <= abi.csa_noalloc_scratch_bytes()
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    out = torch.empty_like(cs["q"])
    lse = torch.empty(B, n_q, h, device=DEV)
    abi.csa_sparse_mqa(cs["q"], cs["kv"], cs["E"], cs["m"], cs["idx"], cs["k"], cs["kwin"],
                       cs["win_pos0"], cs["n_win"], cs["q_pos"], cs["sink"], cs["scale"], out, lse,
                       workspace=ws)
    return out, lse


def _no_alloc(cs):
    out = torch.empty_like(cs["q"])
    lse = torch.empty(cs["q"].shape[:3], device=DEV)
    abi.csa_sparse_mqa_noalloc(cs["q"], cs["kv"], cs["E"], cs["m"], cs["idx"], cs["k"],
                               cs["kwin"], cs["win_pos0"], cs["n_win"], cs["q_pos"], cs["sink"],
                               cs["scale"], out, lse)
    return out, lse


def test_no_alloc_matches_workspace_call_twice_in_a_row():
    abi.csa_get_error()
    first, second = _case(61), _case(62)
    ref1, lref1 = _with_workspace(first)
    ref2, lref2 = _with_workspace(second)
    got1, lgot1 = _no_alloc(first)
    got2, lgot2 = _no_alloc(second)
    abi.csa_get_error()
    for got, ref, lg, lr in ((got1, ref1, lgot1, lref1), (got2, ref2, lgot2, lref2)):
        assert_close_out(to_np(got), to_np(ref), "bf16", "no-alloc vs workspace")
        np.testing.assert_allclose(lg.cpu().numpy(), lr.cpu().numpy(), rtol=0, atol=2.0 ** -8)
    # the two inputs really differ, so the second call did not reuse the first
    assert not torch.equal(got1, got2)


def test_no_alloc_serves_the_8_query_decode_step():
    """The decode step of the 1M-token workload (8 queries, 64 heads, 1024
    selected entries, 128 window rows) fits the fixed scratch."""
    abi.csa_get_error()
    cs = _case(64, B=8, E=8192, k=1024, n_win=128)
    ref, lref = _with_workspace(cs)
    got, lgot = _no_alloc(cs)
    abi.csa_get_error()
    assert_close_out(to_np(got), to_np(ref), "bf16", "no-alloc vs workspace (B=8)")
    np.testing.assert_allclose(lgot.cpu().numpy(), lref.cpu().numpy(), rtol=0, atol=2.0 ** -8)


def test_no_alloc_checks_arguments_before_sizing_its_scratch():
    cs = _case(65, B=2, E=1024)
    bad = Entries(cs["kv"].body, 4096, scale=cs["kv"].scale, rope=cs["kv"].rope, rope_dims=64,
                  scale_group=64)
    out = torch.empty_like(cs["q"])
    with pytest.raises(abi.CsaError) as ei:
        abi.csa_sparse_mqa_noalloc(cs["q"], bad, cs["E"], cs["m"], cs["idx"], cs["k"],
                                   cs["kwin"], cs["win_pos0"], cs["n_win"], cs["q_pos"],
                                   cs["sink"], cs["scale"], out)
    assert ei.value.status in (-1, -2) and "scratch" not in str(ei.value)


def test_no_alloc_refuses_shapes_beyond_its_scratch():
    cs = _case(63, B=16, E=20000, k=4096)
    B, n_q, h, c = cs["q"].shape
    assert abi.csa_mqa_workspace_size(B, n_q, h, c, cs["k"] + cs["n_win"]) > \
        abi.csa_noalloc_scratch_bytes()
    with pytest.raises(abi.CsaError) as ei:
        _no_alloc(cs)
    assert ei.value.status == -2 and "scratch" in str(ei.value)
