"""Pins of the oracle's RMSNorm + partial RoPE (Module D: Q/KV normalisation,
partial RoPE on the last 64 dims, output rotated back by the query position).

* The rotation's sign and frequencies on hand-computed cases: a pair at
  frequency index 0 rotates by the position itself, counter-clockwise; pair p
  of R rotated dims turns at base^(-2p/R).
* Rotating by p and then by -p gives the input back; the first c - R dims
  never change; the rotation keeps the norm.
* Rotated dot products depend only on the difference of the two positions
  (what makes the output's position relative).
* RMSNorm gives a mean square of 1 (gain 1, tiny eps) and ignores a positive
  scale of its input; a gain vector multiplies channel by channel.
* Whole chain: shifting every position (queries, entries, window rows) by the
  same amount leaves the rotated-back attention output unchanged.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import pipeline
from long_context_sparse_07_b200 import workloads as W


def test_rotation_sign_and_frequencies_by_hand():
    x = np.array([[1.0, 0.0]])
    got = oracle.norm_rope(x, [3], 2, normalise=False)
    np.testing.assert_allclose(got, [[math.cos(3.0), math.sin(3.0)]], atol=1e-15)
    # four rotated dims: pair 1 turns at 10000^(-1/2) = 0.01 rad per position
    x = np.array([[0.0, 0.0, 1.0, 0.0]])
    got = oracle.norm_rope(x, [100], 4, normalise=False)
    np.testing.assert_allclose(got, [[0.0, 0.0, math.cos(1.0), math.sin(1.0)]], atol=1e-15)
    # only the last R dims turn
    x = np.arange(1.0, 9.0)[None]
    got = oracle.norm_rope(x, [7], 4, normalise=False, base=100.0)
    np.testing.assert_array_equal(got[0, :4], x[0, :4])
    np.testing.assert_allclose(np.linalg.norm(got), np.linalg.norm(x), rtol=1e-14)


def test_inverse_and_relative_positions():
    g = np.random.default_rng(3)
    x = g.standard_normal((5, 3, 64))
    pos = np.array([0, 9, 1000, 65536, 1048575])
    back = oracle.norm_rope(oracle.norm_rope(x, pos, 64, normalise=False), -pos, 64,
                            normalise=False)
    np.testing.assert_allclose(back, x, atol=1e-11)
    q, k = g.standard_normal((1, 64)), g.standard_normal((1, 64))
    def dot(pq, pk):
        return float((oracle.norm_rope(q, [pq], 64, normalise=False) *
                      oracle.norm_rope(k, [pk], 64, normalise=False)).sum())
    np.testing.assert_allclose(dot(130, 7), dot(1123, 1000), rtol=1e-10)
    np.testing.assert_allclose(dot(7, 130), dot(10, 133), rtol=1e-10)
    assert abs(dot(130, 7) - dot(131, 7)) > 1e-6


def test_rmsnorm_unit_mean_square_scale_invariance_and_gain():
    g = np.random.default_rng(4)
    x = g.standard_normal((4, 2, 32)) * 7.0
    y = oracle.norm_rope(x, np.zeros(4, dtype=np.int64), 0, eps=1e-30)
    np.testing.assert_allclose((y ** 2).mean(-1), 1.0, rtol=1e-12)
    y2 = oracle.norm_rope(3.5 * x, np.zeros(4, dtype=np.int64), 0, eps=1e-30)
    np.testing.assert_allclose(y2, y, rtol=1e-12)
    gam = np.linspace(0.5, 2.0, 32)
    y3 = oracle.norm_rope(x, np.zeros(4, dtype=np.int64), 0, gamma=gam, eps=1e-30)
    np.testing.assert_allclose(y3, y * gam, rtol=1e-12)


def test_chain_is_invariant_to_a_common_position_shift():
    w = W.scaled(W.WORKLOADS["csa_fp32_n256"], n=96, c=64, k=4, n_win=8)
    ops = W.csa_operands(w)
    a = pipeline.csa_prefill_rope(ops, w, rope_dims=64, shift=0)
    b = pipeline.csa_prefill_rope(ops, w, rope_dims=64, shift=12345)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    # equal up to the float32 storage of the rotated q, entries and window rows
    # (the rotated values differ, so their roundings do): a few float32 ulps
    np.testing.assert_allclose(a["out"], b["out"], atol=2e-6)
    # and the rotation changes the result at all
    c = pipeline.csa_prefill(ops, w)
    assert np.abs(a["out"] - c["out"]).max() > 1e-3
