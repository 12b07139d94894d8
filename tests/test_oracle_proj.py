"""Pins of the grouped output projection oracle (Module B step 4).

* Plain loops on a tiny case give the same u and out.
* One group is an ordinary two-layer projection o W_g^T W_o^T.
* The grouping is block-diagonal: zeroing the heads of group j zeroes u's
  slice j and nothing else.
"""
import numpy as np
import torch

from oracle import proj


def test_loops_on_a_tiny_case():
    g = np.random.default_rng(5)
    n, h, c, G, dg, d = 3, 4, 2, 2, 3, 5
    o = g.standard_normal((n, h, c))
    Wg = g.standard_normal((G * dg, h * c // G))
    Wo = g.standard_normal((d, G * dg))
    u, out = proj.grouped_out_proj(o, Wg, Wo, G, store_u=False)
    Kg = h * c // G
    for t in range(n):
        flat = o[t].reshape(-1)
        for j in range(G):
            for e in range(dg):
                ref = sum(flat[j * Kg + x] * Wg[j * dg + e, x] for x in range(Kg))
                assert abs(u[t, j * dg + e] - ref) < 1e-12
        for f in range(d):
            ref = sum(u[t, y] * Wo[f, y] for y in range(G * dg))
            assert abs(out[t, f] - ref) < 1e-12


def test_one_group_is_a_two_layer_projection():
    g = np.random.default_rng(6)
    o = g.standard_normal((7, 4, 8))
    Wg = g.standard_normal((16, 32))
    Wo = g.standard_normal((5, 16))
    u, out = proj.grouped_out_proj(o, Wg, Wo, 1, store_u=False)
    np.testing.assert_allclose(out, o.reshape(7, 32) @ Wg.T @ Wo.T, rtol=1e-12)


def test_groups_are_block_diagonal():
    g = np.random.default_rng(7)
    o = g.standard_normal((5, 8, 4))
    Wg = g.standard_normal((4 * 3, 8))
    Wo = g.standard_normal((6, 12))
    o2 = o.copy()
    o2[:, 2:4] = 0.0                              # the heads of group 1
    u, _ = proj.grouped_out_proj(o, Wg, Wo, 4, store_u=False)
    u2, _ = proj.grouped_out_proj(o2, Wg, Wo, 4, store_u=False)
    np.testing.assert_array_equal(u2[:, 3:6], 0.0)
    np.testing.assert_array_equal(u2[:, :3], u[:, :3])
    np.testing.assert_array_equal(u2[:, 6:], u[:, 6:])


def test_stored_intermediate_is_bf16():
    g = np.random.default_rng(8)
    o = g.standard_normal((2, 2, 64))
    Wg = g.standard_normal((256, 128))
    Wo = g.standard_normal((256, 256))
    u, _ = proj.grouped_out_proj(o, Wg, Wo, 1)
    assert np.array_equal(u, torch.from_numpy(u).to(torch.bfloat16).double().numpy())
