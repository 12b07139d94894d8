"""GPU parity of the grouped output projection (Module B step 4) through the
C ABI: u against the oracle's grouped products of the same bf16 operands,
out against the oracle's final product of the GPU's own u."""
import numpy as np
import pytest
import torch

from oracle import proj
from long_context_sparse_07_b200 import abi, workloads as W
from helpers import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(seed, n, h, c, g, dg, d):
    gen = np.random.default_rng(seed)
    o = W.to_storage(gen.standard_normal((n, h * c)).astype(np.float32), "bf16").view(n, h, c)
    Wg = W.to_storage((gen.standard_normal((g * dg, h * c // g)) * 0.02).astype(np.float32),
                      "bf16")
    Wo = W.to_storage((gen.standard_normal((d, g * dg)) * 0.02).astype(np.float32), "bf16")
    return o, Wg, Wo


def _check(got, ref, what):
    # bf16 results of float32 sums: errors within a bf16 rounding of the
    # result plus the accumulation, relative to the output's own spread
    scale = max(1.0, float(np.sqrt((ref ** 2).mean())))
    err = np.abs(got - ref) / scale
    assert np.isfinite(got).all(), what
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, "%s: max %.3g mean %.3g" % (
        what, err.max(), err.mean())


@pytest.mark.parametrize("n,h,c,g,dg,d", [
    (1000, 64, 512, 8, 1024, 4096),     # the Flash configuration, a ragged last tile
    (300, 32, 512, 4, 512, 2048),
    (129, 16, 64, 2, 256, 256),
])
def test_grouped_out_proj_matches_oracle(n, h, c, g, dg, d):
    o, Wg, Wo = _case(41 + n, n, h, c, g, dg, d)
    u = torch.full((n, g * dg), float("nan"), device=DEV, dtype=torch.bfloat16)
    out = torch.full((n, d), float("nan"), device=DEV, dtype=torch.bfloat16)
    abi.csa_grouped_out_proj(o.to(DEV), Wg.to(DEV), Wo.to(DEV), g, u, out)
    abi.csa_get_error()
    uref, _ = proj.grouped_out_proj(o, Wg, Wo, g, store_u=False)
    _check(to_np(u), uref, "u")
    # the final product on the GPU's own u
    _, oref = proj.grouped_out_proj(o, Wg, Wo, g)
    uo = to_np(u)
    _check(to_np(out), uo @ to_np(Wo).T, "out")
    _check(to_np(out), oref, "out vs the oracle chain")
