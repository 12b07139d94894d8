"""Grouped output projection (DeepSeek-V4 restatement, "Compressed Sparse
Attention" Module B step 4): float64 oracle.

TEST INFRASTRUCTURE ONLY (tests and the benchmark's CPU-baseline leg).

The n_h head outputs of a token are cut into g groups of n_h / g heads; group
j is projected to d_g values with its own weight, the g results are
concatenated and projected to d:
    u_j = o[:, group j] W_g[j]^T,   u = [u_0 .. u_{g-1}],   out = u W_o^T.
Weights are stored [output features, input features]. The intermediate u is
stored in bf16 (as the GPU stores it) before the second product; numpy's
float64 matmul is the only library step.
"""
from __future__ import annotations

import numpy as np
import torch

from . import f64


def grouped_out_proj(o, Wg, Wo, g: int, store_u: bool = True):
    """o [n, h, c] (or [n, h*c]); Wg [g*dg, h*c/g]; Wo [d, g*dg]. Returns
    (u, out) in float64 (u rounded to bf16 when store_u)."""
    O = f64(o)
    n = O.shape[0]
    O = O.reshape(n, -1)
    Kg = O.shape[1] // g
    G = f64(Wg)
    dg = G.shape[0] // g
    u = np.empty((n, g * dg))
    for j in range(g):
        u[:, j * dg:(j + 1) * dg] = O[:, j * Kg:(j + 1) * Kg] @ G[j * dg:(j + 1) * dg].T
    if store_u:
        u = torch.from_numpy(u).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    out = u @ f64(Wo).T
    return u, out
