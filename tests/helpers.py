"""Shared helpers of the parity tests (tolerances, row sampling, comparisons)."""
import numpy as np
import torch

# Tolerances on outputs (compressed entries, attention outputs):
#   float32 path: max-abs 1e-4; bfloat16 path: max-abs 2e-2 and mean-abs 2e-3.
F32_MAX_ABS = 1e-4
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
# Index scores: |gpu - oracle| <= SCORE_REL * S_t, where
# S_t = sum_h |w_th| * ||q_th||_1 * max_s,x |k_sx| bounds every |I[t][s]|; only
# the float32 accumulation order differs between the two sides.
SCORE_REL = 1e-5


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close_out(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(gpu - ref)
    assert np.isfinite(gpu).all(), what + ": non-finite output"
    if dtype == "f32":
        assert err.max() <= F32_MAX_ABS, "%s: max-abs %.3g > %.1g" % (what, err.max(), F32_MAX_ABS)
    else:
        assert err.max() <= BF16_MAX_ABS, "%s: max-abs %.3g" % (what, err.max())
        assert err.mean() <= BF16_MEAN_ABS, "%s: mean-abs %.3g" % (what, err.mean())


def sample_rows(n: int, m: int, count: int, seed: int = 0) -> np.ndarray:
    """Query positions to check on large cases: the first block (t < m),
    block edges, the last token, and uniform picks."""
    g = np.random.default_rng(seed)
    fixed = list(range(min(n, m + 1)))
    for i in (1, 2, 3, n // (2 * m), n // m - 1):
        for t in (m * i - 1, m * i):
            if 0 <= t < n:
                fixed.append(t)
    fixed.append(n - 1)
    extra = g.integers(0, n, size=max(0, count - len(fixed)))
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), extra]))


def score_scale(qI: np.ndarray, wI: np.ndarray, kmax: float) -> np.ndarray:
    """S_t for qI [..., hI, cI] (values), wI [..., hI]."""
    return (np.abs(wI) * np.abs(qI).sum(-1)).sum(-1) * kmax
