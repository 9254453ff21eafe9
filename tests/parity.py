"""Shared helpers of the parity tests: conversions, tolerances and comparisons."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the hybrid attention step (GPU bf16/fp32 path vs the fp64 oracle).
TIE_TOL = 1e-4          # pooled scores closer than this may legally swap at the top-r boundary
O_MAX_ABS = 2e-2        # output, bf16 inputs
O_REL_L2 = 5e-3
STATE_REL_L2 = 1e-5     # fp32 state S and z
SCORE_ABS = 1e-4        # fp32 pooled score vs fp64


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want.ravel())
    return float(np.linalg.norm((got - want).ravel()) / (den if den > 0 else 1.0))


def assert_output_close(got, want, what="O"):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    mx = float(np.abs(got - want).max()) if got.size else 0.0
    rl = rel_l2(got, want)
    assert mx <= O_MAX_ABS and rl <= O_REL_L2, f"{what}: max-abs {mx:.3e} rel-L2 {rl:.3e}"
    return mx, rl


def assert_state_close(S_got, z_got, S_want, z_want):
    rs, rz = rel_l2(S_got, S_want), rel_l2(z_got, z_want)
    assert rs <= STATE_REL_L2 and rz <= STATE_REL_L2, f"state rel-L2: S {rs:.3e} z {rz:.3e}"
    return rs, rz


def assert_masks_match(idx_gpu, idx_oracle, scores, r):
    """Kept-block lists equal, except swaps between blocks whose pooled scores (oracle,
    fp64) are within TIE_TOL of the r-th best score. GPU lists must be ascending,
    distinct and in range."""
    idx_gpu = np.asarray(idx_gpu)
    idx_oracle = np.asarray(idx_oracle)
    assert idx_gpu.shape == idx_oracle.shape
    nKB = scores.shape[-1]
    rows = idx_gpu.reshape(-1, r)
    orows = idx_oracle.reshape(-1, r)
    srows = scores.reshape(-1, nKB)
    n_swaps = 0
    for g, o, s in zip(rows, orows, srows):
        assert np.all(np.diff(g) > 0) and g.min() >= 0 and g.max() < nKB, f"bad list {g}"
        if np.array_equal(g, o):
            continue
        order = np.lexsort((np.arange(nKB), -s))
        thr = s[order[r - 1]]
        diff = np.setxor1d(g, o)
        assert np.all(np.abs(s[diff] - thr) < TIE_TOL), (
            f"mask mismatch beyond the tie tolerance: gpu {g} oracle {o} scores {s[diff]} thr {thr}")
        n_swaps += 1
    return n_swaps
