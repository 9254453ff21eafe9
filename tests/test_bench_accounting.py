"""The bench's FLOP accounting for the attention kernel (host arithmetic only)."""
import numpy as np

import bench
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS


def test_attention_flop_accounting():
    """Algorithmic FLOPs count valid tokens only; the issued ones count whole 128-row tiles
    and blocks plus the three readout MMAs, so they are never fewer."""
    wl = WORKLOADS["832x480"]
    idx = np.tile(np.arange(wl.r, dtype=np.int32), (wl.B, wl.H, wl.nQB, 1))
    F = bench.attn_flops(idx, wl)
    # blocks 0..r-1 are full (128 tokens); the last query block holds 4680 - 36*128 = 72 rows
    sparse = 4.0 * wl.d * wl.r * wl.block * wl.Nq * wl.B * wl.H
    readout = wl.B * wl.H * wl.Nq * (2.0 * wl.d ** 2 + 3.0 * wl.d)
    assert F == sparse + readout
    issued = bench.attn_issued_flops(idx, wl)
    assert issued == 4.0 * 128 * 128 * 128 * wl.r * 12 * 37 + 6.0 * 128 * 128 * 128 * 12 * 37
    assert issued > F


def test_oracle_sample_times_every_call():
    """The CPU baseline's oracle sample reports the selection, attention and absorption
    separately (tiny workload, on the host)."""
    import torch

    from hybrid_sparse_linear_hf_b200.inputs import draw_step_inputs

    wl = WORKLOADS["tiny"]
    x = draw_step_inputs(wl, n_evicted=wl.Ne_step)
    S0 = torch.zeros(wl.B, wl.H, wl.d, wl.d)
    z0 = torch.zeros(wl.B, wl.H, wl.d)
    parts = bench.oracle_sample(wl, x, S0, z0, [0], x["K_ev"], x["V_ev"])
    assert set(parts) == {"select", "attention", "absorb"} and all(v > 0 for v in parts.values())
    t_s, t_a, t_t = bench.oracle_step_sample(wl, x, S0, z0, 0, 2, 0)
    assert t_s > 0 and t_a > 0 and t_t > 0
