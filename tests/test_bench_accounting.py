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


def test_traffic_comes_from_the_profile_of_the_same_kernel_source(tmp_path):
    """roofline.traffic is the ncu figure of the profile only while the kernel source it
    was captured on is unchanged (comments aside); otherwise it is reported as stale."""
    src = tmp_path / "k.cuh"
    src.write_text("// a comment\n__global__ void k() { int a = 1; }\n")
    h = bench.source_hash([str(src)])
    md = tmp_path / "prof.md"
    md.write_text(f"kernel source hash: `{h}`\n\n| traffic (read + write) | 174.1 MB per launch |\n")
    t, prov = bench.profile_traffic(str(md), [str(src)])
    assert t == 174.1e6 and prov["captured_on_hash"] == h
    src.write_text("// another comment\n\n__global__ void k() { int a = 1; }  // trailing\n")
    assert bench.source_hash([str(src)]) == h          # comments and blank lines do not count
    src.write_text("__global__ void k() { int a = 2; }\n")
    t, prov = bench.profile_traffic(str(md), [str(src)])
    assert t is None and prov["status"].startswith("stale")
    t, prov = bench.profile_traffic(str(tmp_path / "missing.md"), [str(src)])
    assert t is None


def test_committed_attention_profile_parses():
    t, prov = bench.profile_traffic(bench.ATTN_PROFILE, bench.ATTN_SOURCES)
    assert prov["captured_on_hash"] is not None
    assert t is None or 1e8 < t < 5e8
