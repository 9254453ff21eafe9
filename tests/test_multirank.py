"""The multi-GPU host logic of bench.py on 2 CPU ranks (gloo): distinct per-rank inputs,
max-over-ranks timing and the whole-job throughput. No GPU; nothing here runs a kernel."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        wl = WORKLOADS["tiny"]
        x = draw_step_inputs(wl, seed=bench.rank_seed(wl.seed, rank), n_evicted=wl.Ne_step)
        t_local = 0.001 * (rank + 1)
        t = bench.max_over_ranks(t_local, dist)
        dist.barrier()
        q.put((rank, float(x["Q"].float().sum()), t, bench.job_throughput(world, wl.B, wl.Nq, t)))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_inputs():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    (r0, s0, t0, v0), (r1, s1, t1, v1) = res
    assert s0 != s1, "ranks must stream different synthetic inputs"
    assert t0 == t1 == pytest.approx(0.002), "every rank reports the slowest rank's time"
    assert v0 == v1 == pytest.approx(world * 64 / 0.002)

