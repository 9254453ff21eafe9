"""Benchmark of the hybrid attention chunk step on B200.

One step = one pass of the whole hot path over one chunk of the 832x480-shaped
workload (B=1, H=12, d=128, 4680 queries, 32760-key window, block 128, top-64 of 256
key blocks, state built from 60 evicted frames):
    hf_select_blocks           block mean pooling, scores, top-r                (2 kernels)
    hf_hybrid_attn_fwd_absorb  sparse attention + linear readout, summed, then the
                               chunk step's 3 evicted frames -> state           (3 kernels)
Metric: query tokens/s per chunk step (whole job, all GPUs), with the roofline fraction
of the dominant kernel (hf_hybrid_attn_fwd, tensor-bound) against the measured bf16
peak (timed alone in its own leg, as are the selection and the absorption). Legs
reported beside the step: the 60-frame state build, the two-stage (frame,
then block) selection, the selection from the pooled-key cache (with the push of the
chunk's keys), the attention at keep 1 / 0.5 / 0.25 / 0.125, a video's first 12 chunks
under the chunk-aware growth keep schedule, the selection and attention with the capped
relative temporal RoPE, the 1280x720-shaped step (attention,
selection, 120-frame state build), and a streaming end-to-end step: the chunk's Q, K, V
copied in from pinned host memory, the device-resident window shifted by the chunk, the
evicted frames absorbed, O copied back.
Inputs are resident in HBM. Between timed calls L2 is flushed: a 256 MiB buffer is
written and then read, so that no dirty line of the flush is written back inside a timed
kernel. Launches are enqueued without host synchronisation, so the host runs ahead and
the CUDA events bracket device work only. Multi-GPU (torchrun): every rank runs its own
chunk stream (weak scaling, no collective on the data path); time = max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

``--impl reference`` times the fp64 CPU oracle instead (per step a bounded sample of
the same step, scaled to the whole step) on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import faulthandler
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs, frame_structured  # noqa: E402

METRIC = "hybrid attn query tokens/s per chunk step; % of bf16 tensor / HBM roofline"
UNIT = "query tokens/s"
WORKLOAD = "832x480"
LARGE_WORKLOAD = "1280x720"
L2_FLUSH_BYTES = 256 << 20
# The attention kernel's DRAM traffic per launch comes from its ncu summary in profiles/,
# which records the hash of the kernel source it was taken on; a changed source makes
# the recorded figure stale and the bench then reports no traffic.
ATTN_PROFILE = os.path.join(ROOT, "profiles", "hybrid_attn_kernel_832x480.md")
ATTN_SOURCES = [os.path.join(ROOT, "hybrid_sparse_linear_hf_b200", "csrc", f) for f in ("hf_attn.cuh", "hf_ptx.cuh")]
# frames kept per query block by the two-stage selection leg (8 of the window's 21 frames:
# at least 12 blocks each, so the 64 kept blocks always come from the kept frames)
TWO_STAGE_FRAMES = 8
# keep ratios of the sparsity sweep leg (1 = dense window attention)
SWEEP_KEEPS = (1.0, 0.5, 0.25, 0.125)
# chunk-aware growth leg: a video's first chunks (the window filling up, then full) under
# the keep schedule with these sparsity ratios, against the same mean sparsity per chunk
SCHEDULE_CHUNKS = 12
SCHEDULE_S_BASE = 0.85
SCHEDULE_S_TARGET = 0.75
# pooled-key cache leg: tokens per granule sum (divides the 4680-key chunk and the block)
KPOOL_GRANULE = 8
# temporal RoPE leg: 44 of the 128 dimensions turned (a 3-D video RoPE's temporal share,
# 128 - 2 x 42), the index capped at 8 frames (a 9-frame window)
ROPE_DT = 44
ROPE_CAP = 8


# ----------------------------------------------------------------------------- helpers
_T0 = time.time()
_VERBOSE = False


def log(msg: str) -> None:
    """Progress line on stderr (``--verbose``)."""
    if _VERBOSE:
        print(f"[bench {time.time() - _T0:8.2f}s] {msg}", file=sys.stderr, flush=True)


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def attn_flops(idx: np.ndarray, wl) -> float:
    """Algorithmic FLOPs of one hf_hybrid_attn_fwd launch: 4*d*L_I*L_J per kept (I, J)
    pair (QK^T and PV), plus 2d^2 + 3d per query for the linear readout."""
    L_I = np.array([min(wl.block, wl.Nq - I * wl.block) for I in range(wl.nQB)], dtype=np.float64)
    L_J = np.array([min(wl.block, wl.Nk - J * wl.block) for J in range(wl.nKB)], dtype=np.float64)
    kept_len = L_J[idx].sum(axis=-1)  # [B,H,nQB]
    sparse = 4.0 * wl.d * float((kept_len * L_I[None, None, :]).sum())
    readout = wl.B * wl.H * wl.Nq * (2.0 * wl.d * wl.d + 3.0 * wl.d)
    return sparse + readout


def attn_issued_flops(idx: np.ndarray, wl) -> float:
    """FLOPs the attention kernel issues on the tensor cores: per kept block 128-row QK^T and
    PV MMAs over the whole block (padding included), plus the three split-precision readout
    MMAs (phi_hi S_hi, phi_hi S_lo, phi_lo S_hi) per 128-row query tile."""
    kept = int(((idx >= 0) & (idx < wl.nKB)).sum())
    tiles = wl.B * wl.H * wl.nQB
    return 4.0 * 128 * wl.block * wl.d * kept + 3 * 2.0 * 128 * wl.d * wl.d * tiles


def attn_bytes(wl) -> float:
    """Algorithmic bytes of one launch: Q and O once, the whole K/V window once, S and z."""
    return 2.0 * wl.B * wl.H * (2 * wl.Nq * wl.d + 2 * wl.Nk * wl.d) + 4.0 * wl.B * wl.H * (wl.d * wl.d + wl.d)


def select_bytes(wl) -> float:
    return 2.0 * wl.B * wl.H * (wl.Nq + wl.Nk) * wl.d


def absorb_bytes(wl, n_tokens) -> float:
    """K_ev and V_ev read once plus a read and a write of S and z."""
    return 2.0 * 2 * wl.B * wl.H * n_tokens * wl.d + 2 * 4.0 * wl.B * wl.H * (wl.d * wl.d + wl.d)


def source_hash(paths) -> str:
    """Hash of the code of the given C++/CUDA sources with comments and blank lines
    removed, so that a change of comments only keeps a recorded measurement valid."""
    h = hashlib.sha256()
    for p in paths:
        text = open(p).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln.strip()).encode())
    return h.hexdigest()[:16]


def profile_traffic(md_path: str, sources) -> tuple:
    """(DRAM bytes per launch or None, provenance) from an ncu summary that holds a line
    ``| traffic (read + write) | X MB per launch |`` and ``kernel source hash: H``."""
    cur = source_hash(sources)
    try:
        text = open(md_path).read()
    except OSError:
        return None, {"status": "no ncu summary", "kernel_source_hash": cur}
    m_t = re.search(r"\|\s*traffic \(read \+ write\)\s*\|\s*([0-9.]+) MB per launch", text)
    m_h = re.search(r"kernel source hash:\s*`?([0-9a-f]{16})", text)
    prov = {"file": os.path.relpath(md_path, ROOT), "kernel_source_hash": cur,
            "captured_on_hash": m_h.group(1) if m_h else None}
    if not (m_t and m_h):
        return None, dict(prov, status="summary lacks a traffic line or a source hash")
    if m_h.group(1) != cur:
        return None, dict(prov, status="stale: the kernel source changed since the ncu capture")
    return float(m_t.group(1)) * 1e6, dict(prov, status="ncu dram__bytes_read.sum + dram__bytes_write.sum, "
                                                       "one launch, same kernel source")


def max_over_ranks(t_local: float, dist=None, device="cpu") -> float:
    """The slowest rank's time (every rank takes the same collective step)."""
    if dist is None:
        return t_local
    tt = torch.tensor([t_local], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_throughput(world: int, B: int, Nq: int, t_step: float) -> float:
    """Whole-job query tokens/s: every rank processes its own B x Nq chunk per step."""
    return world * B * Nq / t_step


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank streams its own synthetic chunk (independent inputs, same recipe)."""
    return base_seed + 1000 * rank


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.out = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self) -> dict:
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "sm_mhz_min": min(sm)}


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
        return int(n)
    except Exception:
        return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------- oracle leg
def oracle_sample(wl, x: dict, S0: torch.Tensor, z0: torch.Tensor, heads, ev_k, ev_v) -> dict:
    """Seconds the fp64 oracle takes for the whole step on the given heads, per call:
    {"select", "attention", "absorb"} (the absorption of the step's evicted tokens)."""
    import oracle

    f64 = lambda t: t.detach().cpu().to(torch.float64).numpy()  # noqa: E731
    parts = {"select": 0.0, "attention": 0.0, "absorb": 0.0}
    for h in heads:
        Q = f64(x["Q"][:, h:h + 1])
        K = f64(x["K"][:, h:h + 1])
        V = f64(x["V"][:, h:h + 1])
        S = f64(S0[:, h:h + 1])
        z = f64(z0[:, h:h + 1])
        Ke = f64(ev_k[:, h:h + 1])
        Ve = f64(ev_v[:, h:h + 1])
        t0 = time.perf_counter()
        idx, _ = oracle.select_blocks(Q, K, wl.block, wl.r)
        t1 = time.perf_counter()
        oracle.hybrid_attention(Q, K, V, idx, S, z, wl.block)
        t2 = time.perf_counter()
        oracle.absorb(S, z, Ke, Ve)
        t3 = time.perf_counter()
        parts["select"] += t1 - t0
        parts["attention"] += t2 - t1
        parts["absorb"] += t3 - t2
    return parts


REFERENCE_BUDGET_S = 150.0  # CPU seconds the whole reference run (warm-up + timed) aims at


def oracle_step_sample(wl, x: dict, S0: torch.Tensor, z0: torch.Tensor, h: int, n_tiles: int, first_tile: int):
    """One bounded sample of the step on head h: the whole selection and absorption of the
    head and the hybrid attention of n_tiles query blocks. Returns the seconds of the
    selection, of the absorption and of the n_tiles attention tiles."""
    import oracle

    f64 = lambda t: t.detach().cpu().to(torch.float64).numpy()  # noqa: E731
    Q, K, V = (f64(x[k][:, h:h + 1]) for k in ("Q", "K", "V"))
    S, z = f64(S0[:, h:h + 1]), f64(z0[:, h:h + 1])
    Ke, Ve = f64(x["K_ev"][:, h:h + 1]), f64(x["V_ev"][:, h:h + 1])
    t0 = time.perf_counter()
    idx, _ = oracle.select_blocks(Q, K, wl.block, wl.r)
    ta = time.perf_counter()
    oracle.absorb(S, z, Ke, Ve)
    t1 = time.perf_counter()
    for k in range(n_tiles):
        oracle.hybrid_attention_tile(Q, K, V, idx, S, z, wl.block, 0, 0, (first_tile + k) % wl.nQB)
    t2 = time.perf_counter()
    return ta - t0, t1 - ta, t2 - t1


def run_reference(args, wl) -> None:
    """Reference arm: the fp64 CPU oracle. Every step is a bounded sample of the step (one
    head's selection and absorption and as many of its query blocks' hybrid attention as
    the run's time budget allows), scaled to the whole step: per head, the selection and
    absorption as timed plus the attention time per query block times the query blocks;
    times the heads."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = draw_step_inputs(wl, n_evicted=wl.Ne_step)
    g = torch.Generator().manual_seed(wl.seed + 77)
    S0 = torch.randn(wl.B, wl.H, wl.d, wl.d, generator=g).abs() * 50.0
    z0 = torch.rand(wl.B, wl.H, wl.d, generator=g) * 1e5
    # size the per-step sample from one probe (one query block) against the budget
    t_sel, t_abs, t_tile = oracle_step_sample(wl, x, S0, z0, 0, 1, 0)
    t_fix = t_sel + t_abs
    per_step = REFERENCE_BUDGET_S / max(1, args.steps + args.warmup)
    n_tiles = int(max(1, min(wl.nQB, (per_step - t_fix) / max(t_tile, 1e-9))))
    for i in range(args.warmup):
        oracle_step_sample(wl, x, S0, z0, i % wl.H, n_tiles, i * n_tiles)
    times, parts, sampled = [], {"select": [], "attention": [], "absorb": []}, []
    for i in range(args.steps):
        t_s, t_a, t_t = oracle_step_sample(wl, x, S0, z0, i % wl.H, n_tiles, i * n_tiles)
        sampled.append(t_s + t_a + t_t)
        parts["select"].append(t_s * wl.H)
        parts["absorb"].append(t_a * wl.H)
        parts["attention"].append(t_t / n_tiles * wl.nQB * wl.H)
        times.append(parts["select"][-1] + parts["absorb"][-1] + parts["attention"][-1])
    t_step = statistics.mean(times)
    value = wl.B * wl.Nq / t_step
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"fp64 numpy oracle per step: 1 of {wl.H} heads (its selection and the absorb "
                                   f"of {wl.Ne_step} evicted tokens, and the hybrid attention of {n_tiles} of its "
                                   f"{wl.nQB} query blocks), scaled to all query blocks and heads",
                         "ms_per_call": {k: statistics.mean(v) * 1e3 for k, v in parts.items()},
                         "sample_ms_per_step": statistics.mean(sampled) * 1e3,
                         "projection": f"ms_per_step = the sample's selection and absorption x {wl.H} heads + its "
                                       f"attention x {wl.nQB}/{n_tiles} query blocks x {wl.H} heads; the timed "
                                       f"region ran {len(sampled)} samples of sample_ms_per_step each"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(wl) -> dict:
    return {"workload": f"{wl.name} hybrid attention chunk step", "B": wl.B, "H": wl.H, "d": wl.d,
            "Nq": wl.Nq, "Nk": wl.Nk, "block": wl.block, "keep": wl.keep, "r": wl.r,
            "state_frames": wl.state_frames, "evict_frames_per_step": wl.evict_frames,
            "l2": "flushed between timed calls (256 MiB written, then read back: no dirty line is left)",
            "parallelism": "independent streams per GPU"}


# ----------------------------------------------------------------------------- GPU leg
class DeviceTimer:
    """Times calls on one stream with CUDA events, an L2 flush before each call (a 256 MiB
    write, then a read of it, so the flush's dirty lines are written back before the
    timed call starts) and no host synchronisation between calls: the host enqueues
    ahead of the device, so each event pair brackets device work only."""

    def __init__(self, dev, stream):
        self.dev, self.stream = dev, stream
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush(self) -> None:
        self.buf.fill_(1)
        self.buf.view(torch.int64).sum()

    def run(self, fn, n: int, warm: int = 2) -> list:
        """Seconds of each of n calls of fn() (after `warm` untimed ones)."""
        pairs = []
        for k in range(warm + n):
            self.flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            fn()
            e1.record(self.stream)
            if k >= warm:
                pairs.append((e0, e1))
        torch.cuda.synchronize(self.dev)
        return [a.elapsed_time(b) * 1e-3 for a, b in pairs]


def check_status(hf, where: str) -> None:
    rc, word = hf.hf_query_status()
    if rc != hf.HF_OK:
        raise RuntimeError(f"device status after {where}: {hf.hf_status_string(rc)} ({word:#x})")


def large_workload_leg(hf, dev, timer: DeviceTimer, peaks: dict, rank: int) -> dict:
    """The 1280x720-shaped step (B=1, H=40, d=128, 10800 queries, 43200-key window, r=68,
    state from 120 evicted frames): the state build, the selection and the attention,
    each timed alone."""
    wl = WORKLOADS[LARGE_WORKLOAD]
    gen = torch.Generator(device=dev).manual_seed(wl.seed + 5000 + rank)
    S = torch.empty(wl.B, wl.H, wl.d, wl.d, dtype=torch.float32, device=dev)
    z = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device=dev)
    st = hf.hf_state_init(S, z)
    bK = frame_structured(gen, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, device=dev)
    bV = frame_structured(gen, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, device=dev)
    ws_b = torch.empty(hf.hf_workspace_size(hf.HF_WS_ABSORB, wl.B, wl.H, 0, wl.Ne_state, wl.d, 0, 0),
                       dtype=torch.uint8, device=dev)
    Sb, zb = torch.empty_like(S), torch.empty_like(z)
    stb = hf.hf_state_init(Sb, zb)
    t_build = timer.run(lambda: hf.hf_absorb_evicted(stb, bK, bV, ws=ws_b), n=3, warm=1)
    hf.hf_absorb_evicted(st, bK, bV, ws=ws_b)
    torch.cuda.synchronize(dev)
    del bK, bV, ws_b, Sb, zb, stb
    torch.cuda.empty_cache()
    x = draw_step_inputs(wl, seed=rank_seed(wl.seed, rank), n_evicted=1, device=dev)
    Q, K, V = x["Q"], x["K"], x["V"]
    ws_s = torch.empty(hf.hf_workspace_size(hf.HF_WS_SELECT, wl.B, wl.H, wl.Nq, wl.Nk, wl.d, wl.block, wl.r),
                       dtype=torch.uint8, device=dev)
    idx = torch.empty(wl.B, wl.H, wl.nQB, wl.r, dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    t_sel = timer.run(lambda: hf.hf_select_blocks(Q, K, wl.block, wl.r, idx_out=idx, ws=ws_s), n=5)
    t_att = timer.run(lambda: hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx, st, O=O), n=5)
    check_status(hf, "the 1280x720 leg")
    F = attn_flops(idx.cpu().numpy(), wl)
    ta, ts, tb = statistics.mean(t_att), statistics.mean(t_sel), statistics.mean(t_build)
    out = {
        "config": {"B": wl.B, "H": wl.H, "d": wl.d, "Nq": wl.Nq, "Nk": wl.Nk, "block": wl.block, "keep": wl.keep,
                   "r": wl.r, "state_frames": wl.state_frames},
        "hf_hybrid_attn_fwd": {"us": ta * 1e6, "flops_per_launch": F, "tflops": F / ta / 1e12,
                               "frac": F / ta / 1e12 / peaks["bf16_tflops"]},
        "hf_select_blocks": {"us": ts * 1e6, "bytes": select_bytes(wl),
                             "hbm_frac": select_bytes(wl) / ts / 1e9 / peaks["hbm_gbs"]},
        "hf_absorb_evicted_state_build": {"us": tb * 1e6, "tokens": wl.Ne_state,
                                          "bytes": absorb_bytes(wl, wl.Ne_state),
                                          "hbm_frac": absorb_bytes(wl, wl.Ne_state) / tb / 1e9 / peaks["hbm_gbs"]},
        "step_query_tokens_per_s": wl.B * wl.Nq / (ta + ts),
    }
    del x, Q, K, V, O, idx, ws_s, S, z, st
    torch.cuda.empty_cache()
    return out


def run_gpu(args, wl) -> None:
    import hybrid_sparse_linear_hf_b200 as hf

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=120))
        dist = dist_mod
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    timer = DeviceTimer(dev, stream)
    peaks = load_peaks()

    log(f"rank {rank}/{world} on {dev}")
    # ---- inputs, drawn on the device (same recipe, device generator), resident in HBM
    x = draw_step_inputs(wl, seed=rank_seed(wl.seed, rank), n_evicted=wl.Ne_step, device=dev)
    Q, K, V, K_ev, V_ev = (x[k] for k in ("Q", "K", "V", "K_ev", "V_ev"))
    S = torch.empty(wl.B, wl.H, wl.d, wl.d, dtype=torch.float32, device=dev)
    z = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device=dev)
    st = hf.hf_state_init(S, z)
    # the state is built from `state_frames` evicted frames (absorbed in slices)
    gen = torch.Generator(device=dev).manual_seed(wl.seed + 5000 + rank)
    build_K = frame_structured(gen, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, device=dev)
    build_V = frame_structured(gen, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, device=dev)
    ws_abs_build = torch.empty(hf.hf_workspace_size(hf.HF_WS_ABSORB, wl.B, wl.H, 0, wl.Ne_state, wl.d, 0, 0),
                               dtype=torch.uint8, device=dev)
    # time the full state build (the absorption's HBM roofline case) on a scratch state
    Sb = torch.empty_like(S)
    zb = torch.empty_like(z)
    stb = hf.hf_state_init(Sb, zb)
    torch.cuda.synchronize(dev)
    log("inputs drawn; timing the state build")
    build_times = timer.run(lambda: hf.hf_absorb_evicted(stb, build_K, build_V, ws=ws_abs_build), n=5, warm=2)
    hf.hf_absorb_evicted(st, build_K, build_V, ws=ws_abs_build)
    torch.cuda.synchronize(dev)
    del build_K, build_V, ws_abs_build, Sb, zb, stb
    torch.cuda.empty_cache()
    ws_sel = torch.empty(hf.hf_workspace_size(hf.HF_WS_SELECT, wl.B, wl.H, wl.Nq, wl.Nk, wl.d, wl.block, wl.r),
                         dtype=torch.uint8, device=dev)
    ws_abs = torch.empty(hf.hf_workspace_size(hf.HF_WS_ABSORB, wl.B, wl.H, 0, wl.Ne_step, wl.d, 0, 0),
                         dtype=torch.uint8, device=dev)
    idx = torch.empty(wl.B, wl.H, wl.nQB, wl.r, dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)

    def step(ev=None):
        # select, then the attention and the absorption of the step's evicted frames in one
        # call (the absorption's partial sums run beside the attention's last CTAs); events
        # only around the whole step, so that no event sits between dependent launches
        if ev:
            ev[0].record(stream)
        hf.hf_select_blocks(Q, K, wl.block, wl.r, idx_out=idx, ws=ws_sel)
        hf.hf_hybrid_attn_fwd_absorb(Q, K, V, wl.block, wl.r, idx, st, K_ev, V_ev, O=O, ws=ws_abs)
        if ev:
            ev[1].record(stream)

    log("warm-up")
    for i in range(max(args.warmup, 3)):
        timer.flush()
        step()
        if _VERBOSE:
            torch.cuda.synchronize(dev)
            log(f"warm-up step {i} done")
    torch.cuda.synchronize(dev)
    check_status(hf, "warm-up")
    idx_host = idx.cpu().numpy()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    log("timed steps")
    launches0 = hf.hf_launch_count()
    with ClockSampler(dev.index) as clk:
        for k in range(args.steps):
            timer.flush()
            step(events[k])
        torch.cuda.synchronize(dev)
    launches = hf.hf_launch_count() - launches0
    if dist:
        dist.barrier()
    check_status(hf, "timing")
    t_step_local = sum(e[0].elapsed_time(e[1]) for e in events) * 1e-3 / args.steps
    t_step = max_over_ranks(t_step_local, dist, dev)

    # ---- each call of the step timed alone (the attention's time gives the roofline)
    log("per-call legs")
    n_leg = max(3, min(args.steps, 50))
    t_sel = timer.run(lambda: hf.hf_select_blocks(Q, K, wl.block, wl.r, idx_out=idx, ws=ws_sel), n=n_leg, warm=3)
    attn_launches0 = hf.hf_launch_count()
    t_fwd = timer.run(lambda: hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx, st, O=O), n=n_leg, warm=3)
    attn_launches = hf.hf_launch_count() - attn_launches0
    t_abs = timer.run(lambda: hf.hf_absorb_evicted(st, K_ev, V_ev, ws=ws_abs), n=n_leg, warm=3)
    t_fused = timer.run(lambda: hf.hf_hybrid_attn_fwd_absorb(Q, K, V, wl.block, wl.r, idx, st, K_ev, V_ev, O=O,
                                                             ws=ws_abs), n=n_leg, warm=3)
    check_status(hf, "the per-call legs")
    # ---- capped relative temporal RoPE: the selection and the attention on turned Q, K
    log("rope leg")
    rope = hf.hf_rope(ROPE_DT, wl.tokens_per_frame, ROPE_CAP, wl.window_frames - wl.chunk_frames)
    idx_rope = torch.empty_like(idx)
    t_sel_rope = timer.run(lambda: hf.hf_select_blocks_rope(Q, K, wl.block, wl.r, rope, idx_out=idx_rope,
                                                            ws=ws_sel), n=n_leg, warm=3)
    t_fwd_rope = timer.run(lambda: hf.hf_hybrid_attn_fwd_rope(Q, K, V, wl.block, wl.r, idx_rope, st, rope, O=O),
                           n=n_leg, warm=3)
    check_status(hf, "the rope leg")
    F_rope = attn_flops(idx_rope.cpu().numpy(), wl)

    log(f"timed: {t_step_local * 1e3:.3f} ms/step; two-stage selection leg")
    # ---- two-stage (frame, then block) selection, timed alone beside the step
    ws_sel2 = torch.empty(hf.hf_workspace_size(hf.HF_WS_SELECT_TWO_STAGE, wl.B, wl.H, wl.Nq, wl.Nk, wl.d, wl.block,
                                               wl.r), dtype=torch.uint8, device=dev)
    idx2 = torch.empty_like(idx)
    t_sel2 = timer.run(lambda: hf.hf_select_blocks_two_stage(Q, K, wl.block, wl.r, wl.tokens_per_frame,
                                                             TWO_STAGE_FRAMES, idx_out=idx2, ws=ws_sel2),
                       n=n_leg, warm=3)
    check_status(hf, "the two-stage leg")
    # ---- pooled-key cache: per step the chunk's keys enter the cache and the oldest chunk
    # leaves (hf_kpool_push), then the selection pools its key blocks from the granule sums
    log("pooled-key cache leg")
    kp_sums = torch.empty(wl.B, wl.H, wl.Nk // KPOOL_GRANULE, wl.d, dtype=torch.float32, device=dev)
    kp = hf.hf_kpool_init(kp_sums, KPOOL_GRANULE)
    for c0 in range(0, wl.Nk, wl.Nq):
        hf.hf_kpool_push(kp, K[:, :, c0:c0 + wl.Nq].contiguous())
    K_in = K[:, :, wl.Nk - wl.Nq:].contiguous()  # stands in for the chunk's new keys
    idx_c = torch.empty_like(idx)
    t_push = timer.run(lambda: hf.hf_kpool_push(kp, K_in, n_evict=wl.Nq), n=n_leg, warm=3)
    t_selc = timer.run(lambda: hf.hf_select_blocks_cached(Q, kp, wl.block, wl.r, idx_out=idx_c, ws=ws_sel),
                       n=n_leg, warm=3)
    # the same step as one call: the push's sums computed in the Q pooling launch
    t_selcp = timer.run(lambda: hf.hf_select_blocks_cached_push(Q, kp, K_in, wl.block, wl.r, n_evict=wl.Nq,
                                                                idx_out=idx_c, ws=ws_sel), n=n_leg, warm=3)
    del kp_sums, K_in
    check_status(hf, "the pooled-key cache leg")
    # ---- sparsity sweep: the attention alone at other keep ratios (same inputs and state)
    log("sweep leg")
    sweep = {}
    for keep in SWEEP_KEEPS:
        wk = wl.with_keep(keep)
        idx_k = torch.empty(wl.B, wl.H, wl.nQB, wk.r, dtype=torch.int32, device=dev)
        hf.hf_select_blocks(Q, K, wl.block, wk.r, idx_out=idx_k, ws=ws_sel)
        t_k = statistics.mean(timer.run(lambda: hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wk.r, idx_k, st, O=O),
                                        n=10))
        F_k = attn_flops(idx_k.cpu().numpy(), wk)
        sweep[f"{keep:g}"] = {"r": wk.r, "us": t_k * 1e6, "tflops": F_k / t_k / 1e12}
    check_status(hf, "the sweep leg")
    # ---- chunk-aware growth: the attention of a video's first chunks under the keep
    # schedule (chunk i's window holds the newest min(i + 1, full) chunks of keys)
    log("keep schedule leg")
    per_window = wl.window_frames // wl.chunk_frames
    wls = [dataclasses.replace(wl, window_frames=min(i + 1, per_window) * wl.chunk_frames)
           for i in range(SCHEDULE_CHUNKS)]
    nKB_s = [w.nKB for w in wls]
    r_s, s_s, beta_s = hf.hf_keep_schedule(nKB_s, SCHEDULE_S_BASE, SCHEDULE_S_TARGET)
    r_u = [max(1, math.ceil((1.0 - SCHEDULE_S_TARGET) * n - 1e-9)) for n in nKB_s]
    kv_win = {}
    for w in wls:
        if w.Nk not in kv_win:
            kv_win[w.Nk] = (K[:, :, K.shape[2] - w.Nk:].contiguous(), V[:, :, V.shape[2] - w.Nk:].contiguous())

    def time_chunk(w, r_c):
        Kc, Vc = kv_win[w.Nk]
        idx_c = torch.empty(wl.B, wl.H, wl.nQB, r_c, dtype=torch.int32, device=dev)
        hf.hf_select_blocks(Q, Kc, wl.block, r_c, idx_out=idx_c, ws=ws_sel)
        return statistics.mean(timer.run(lambda: hf.hf_hybrid_attn_fwd(Q, Kc, Vc, wl.block, r_c, idx_c, st, O=O),
                                         n=3)) * 1e6

    us_s = [time_chunk(w, rc_) for w, rc_ in zip(wls, r_s)]
    us_u = [time_chunk(w, rc_) for w, rc_ in zip(wls, r_u)]
    del kv_win
    check_status(hf, "the keep schedule leg")
    schedule = {"s_base": SCHEDULE_S_BASE, "s_target": SCHEDULE_S_TARGET, "beta": beta_s, "nKB": nKB_s,
                "r": r_s, "attn_us": [round(u, 1) for u in us_s], "attn_us_total": sum(us_s),
                "uniform_r": r_u, "uniform_attn_us_total": sum(us_u)}

    log("end-to-end leg")
    # ---- streaming end to end through the public API: per step the chunk's Q, K, V come
    # from pinned host memory (on a copy stream, overlapping the previous step's compute),
    # the device-resident window drops its oldest chunk (absorbed into the state) and takes
    # the chunk's keys, then select + attention, and O goes back to pinned host memory.
    e2e = streaming_e2e_leg(hf, wl, dev, stream, x, st, ws_sel, ws_abs, args, dist)

    log("1280x720 leg")
    del ws_sel, ws_abs, ws_sel2, idx2, idx_c
    torch.cuda.empty_cache()
    large = large_workload_leg(hf, dev, timer, peaks, rank) if not args.no_large else None
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    F = attn_flops(idx_host, wl)
    fwd_mean = statistics.mean(t_fwd)
    achieved_tf = F / fwd_mean / 1e12
    sel_mean, abs_mean = statistics.mean(t_sel), statistics.mean(t_abs)
    build_mean = statistics.mean(build_times)
    value = job_throughput(world, wl.B, wl.Nq, t_step)
    traffic, traffic_src = profile_traffic(ATTN_PROFILE, ATTN_SOURCES)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(wl),
        "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved_tf / peaks["bf16_tflops"], "traffic": traffic, "traffic_source": traffic_src,
                     "kernel": "hybrid_attn_kernel<128,128>", "flops_per_launch": F,
                     "issued_flops_per_launch": attn_issued_flops(idx_host, wl),
                     "peak_source": f"{peaks['source']} dense bf16 (burst)"},
        "kernels": {
            "hf_hybrid_attn_fwd": {"us": fwd_mean * 1e6, "tflops": achieved_tf,
                                   "bytes": attn_bytes(wl), "gbs": attn_bytes(wl) / fwd_mean / 1e9},
            "hf_select_blocks": {"us": sel_mean * 1e6, "bytes": select_bytes(wl),
                                 "gbs": select_bytes(wl) / sel_mean / 1e9,
                                 "hbm_frac": select_bytes(wl) / sel_mean / 1e9 / peaks["hbm_gbs"]},
            "hf_select_blocks_two_stage": {"us": statistics.mean(t_sel2) * 1e6, "n_frames": TWO_STAGE_FRAMES,
                                           "bytes": select_bytes(wl),
                                           "gbs": select_bytes(wl) / statistics.mean(t_sel2) / 1e9,
                                           "hbm_frac": select_bytes(wl) / statistics.mean(t_sel2) / 1e9
                                           / peaks["hbm_gbs"]},
            "hf_select_blocks_cached": {"us": statistics.mean(t_selc) * 1e6,
                                        "push_us": statistics.mean(t_push) * 1e6,
                                        "push_and_select_one_call_us": statistics.mean(t_selcp) * 1e6,
                                        "granule": KPOOL_GRANULE,
                                        "note": "per step: hf_kpool_push of the 4680 new keys (and eviction "
                                                "of the oldest 4680), then the selection from the granule sums; "
                                                "hf_select_blocks_cached_push does both in one call"},
            "hf_absorb_evicted_step": {"us": abs_mean * 1e6, "tokens": wl.Ne_step,
                                       "bytes": absorb_bytes(wl, wl.Ne_step),
                                       "gbs": absorb_bytes(wl, wl.Ne_step) / abs_mean / 1e9},
            "hf_hybrid_attn_fwd_absorb": {"us": statistics.mean(t_fused) * 1e6,
                                          "saved_us": (fwd_mean + abs_mean - statistics.mean(t_fused)) * 1e6,
                                          "note": "attention + the step's absorption in one call, against the two "
                                                  "calls timed alone"},
            "rope": {"d_t": ROPE_DT, "cap": ROPE_CAP, "q_frame0": wl.window_frames - wl.chunk_frames,
                     "hf_select_blocks_rope_us": statistics.mean(t_sel_rope) * 1e6,
                     "hf_hybrid_attn_fwd_rope_us": statistics.mean(t_fwd_rope) * 1e6,
                     "attn_tflops": F_rope / statistics.mean(t_fwd_rope) / 1e12,
                     "attn_frac": F_rope / statistics.mean(t_fwd_rope) / 1e12 / peaks["bf16_tflops"],
                     "attn_cost_vs_plain": statistics.mean(t_fwd_rope) / fwd_mean - 1.0,
                     "select_cost_vs_plain": statistics.mean(t_sel_rope) / sel_mean - 1.0},
            "hf_absorb_evicted_state_build": {"us": build_mean * 1e6, "tokens": wl.Ne_state,
                                              "bytes": absorb_bytes(wl, wl.Ne_state),
                                              "gbs": absorb_bytes(wl, wl.Ne_state) / build_mean / 1e9,
                                              "hbm_frac": absorb_bytes(wl, wl.Ne_state) / build_mean / 1e9
                                              / peaks["hbm_gbs"]},
            "hbm_peak_gbs": peaks["hbm_gbs"],
        },
        "sweep": {k: dict(v, frac=v["tflops"] / peaks["bf16_tflops"]) for k, v in sweep.items()},
        "keep_schedule": schedule,
        "large_workload": large,
        "gpu_launches": launches,
        "gpu_launches_source": "hf_launch_count() difference over the timed steps (the library's own launches)",
        "attn_launches_per_call": attn_launches / (n_leg + 3),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    log("cpu baseline")
    if world == 1 and not args.no_cpu_baseline:
        # bounded sample of the fp64 oracle on the host cores: whole heads until ~10 s
        ev_k, ev_v = K_ev.cpu(), V_ev.cpu()
        xs = {k: x[k].cpu() for k in ("Q", "K", "V")}
        heads, spent = [], 0.0
        per_call = {"select": 0.0, "attention": 0.0, "absorb": 0.0}
        for h in range(wl.H):
            part = oracle_sample(wl, xs, S.cpu(), z.cpu(), [h], ev_k, ev_v)
            for k in per_call:
                per_call[k] += part[k]
            spent += sum(part.values())
            heads.append(h)
            if spent >= 10.0:
                break
        t_cpu_step = spent / len(heads) * wl.H
        line["cpu_baseline"] = {
            "value": wl.B * wl.Nq / t_cpu_step, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle on {len(heads)} of {wl.H} heads (select + hybrid attention + absorb "
                      f"of the step's {wl.Ne_step} evicted tokens), {spent:.1f} s, scaled to all heads",
            "ms_per_call": {k: v / len(heads) * wl.H * 1e3 for k, v in per_call.items()}}
    print(json.dumps(line), flush=True)


def streaming_e2e_leg(hf, wl, dev, stream, x, st, ws_sel, ws_abs, args, dist) -> dict:
    """Streaming chunk steps end to end through the public API, timed on the device from
    the first host-to-device copy to the last device-to-host copy. Per step: the chunk's
    Q and its new K, V (Nq tokens each) are copied from pinned host memory on an upload
    stream (double-buffered, so step k+1's copy overlaps step k's compute); the window
    (device-resident, ping-pong buffers) drops its oldest Nq tokens (absorbed into the
    state at the end of the previous step) and appends the chunk's keys and values; then
    the selection and, in one call, the chunk's hybrid attention and the absorption of the
    window's oldest chunk, which leaves it at the next step; O goes back to pinned host
    memory on a download stream. Bytes: 3 x Nq x d bf16 per head in, Nq x d bf16 per head out."""
    B, H, Nq, Nk, d = wl.B, wl.H, wl.Nq, wl.Nk, wl.d
    shp = (B, H, Nq, d)
    host_in = [torch.empty(shp, dtype=torch.bfloat16, pin_memory=True) for _ in range(3)]
    host_in[0].copy_(x["Q"].cpu())
    host_in[1].copy_(x["K"][:, :, Nk - Nq:].cpu())
    host_in[2].copy_(x["V"][:, :, Nk - Nq:].cpu())
    host_out = [torch.empty(shp, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    dev_in = [[torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(3)] for _ in range(2)]
    dev_out = [torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    win_k = [x["K"].clone(), torch.empty_like(x["K"])]
    win_v = [x["V"].clone(), torch.empty_like(x["V"])]
    k_ev = torch.empty(shp, dtype=torch.bfloat16, device=dev)
    v_ev = torch.empty(shp, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(B, H, wl.nQB, wl.r, dtype=torch.int32, device=dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    state = {"k": 0, "cur": 0}

    def e2e_step():
        k, b = state["k"], state["k"] % 2
        cur, nxt = state["cur"], 1 - state["cur"]
        if k >= 2:
            up.wait_event(computed[b])        # step k-2 has read this upload buffer
        with torch.cuda.stream(up):
            for i in range(3):
                dev_in[b][i].copy_(host_in[i], non_blocking=True)
            uploaded[b].record(up)
        stream.wait_event(uploaded[b])
        if k >= 2:
            stream.wait_event(downloaded[b])  # O of step k-2 has left this output buffer
        q, k_new, v_new = dev_in[b]
        # the window drops its oldest chunk (absorbed at the end of the previous step) and
        # takes the new one
        win_k[nxt][:, :, :Nk - Nq].copy_(win_k[cur][:, :, Nq:])
        win_v[nxt][:, :, :Nk - Nq].copy_(win_v[cur][:, :, Nq:])
        win_k[nxt][:, :, Nk - Nq:].copy_(k_new)
        win_v[nxt][:, :, Nk - Nq:].copy_(v_new)
        # the chunk that leaves the window next: absorbed right after this step's attention
        k_ev.copy_(win_k[nxt][:, :, :Nq])
        v_ev.copy_(win_v[nxt][:, :, :Nq])
        hf.hf_select_blocks(q, win_k[nxt], wl.block, wl.r, idx_out=idx, ws=ws_sel)
        hf.hf_hybrid_attn_fwd_absorb(q, win_k[nxt], win_v[nxt], wl.block, wl.r, idx, st, k_ev, v_ev,
                                     O=dev_out[b], ws=ws_abs)
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            host_out[b].copy_(dev_out[b], non_blocking=True)
            downloaded[b].record(down)
        state["k"] += 1
        state["cur"] = nxt

    n_e2e = max(3, min(args.steps, 50))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up.wait_stream(stream)
    down.wait_stream(stream)
    e0.record(up)
    for _ in range(n_e2e):
        e2e_step()
    stream.wait_stream(down)
    stream.wait_stream(up)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t = max_over_ranks(e0.elapsed_time(e1) * 1e-3 / n_e2e, dist, dev)
    world = dist.get_world_size() if dist else 1
    nbytes = 2 * B * H * Nq * d
    # the link alone: the same three host-to-device copies per step, nothing else
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(up)
    for j in range(n_e2e):
        with torch.cuda.stream(up):
            for i in range(3):
                dev_in[j % 2][i].copy_(host_in[i], non_blocking=True)
    c1.record(up)
    torch.cuda.synchronize(dev)
    t_copy = c0.elapsed_time(c1) * 1e-3 / n_e2e
    return {"value": job_throughput(world, B, Nq, t), "unit": UNIT, "h2d_bytes_per_step": 3 * nbytes,
            "d2h_bytes_per_step": nbytes, "steps": n_e2e, "ms_per_step": t * 1e3,
            "h2d_gbs": 3 * nbytes / t / 1e9, "h2d_copies_alone_gbs": 3 * nbytes / t_copy / 1e9,
            "note": "streaming: per step the chunk's Q, K, V (4680 tokens) in from pinned host memory on an upload "
                    "stream overlapping the previous step, window shift on the device, select, attention + "
                    "absorption of the chunk leaving the window (one call), O out to pinned host memory"}


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["hf", "reference"], default="hf")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle CPU-baseline leg")
    ap.add_argument("--no-large", action="store_true", help="skip the 1280x720 leg")
    ap.add_argument("--verbose", action="store_true", help="progress lines on stderr")
    ap.add_argument("--watchdog", type=float, default=0.0,
                    help="dump the Python stacks and exit if the run exceeds this many seconds")
    args = ap.parse_args()
    global _VERBOSE
    _VERBOSE = args.verbose
    if args.watchdog > 0:
        faulthandler.dump_traceback_later(args.watchdog, exit=True)
    wl = WORKLOADS[WORKLOAD]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
