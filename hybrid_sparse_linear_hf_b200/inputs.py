"""Seeded synthetic inputs for the hybrid attention chunk step.

This module only draws random numbers and describes workload shapes. It holds
none of the method's arithmetic, so both the fp64 oracle (through the tests) and
the CUDA path consume exactly the same bytes.

Recipe (one tensor at a time, in the order Q, K, V, K_ev, V_ev):
  x[b, h, tok, :] = n[b, h, tok, :] + w * c[b, h, frame(tok), :]
with n, c ~ N(0, 1) in fp32, drawn from one ``torch.Generator`` seeded with the
workload's seed (n first, then c when w != 0), frame(tok) = tok // tokens_per_frame,
then cast fp32 -> bf16 with round-to-nearest-even. The per-frame shared component
c (weight w) gives the block scores the frame structure that a video model's
tokens have; w = 0 gives plain N(0, 1) tensors.

Streaming step t of the long-horizon workload draws its tensors with seed
10000 + t.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from fractions import Fraction

import torch

__all__ = ["Workload", "WORKLOADS", "frame_structured", "draw_step_inputs", "keep_to_r"]


def keep_to_r(keep: float, n_key_blocks: int) -> int:
    """Number of key blocks kept per query block: clamp(ceil(keep * nKB), 1, nKB).

    The keep ratio is read as an exact decimal so that e.g. 0.2 * 338 rounds up to 68
    and 0.25 * 256 gives exactly 64.
    """
    frac = Fraction(str(keep))
    r = math.ceil(frac * n_key_blocks)
    return max(1, min(n_key_blocks, r))


@dataclass(frozen=True)
class Workload:
    """Shapes of one hybrid attention chunk step.

    The query chunk is ``chunk_frames`` frames of ``tokens_per_frame`` tokens; the
    sliding window holds ``window_frames`` frames; the linear state was built from
    ``state_frames`` evicted frames; every chunk step evicts ``evict_frames`` frames.
    """

    name: str
    B: int
    H: int
    d: int
    tokens_per_frame: int
    chunk_frames: int
    window_frames: int
    state_frames: int
    block: int
    keep: float
    w: float
    seed: int
    evict_frames: int = 3
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def Nq(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    @property
    def Nk(self) -> int:
        return self.window_frames * self.tokens_per_frame

    @property
    def Ne_state(self) -> int:
        return self.state_frames * self.tokens_per_frame

    @property
    def Ne_step(self) -> int:
        return self.evict_frames * self.tokens_per_frame

    @property
    def nQB(self) -> int:
        return -(-self.Nq // self.block)

    @property
    def nKB(self) -> int:
        return -(-self.Nk // self.block)

    @property
    def r(self) -> int:
        return keep_to_r(self.keep, self.nKB)

    def with_keep(self, keep: float) -> "Workload":
        return Workload(self.name + f"_keep{keep}", self.B, self.H, self.d, self.tokens_per_frame,
                        self.chunk_frames, self.window_frames, self.state_frames, self.block,
                        keep, self.w, self.seed, self.evict_frames)

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "d": self.d,
                "tokens_per_frame": self.tokens_per_frame, "Nq": self.Nq, "Nk": self.Nk,
                "block": self.block, "keep": self.keep, "r": self.r, "nKB": self.nKB,
                "state_frames": self.state_frames, "evict_frames": self.evict_frames}


WORKLOADS = {
    # 64 tokens/frame, 1-frame chunk, 4-frame window, 3 frames in the state,
    # block 32, top-2 of 8 key blocks, plain N(0,1) tensors, seed 0.
    "tiny": Workload("tiny", B=1, H=1, d=64, tokens_per_frame=64, chunk_frames=1,
                     window_frames=4, state_frames=3, block=32, keep=0.25, w=0.0, seed=0),
    # 832x480 video: 30x52 token grid per frame, 3-frame chunk, 21-frame window,
    # state built from 60 evicted frames, block 128, 25% of key blocks kept.
    "832x480": Workload("832x480", B=1, H=12, d=128, tokens_per_frame=1560, chunk_frames=3,
                        window_frames=21, state_frames=60, block=128, keep=0.25, w=0.5, seed=1),
    # 1280x720 video, 40 heads: 45x80 token grid per frame, 3-frame chunk, 12-frame
    # window, 120 evicted frames in the state, block 128, 20% of key blocks kept.
    "1280x720": Workload("1280x720", B=1, H=40, d=128, tokens_per_frame=3600, chunk_frames=3,
                         window_frames=12, state_frames=120, block=128, keep=0.2, w=0.5, seed=4),
}


def frame_structured(gen: torch.Generator, B: int, H: int, N: int, d: int,
                     tokens_per_frame: int, w: float, device="cpu") -> torch.Tensor:
    """One bf16 tensor [B, H, N, d] = N(0,1) noise + w * per-frame N(0,1) component."""
    x = torch.randn(B, H, N, d, generator=gen, dtype=torch.float32, device=device)
    if w != 0.0 and N > 0:
        n_frames = -(-N // tokens_per_frame)
        c = torch.randn(B, H, n_frames, d, generator=gen, dtype=torch.float32, device=device)
        frame = torch.arange(N, device=device) // tokens_per_frame
        x.add_(c[:, :, frame, :], alpha=w)
    return x.to(torch.bfloat16)


def draw_step_inputs(wl: Workload, seed: int | None = None, n_evicted: int | None = None,
                     device="cpu") -> dict:
    """Q, K, V (window) and K_ev, V_ev (evicted tokens for the state) in bf16.

    ``n_evicted`` defaults to the tokens of the state build (``state_frames``).
    On ``device="cpu"`` the bytes are identical on every machine with this torch.
    """
    seed = wl.seed if seed is None else seed
    n_ev = wl.Ne_state if n_evicted is None else n_evicted
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    t = wl.tokens_per_frame
    Q = frame_structured(gen, wl.B, wl.H, wl.Nq, wl.d, t, wl.w, device)
    K = frame_structured(gen, wl.B, wl.H, wl.Nk, wl.d, t, wl.w, device)
    V = frame_structured(gen, wl.B, wl.H, wl.Nk, wl.d, t, wl.w, device)
    K_ev = frame_structured(gen, wl.B, wl.H, n_ev, wl.d, t, wl.w, device)
    V_ev = frame_structured(gen, wl.B, wl.H, n_ev, wl.d, t, wl.w, device)
    return {"Q": Q, "K": K, "V": V, "K_ev": K_ev, "V_ev": V_ev}
