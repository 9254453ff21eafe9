"""GPU parity of the capped relative temporal RoPE path against the fp64 oracle.

Hybrid Forcing, German technical summary section 2 C; Portuguese technical summary
section 2 B.2. The kernels take raw Q and K and turn them on the fly: the selection pools
the turned tokens (per-frame sums turned by the frame's index), the attention turns the Q
tile and every kept K tile in shared memory (in bf16, the tensor cores' operand type),
and the linear readout reads the raw Q. Oracle: ``oracle.select_blocks_rope`` and
``oracle.hybrid_attention_rope`` in float64; tolerances as for the step without RoPE.
"""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs, frame_structured
from tests.parity import SCORE_ABS, assert_masks_match, assert_output_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _state(K_ev, V_ev, d):
    B, H = K_ev.shape[:2]
    S = torch.empty(B, H, d, d, device=DEV)
    z = torch.empty(B, H, d, device=DEV)
    st = hf.hf_state_init(S, z)
    if K_ev.shape[2]:
        hf.hf_absorb_evicted(st, K_ev.to(DEV), V_ev.to(DEV))
    return st


def _rope_dict(r):
    return {"d_t": r.d_t, "tokens_per_frame": r.tokens_per_frame, "cap": r.cap, "q_frame0": r.q_frame0,
            "base": float(r.base)}


def _run(B, H, T, q_frames, w_frames, d, block, keep_r, d_t, cap, n_state=100, seed=0, w=0.5):
    """A chunk of q_frames frames at the end of a window of w_frames frames of T tokens."""
    g = torch.Generator().manual_seed(seed)
    Nq, Nk = q_frames * T, w_frames * T
    Q, K, V, Ke, Ve = (frame_structured(g, B, H, n, d, T, w) for n in (Nq, Nk, Nk, n_state, n_state))
    rope = hf.hf_rope(d_t, T, cap, w_frames - q_frames)
    st = _state(Ke, Ve, d)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    scores = torch.empty(B, H, nQB, nKB, device=DEV)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    idx = hf.hf_select_blocks_rope(Qd, Kd, block, keep_r, rope, scores_out=scores)
    O = hf.hf_hybrid_attn_fwd_rope(Qd, Kd, Vd, block, keep_r, idx, st, rope)
    torch.cuda.synchronize()
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_OK, (rc, hex(word))
    return Q, K, V, st, rope, idx.cpu().numpy(), scores.cpu().numpy().astype(np.float64), O


@pytest.mark.parametrize("B,H,T,qf,wf,d,block,r,d_t,cap", [
    (1, 2, 64, 1, 4, 64, 32, 2, 16, 2),          # tiny-like: frames of 64, block 32
    (1, 2, 200, 2, 6, 128, 128, 4, 44, 3),       # blocks straddling frames; cap below the window
    (2, 1, 130, 3, 7, 128, 64, 5, 64, 63),       # ragged frames (130 tokens), the whole first chunk turned
    (1, 3, 96, 1, 5, 64, 32, 6, 8, 1),           # cap 1: all but the newest frame at index 0
    (1, 2, 256, 2, 4, 128, 128, 8, 44, 20),      # r = nKB: the dense window, cap above every offset
])
def test_rope_select_and_attention_match_oracle(B, H, T, qf, wf, d, block, r, d_t, cap):
    Q, K, V, st, rope, idx, scores, O = _run(B, H, T, qf, wf, d, block, r, d_t, cap, seed=T + d_t + cap)
    rd = _rope_dict(rope)
    Q64, K64, V64 = f64(Q), f64(K), f64(V)
    oidx, osc = oracle.select_blocks_rope(Q64, K64, block, r, rd)
    assert np.abs(scores - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, r)
    want = oracle.hybrid_attention_rope(Q64, K64, V64, idx, f64(st.S), f64(st.z), block, rd)
    for b in range(B):
        for h in range(H):
            for I, (lo, hi) in enumerate(oracle.block_ranges(Q.shape[2], block)):
                assert_output_close(f64(O)[b, h, lo:hi], want[b, h, lo:hi], what=f"O tile {(b, h, I)}")


def test_rope_cap_zero_is_the_plain_step():
    """With cap 0 every index is 0: the turned attention gives bit-identically the plain
    kernel's output, and the selection the same blocks."""
    B, H, T, d, block, r = 1, 2, 128, 128, 128, 3
    g = torch.Generator().manual_seed(3)
    Q, K, V, Ke, Ve = (frame_structured(g, B, H, n, d, T, 0.5).to(DEV) for n in (2 * T, 8 * T, 8 * T, 64, 64))
    st = _state(Ke, Ve, d)
    rope = hf.hf_rope(44, T, 0, 6)
    idx = hf.hf_select_blocks(Q, K, block, r)
    idx_r = hf.hf_select_blocks_rope(Q, K, block, r, rope)
    O = hf.hf_hybrid_attn_fwd(Q, K, V, block, r, idx, st)
    O_r = hf.hf_hybrid_attn_fwd_rope(Q, K, V, block, r, idx, st, rope)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    assert torch.equal(idx, idx_r)
    assert torch.equal(O, O_r)


def test_rope_832x480_every_tile():
    """The 832x480 step with the temporal slice of 44 dimensions and the cap at 8 frames
    (the 9-frame window of the pages): every mask and every query tile."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, n_evicted=wl.tokens_per_frame)
    rope = hf.hf_rope(44, wl.tokens_per_frame, 8, wl.window_frames - wl.chunk_frames)
    rd = _rope_dict(rope)
    st = _state(x["K_ev"], x["V_ev"], wl.d)
    Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
    scores = torch.empty(wl.B, wl.H, wl.nQB, wl.nKB, device=DEV)
    idx_t = hf.hf_select_blocks_rope(Qd, Kd, wl.block, wl.r, rope, scores_out=scores)
    O = hf.hf_hybrid_attn_fwd_rope(Qd, Kd, Vd, wl.block, wl.r, idx_t, st, rope)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    idx = idx_t.cpu().numpy()
    Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
    oidx, osc = oracle.select_blocks_rope(Q64, K64, wl.block, wl.r, rd)
    assert np.abs(scores.cpu().numpy() - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, wl.r)
    S64, z64, Og = f64(st.S), f64(st.z), f64(O)
    for h in range(wl.H):
        sl = (slice(0, 1), slice(h, h + 1))
        want = oracle.hybrid_attention_rope(Q64[sl], K64[sl], V64[sl], idx[sl], S64[sl], z64[sl], wl.block, rd)
        for I, (lo, hi) in enumerate(oracle.block_ranges(wl.Nq, wl.block)):
            assert_output_close(Og[0, h, lo:hi], want[0, 0, lo:hi], what=f"O tile {(0, h, I)}")
