"""GPU parity of the two-stage (frame, then block) selection against the fp64 oracle.

Light Forcing, German technical summary, section 2.2. The frame stage is compared with
the oracle's frames (swaps allowed only between frames whose fp64 scores are within the
tie tolerance of the n_frames-th best); the block stage is then compared with the oracle's
block ranking restricted to the GPU's own frames (candidates first), with the same
near-tie rule. Inputs are the seeded bf16 tensors of ``inputs.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs, frame_structured
from tests.parity import SCORE_ABS, TIE_TOL, assert_masks_match, assert_output_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_two_stage(Q, K, block, r, T, nf):
    B, H, Nq, d = Q.shape
    Nk = K.shape[2]
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    frames = torch.full((B, H, nQB, nf), -1, dtype=torch.int32, device=DEV)
    scores = torch.empty(B, H, nQB, nKB, dtype=torch.float32, device=DEV)
    idx = hf.hf_select_blocks_two_stage(Q.to(DEV), K.to(DEV), block, r, T, nf, frames_out=frames,
                                        scores_out=scores)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    idx, frames, scores = idx.cpu().numpy(), frames.cpu().numpy(), scores.cpu().numpy()
    Q64, K64 = f64(Q), f64(K)
    oidx, ofr, osc, ofs = oracle.select_blocks_two_stage(Q64, K64, block, r, T, nf)
    assert np.abs(scores - osc).max() <= SCORE_ABS
    # stage 1: frames (near-ties may swap)
    assert_masks_match(frames, ofr, ofs, nf)
    # stage 2: the oracle's ranking on the GPU's frames: candidates first, then score, then J
    want = np.empty_like(idx)
    ranked_scores = np.empty_like(osc)
    for b, h, I in np.ndindex(B, H, nQB):
        cand = np.zeros(nKB, dtype=bool)
        cand[oracle.candidate_blocks(frames[b, h, I], Nk, block, T)] = True
        s = osc[b, h, I]
        want[b, h, I] = np.sort(np.lexsort((np.arange(nKB), -s, ~cand))[:r])
        # the same order as one score: candidates lifted above every other block
        ranked_scores[b, h, I] = np.where(cand, s + 1e6, s)
    assert_masks_match(idx, want, ranked_scores, r)
    return idx, frames


@pytest.mark.parametrize("B,H,Nq,Nk,d,block,T,nf,r", [
    (1, 1, 64, 256, 64, 32, 64, 2, 3),         # the tiny shape, frames of 2 blocks
    (1, 2, 100, 1000, 64, 32, 150, 3, 8),      # frames not a multiple of the block, ragged
    (2, 3, 257, 3000, 128, 128, 400, 2, 4),    # partial last frame and block
    (1, 4, 128, 3120, 128, 128, 1560, 1, 20),  # one frame (13 blocks) < r: filled
    (1, 2, 300, 4096, 128, 64, 128, 8, 16),    # frames of two blocks
    (1, 1, 64, 640, 128, 64, 640, 1, 10),      # one frame = the whole window: one-stage
])
def test_two_stage_matches_oracle(B, H, Nq, Nk, d, block, T, nf, r):
    g = torch.Generator().manual_seed(Nq + Nk + nf)
    Q = frame_structured(g, B, H, Nq, d, T, 0.5)
    K = frame_structured(g, B, H, Nk, d, T, 0.5)
    _check_two_stage(Q, K, block, r, T, nf)


def test_two_stage_all_frames_equals_one_stage():
    g = torch.Generator().manual_seed(5)
    Q = frame_structured(g, 1, 3, 300, 128, 400, 0.5).to(DEV)
    K = frame_structured(g, 1, 3, 4000, 128, 400, 0.5).to(DEV)
    W = -(-4000 // 400)
    two = hf.hf_select_blocks_two_stage(Q, K, 128, 12, 400, W)
    one = hf.hf_select_blocks(Q, K, 128, 12)
    torch.cuda.synchronize()
    assert torch.equal(two, one)


def test_two_stage_832x480_feeds_the_attention():
    """The 832x480 window (21 frames of 1560 tokens), 8 frames then 64 blocks per query
    block; the lists drive hf_hybrid_attn_fwd."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, n_evicted=wl.tokens_per_frame)
    idx, _ = _check_two_stage(x["Q"], x["K"], wl.block, wl.r, wl.tokens_per_frame, 8)
    S = torch.empty(wl.B, wl.H, wl.d, wl.d, device=DEV)
    z = torch.empty(wl.B, wl.H, wl.d, device=DEV)
    st = hf.hf_state_init(S, z)
    hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
    O = hf.hf_hybrid_attn_fwd(x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV), wl.block, wl.r,
                              torch.from_numpy(idx).to(DEV), st)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    # every query tile of the attention over the two-stage lists against the oracle
    Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
    S64, z64 = f64(st.S), f64(st.z)
    Og = f64(O)
    for h in range(wl.H):
        sl = (slice(0, 1), slice(h, h + 1))
        want = oracle.hybrid_attention(Q64[sl], K64[sl], V64[sl], idx[sl], S64[sl], z64[sl], wl.block)
        for I, (lo, hi) in enumerate(oracle.block_ranges(wl.Nq, wl.block)):
            assert_output_close(Og[0, h, lo:hi], want[0, 0, lo:hi], what=f"O tile {(0, h, I)}")
