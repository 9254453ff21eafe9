"""GPU: the pooled-key cache. hf_select_blocks_cached over a window built and moved by
hf_kpool_push must select what the oracle selects over that window's keys (masks exact
except near-ties, scores within SCORE_ABS), through ring wrap-around and windows whose
shift is not a multiple of the block."""
import numpy as np
import pytest
import torch

import hybrid_sparse_linear_hf_b200 as hf
import oracle
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs, frame_structured
from tests.parity import SCORE_ABS, assert_masks_match, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed, B, H, N, d, tpf=64, w=0.5):
    g = torch.Generator().manual_seed(seed)
    return frame_structured(g, B, H, N, d, tpf, w)


def _check(Q, K_window, kp, block, r):
    nQB, nKB = -(-Q.shape[2] // block), -(-K_window.shape[2] // block)
    scores = torch.empty(Q.shape[0], Q.shape[1], nQB, nKB, dtype=torch.float32, device=DEV)
    idx = hf.hf_select_blocks_cached(Q.to(DEV), kp, block, r, scores_out=scores)
    torch.cuda.synchronize()
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_OK, (hf.hf_status_string(rc), hex(word))
    oidx, osc = oracle.select_blocks(f64(Q), f64(K_window), block, r)
    assert np.abs(f64(scores) - osc).max() <= SCORE_ABS
    assert_masks_match(idx.cpu().numpy(), oidx, osc, r)


@pytest.mark.parametrize("B,H,d,G,block,chunks,Nq,r", [
    (1, 2, 64, 8, 32, [72, 72, 112], 64, 3),      # 256 keys in pieces that cut blocks
    (2, 3, 128, 8, 128, [1000, 560, 8], 200, 4),  # ragged last block (1568 = 12 * 128 + 32)
    (1, 2, 128, 32, 64, [640, 320], 100, 5),
    (1, 1, 64, 128, 128, [256, 128, 1024], 129, 7),
    (1, 2, 128, 1, 32, [33, 31, 64], 40, 2),      # one-token granules
])
def test_cached_select_matches_oracle(B, H, d, G, block, chunks, Nq, r):
    Nk = sum(chunks)
    Q = _gen(1, B, H, Nq, d)
    K = _gen(2, B, H, Nk, d)
    sums = torch.empty(B, H, Nk // G + 3, d, dtype=torch.float32, device=DEV)
    kp = hf.hf_kpool_init(sums, G)
    t = 0
    for n in chunks:
        hf.hf_kpool_push(kp, K[:, :, t:t + n].contiguous().to(DEV))
        t += n
    assert kp.n_tokens == Nk
    _check(Q, K, kp, block, r)


def test_cached_select_window_moves_and_ring_wraps():
    """A 256-key window moving by 72 keys a step (not a multiple of the 32-key block) in a
    ring that holds exactly the window: every step wraps the ring."""
    B, H, d, G, block, r = 1, 2, 64, 8, 32, 3
    W, step = 256, 72
    stream_keys = _gen(7, B, H, W + 10 * step, d)
    sums = torch.empty(B, H, W // G, d, dtype=torch.float32, device=DEV)
    kp = hf.hf_kpool_init(sums, G)
    hf.hf_kpool_push(kp, stream_keys[:, :, :W].contiguous().to(DEV))
    for s in range(11):
        lo = s * step
        Q = _gen(100 + s, B, H, 64, d)
        _check(Q, stream_keys[:, :, lo:lo + W], kp, block, r)
        if s < 10:
            hf.hf_kpool_push(kp, stream_keys[:, :, lo + W:lo + W + step].contiguous().to(DEV), n_evict=step)
        assert kp.n_tokens == W


def test_cached_select_832x480_window():
    """The 832x480 window (21 frames of 1560 keys) built from its seven 4680-key chunks with
    8-key granules, then moved by one chunk: the cached selection matches the oracle and the
    uncached one."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, n_evicted=wl.Ne_step)
    Q, K = x["Q"], x["K"]
    new = _gen(11, wl.B, wl.H, wl.Nq, wl.d, tpf=wl.tokens_per_frame, w=wl.w)  # the chunk that enters
    G = 8
    sums = torch.empty(wl.B, wl.H, wl.Nk // G, wl.d, dtype=torch.float32, device=DEV)
    kp = hf.hf_kpool_init(sums, G)
    for c in range(wl.Nk // wl.Nq):
        hf.hf_kpool_push(kp, K[:, :, c * wl.Nq:(c + 1) * wl.Nq].contiguous().to(DEV))
    _check(Q, K, kp, wl.block, wl.r)
    idx_u = hf.hf_select_blocks(Q.to(DEV), K.to(DEV), wl.block, wl.r)
    idx_c = hf.hf_select_blocks_cached(Q.to(DEV), kp, wl.block, wl.r)
    torch.cuda.synchronize()
    assert (idx_u != idx_c).float().mean().item() < 1e-3  # near-ties only
    hf.hf_kpool_push(kp, new.contiguous().to(DEV), n_evict=wl.Nq)
    moved = torch.cat([K[:, :, wl.Nq:], new], dim=2)
    _check(Q, moved, kp, wl.block, wl.r)


@pytest.mark.parametrize("d,G,block,W,step", [(128, 8, 64, 640, 200), (64, 4, 32, 512, 100)])
def test_cached_push_equals_push_then_select(d, G, block, W, step):
    """hf_select_blocks_cached_push (the push's sums computed in the Q pooling launch) gives
    the same ring, blocks and scores, bit for bit, as hf_kpool_push then
    hf_select_blocks_cached, step after step of a moving window that wraps its ring."""
    B, H, r = 2, 3, 3
    keys = _gen(21, B, H, W + 6 * step, d).to(DEV)
    sums_a = torch.zeros(B, H, W // G + 5, d, dtype=torch.float32, device=DEV)
    sums_b = torch.zeros_like(sums_a)
    kp_a, kp_b = hf.hf_kpool_init(sums_a, G), hf.hf_kpool_init(sums_b, G)
    hf.hf_kpool_push(kp_a, keys[:, :, :W].contiguous())
    hf.hf_kpool_push(kp_b, keys[:, :, :W].contiguous())
    for s in range(6):
        Q = _gen(200 + s, B, H, 150, d).to(DEV)
        new = keys[:, :, W + s * step:W + (s + 1) * step].contiguous()
        nKB = -(-W // block)
        sc_a = torch.empty(B, H, -(-150 // block), nKB, dtype=torch.float32, device=DEV)
        sc_b = torch.empty_like(sc_a)
        hf.hf_kpool_push(kp_a, new, n_evict=step)
        idx_a = hf.hf_select_blocks_cached(Q, kp_a, block, r, scores_out=sc_a)
        idx_b = hf.hf_select_blocks_cached_push(Q, kp_b, new, block, r, n_evict=step, scores_out=sc_b)
        torch.cuda.synchronize()
        assert hf.hf_query_status()[0] == hf.HF_OK
        assert (kp_a.c.head, kp_a.c.n_gran) == (kp_b.c.head, kp_b.c.n_gran)
        assert torch.equal(idx_a, idx_b) and torch.equal(sc_a, sc_b)
        assert torch.equal(sums_a, sums_b)
    # and against the oracle over the last window
    _check(Q.cpu(), keys[:, :, 6 * step:6 * step + W].cpu(), kp_b, block, r)
