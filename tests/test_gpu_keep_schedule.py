"""GPU: a video's first chunks under the chunk-aware growth keep schedule (the window
filling up, then full). Every chunk runs select + hybrid attention through the C ABI at
the schedule's r and is checked against the oracle (its own schedule, masks and output).
"""
import dataclasses

import pytest
import torch

import hybrid_sparse_linear_hf_b200 as hf
import oracle
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs
from tests.parity import assert_masks_match, assert_output_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_schedule_chunks_tiny():
    base = WORKLOADS["tiny"]  # 64-token frames, one-frame chunks, a 4-frame window, block 32
    wls = [dataclasses.replace(base, window_frames=min(i + 1, base.window_frames), seed=300 + i) for i in range(7)]
    nKB = [w.nKB for w in wls]
    r, s, _ = hf.hf_keep_schedule(nKB, 0.8, 0.5)
    r_o, s_o, _ = oracle.keep_schedule(nKB, 0.8, 0.5)
    assert r == r_o.tolist() and r[0] == nKB[0]
    for w, r_c in zip(wls, r):
        x = draw_step_inputs(w)
        Q, K, V = (x[k].to(DEV) for k in ("Q", "K", "V"))
        S = torch.empty(w.B, w.H, w.d, w.d, dtype=torch.float32, device=DEV)
        z = torch.empty(w.B, w.H, w.d, dtype=torch.float32, device=DEV)
        st = hf.hf_state_init(S, z)
        hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
        idx = hf.hf_select_blocks(Q, K, w.block, r_c)
        O = hf.hf_hybrid_attn_fwd(Q, K, V, w.block, r_c, idx, st)
        torch.cuda.synchronize()
        idx = idx.cpu().numpy()
        oidx, osc = oracle.select_blocks(f64(x["Q"]), f64(x["K"]), w.block, r_c)
        assert_masks_match(idx, oidx, osc, r_c)
        S_o, z_o = oracle.absorb_batch(f64(x["K_ev"]), f64(x["V_ev"]))
        want = oracle.hybrid_attention(f64(x["Q"]), f64(x["K"]), f64(x["V"]), idx, S_o, z_o, w.block)
        assert_output_close(f64(O), want, what=f"O (window {w.Nk} tokens, r {r_c})")
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_OK, (hf.hf_status_string(rc), hex(word))
