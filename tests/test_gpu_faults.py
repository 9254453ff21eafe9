"""Failure detection on the GPU without a GPU fault: a test-only switch makes a kernel
skip one barrier arrival, so one of its bounded waits runs out (20 ms here). The kernel
must record HF_ERR_DEVICE_TIMEOUT, drain its own copies and MMAs, free its tensor memory
and return; the context stays usable and the next call is correct."""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, draw_step_inputs
from tests.parity import assert_output_close, assert_state_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_NS = 20_000_000


def _fresh_state(wl):
    S = torch.empty(wl.B, wl.H, wl.d, wl.d, device=DEV)
    z = torch.empty(wl.B, wl.H, wl.d, device=DEV)
    return hf.hf_state_init(S, z)


def test_absorb_timeout_is_reported_and_recoverable():
    wl = WORKLOADS["tiny"]
    x = draw_step_inputs(wl)
    assert hf.hf_query_status()[0] == hf.HF_OK
    st = _fresh_state(wl)
    hf.hf_debug_inject_timeout(2, 1, LIMIT_NS)
    hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_ERR_DEVICE_TIMEOUT, (rc, hex(word))
    assert (word >> 8) & 0xFF == 2, hex(word)  # reported by the absorption kernel
    assert hf.hf_query_status()[0] == hf.HF_OK  # the word was cleared
    st = _fresh_state(wl)
    hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    S_o, z_o = oracle.absorb_batch(f64(x["K_ev"]), f64(x["V_ev"]))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)


@pytest.mark.parametrize("name,H", [("tiny", 1), ("832x480", 2)])
def test_attention_timeout_is_reported_and_recoverable(name, H):
    base = WORKLOADS[name]
    wl = type(base)(base.name, base.B, H, base.d, base.tokens_per_frame, base.chunk_frames,
                    base.window_frames, 1, base.block, base.keep, base.w, base.seed)
    x = draw_step_inputs(wl)
    st = _fresh_state(wl)
    hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
    Q, K, V = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
    idx = hf.hf_select_blocks(Q, K, wl.block, wl.r)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    hf.hf_debug_inject_timeout(3, 1, LIMIT_NS)
    hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx, st)
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_ERR_DEVICE_TIMEOUT, (rc, hex(word))
    assert (word >> 8) & 0xFF == 3, hex(word)
    O = hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx, st)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    want = oracle.hybrid_attention(f64(x["Q"]), f64(x["K"]), f64(x["V"]), idx.cpu().numpy(), f64(st.S),
                                   f64(st.z), wl.block)
    assert_output_close(f64(O), want)


def test_select_timeout_is_reported_and_recoverable():
    """The scoring kernel gives up on the pooled key rows that never arrive in shared
    memory (their bulk copies are not issued)."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, n_evicted=1)
    Q, K = x["Q"][:, :2].contiguous().to(DEV), x["K"][:, :2].contiguous().to(DEV)
    ref = hf.hf_select_blocks(Q, K, wl.block, wl.r)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    hf.hf_debug_inject_timeout(1, 1, LIMIT_NS)
    hf.hf_select_blocks(Q, K, wl.block, wl.r)
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_ERR_DEVICE_TIMEOUT, (rc, hex(word))
    assert (word >> 8) & 0xFF == 1, hex(word)  # reported by the selection's scoring kernel
    assert word & 0xFF == 4, hex(word)  # at the wait for the staged key rows
    idx = hf.hf_select_blocks(Q, K, wl.block, wl.r)
    torch.cuda.synchronize()
    assert hf.hf_query_status()[0] == hf.HF_OK
    assert torch.equal(idx, ref)
