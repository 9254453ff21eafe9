"""hf_select_blocks_noalloc: the select call served from the library's fixed scratch.

Collected last (file name), so that on a GPU it runs both alone and after every other
test. Each GPU case calls the existing hf_select_blocks (with a workspace) and then the
no-workspace entry twice in a row, all through the C ABI, and compares: the same kernels
run on the same bytes, so the block lists must be identical and the scores equal within
the select tolerance (they are expected bit-identical). The CPU cases check the argument
and size checks, which return before any CUDA call.
"""
import ctypes

import pytest
import torch

import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200 import _binding as B
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, frame_structured
from tests.parity import SCORE_ABS

A = 0x100000  # a 16-byte aligned fake device address; never dereferenced on the CPU paths


def _noalloc_raw(**kw):
    a = dict(Q=A, K=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, scores=None)
    a.update(kw)
    return hf.lib().hf_select_blocks_noalloc(a["Q"], a["K"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["block"],
                                             a["r"], a["idx"], a["scores"], None)


def test_noalloc_rejects_before_any_cuda_call():
    assert _noalloc_raw(d=96) == B.HF_ERR_UNSUPPORTED
    assert _noalloc_raw(block=48) == B.HF_ERR_UNSUPPORTED
    assert _noalloc_raw(r=0) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(r=9) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(Nk=0) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(B=0) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(Nq=0) == B.HF_OK  # empty query chunk: nothing to do, no set-up
    # pointer, alignment and key-block limits are checked before the set-up too
    assert _noalloc_raw(Q=None) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(idx=None) == B.HF_ERR_INVALID_ARG
    assert _noalloc_raw(idx=A + 4) == B.HF_ERR_ALIGNMENT
    assert _noalloc_raw(K=A + 2) == B.HF_ERR_ALIGNMENT
    assert _noalloc_raw(scores=A + 8) == B.HF_ERR_ALIGNMENT
    assert _noalloc_raw(Nk=8193 * 32, r=2) == B.HF_ERR_UNSUPPORTED  # more than 8192 key blocks


def test_noalloc_size_limit():
    assert B.HF_SELECT_NOALLOC_SCRATCH_BYTES == 16 << 20
    # 80 heads x 10800 query x 43200 key tokens (d 128, block 128): 17.3 MB of pooled rows
    shape = dict(B=2, H=40, Nq=10800, Nk=43200, d=128, block=128, r=68)
    need = hf.hf_workspace_size(B.HF_WS_SELECT, shape["B"], shape["H"], shape["Nq"], shape["Nk"], shape["d"],
                                shape["block"], shape["r"])
    assert need > B.HF_SELECT_NOALLOC_SCRATCH_BYTES
    assert _noalloc_raw(**shape) == B.HF_ERR_WORKSPACE
    # one head fewer per batch fits
    shape["H"] = 30
    need = hf.hf_workspace_size(B.HF_WS_SELECT, shape["B"], shape["H"], shape["Nq"], shape["Nk"], shape["d"],
                                shape["block"], shape["r"])
    assert need <= B.HF_SELECT_NOALLOC_SCRATCH_BYTES


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _with_workspace(Q, K, block, r, idx, scores):
    Bn, H, Nq, d = Q.shape
    Nk = K.shape[2]
    ws = torch.empty(hf.hf_workspace_size(B.HF_WS_SELECT, Bn, H, Nq, Nk, d, block, r), dtype=torch.uint8,
                     device=Q.device)
    rc = hf.lib().hf_select_blocks(Q.data_ptr(), K.data_ptr(), Bn, H, Nq, Nk, d, block, r, idx.data_ptr(),
                                   scores.data_ptr() if scores is not None else None, ws.data_ptr(), ws.numel(),
                                   _stream())
    assert rc == B.HF_OK, hf.hf_status_string(rc)


def _without_workspace(Q, K, block, r, idx, scores):
    Bn, H, Nq, d = Q.shape
    Nk = K.shape[2]
    rc = hf.lib().hf_select_blocks_noalloc(Q.data_ptr(), K.data_ptr(), Bn, H, Nq, Nk, d, block, r, idx.data_ptr(),
                                           scores.data_ptr() if scores is not None else None, _stream())
    assert rc == B.HF_OK, hf.hf_status_string(rc)


CASES = [
    # (B, H, Nq, Nk, d, tokens per frame, w, block, r, with scores)
    pytest.param(2, 3, 200, 1000, 64, 64, 0.0, 32, 5, True, id="ragged-d64-b32"),
    pytest.param(1, 5, 300, 700, 128, 100, 0.5, 64, 4, False, id="ragged-d128-b64-noscores"),
    pytest.param(*(lambda w: (w.B, w.H, w.Nq, w.Nk, w.d, w.tokens_per_frame, w.w, w.block, w.r, True))(
        WORKLOADS["832x480"]), id="832x480"),
    pytest.param(*(lambda w: (w.B, w.H, w.Nq, w.Nk, w.d, w.tokens_per_frame, w.w, w.block, w.r, True))(
        WORKLOADS["1280x720"]), id="1280x720"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("Bn,H,Nq,Nk,d,tpf,w,block,r,with_scores", CASES)
def test_noalloc_matches_workspace_entry_twice_in_a_row(Bn, H, Nq, Nk, d, tpf, w, block, r, with_scores):
    dev = "cuda"
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + Nq + Nk)
    Q = frame_structured(gen, Bn, H, Nq, d, tpf, w, dev)
    K = frame_structured(gen, Bn, H, Nk, d, tpf, w, dev)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    assert hf.hf_workspace_size(B.HF_WS_SELECT, Bn, H, Nq, Nk, d, block, r) <= B.HF_SELECT_NOALLOC_SCRATCH_BYTES

    idx_ref = torch.full((Bn, H, nQB, r), -7, dtype=torch.int32, device=dev)
    sc_ref = torch.full((Bn, H, nQB, nKB), float("nan"), device=dev) if with_scores else None
    _with_workspace(Q, K, block, r, idx_ref, sc_ref)

    for call in range(2):
        idx = torch.full_like(idx_ref, -7)
        sc = torch.full_like(sc_ref, float("nan")) if with_scores else None
        _without_workspace(Q, K, block, r, idx, sc)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref), f"call {call}: block lists differ"
        if with_scores:
            torch.testing.assert_close(sc, sc_ref, rtol=0.0, atol=SCORE_ABS, msg=lambda m: f"call {call}: {m}")
    status, word = hf.hf_query_status()
    assert status == B.HF_OK and word == 0


@pytest.mark.gpu
def test_noalloc_python_binding_same_result():
    wl = WORKLOADS["tiny"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed)
    Q = frame_structured(gen, wl.B, wl.H, wl.Nq, wl.d, wl.tokens_per_frame, wl.w, "cuda")
    K = frame_structured(gen, wl.B, wl.H, wl.Nk, wl.d, wl.tokens_per_frame, wl.w, "cuda")
    ref = hf.hf_select_blocks(Q, K, wl.block, wl.r)
    out = torch.full_like(ref, -7)
    hf.hf_select_blocks_noalloc(Q, K, wl.block, wl.r, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
