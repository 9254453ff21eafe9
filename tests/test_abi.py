"""The C-ABI library on the CPU machine: it loads, exports every declared entry point, and
rejects bad arguments before any CUDA call (no GPU needed for these paths)."""
import ctypes
import os
import re

import pytest

import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hf.h")
SIZE_MAX = (1 << (8 * ctypes.sizeof(ctypes.c_size_t))) - 1
A = 0x100000  # a 16-byte aligned fake device address; never dereferenced on these paths


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"HF_API\s+[\w\s\*]+?\b(hf_\w+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = hf.lib()
    names = declared_symbols()
    core = {"hf_state_init", "hf_absorb_evicted", "hf_select_blocks", "hf_hybrid_attn_fwd", "hf_workspace_size",
            "hf_query_status", "hf_status_string", "hf_version", "hf_debug_inject_timeout"}
    assert core <= set(names), sorted(core - set(names))
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/hf.h but not exported"
    assert hf.hf_version().startswith("hf-b200")


def test_status_strings():
    for code in range(8):
        s = hf.hf_status_string(code)
        assert s.startswith("HF_")
    assert "unknown" in hf.hf_status_string(42)


def test_workspace_sizes():
    # select: pooled Q and K, fp32, each 256-byte aligned
    n = hf.hf_workspace_size(B.HF_WS_SELECT, 1, 12, 4680, 32760, 128, 128, 64)
    assert n == 12 * 37 * 128 * 4 + 12 * 256 * 128 * 4
    assert hf.hf_workspace_size(B.HF_WS_ATTN, 1, 12, 4680, 32760, 128, 128, 64) == 0
    assert hf.hf_workspace_size(B.HF_WS_ABSORB, 1, 1, 0, 0, 64, 0, 0) == 0
    # absorb: 12 heads spread over 12 slices each (144 CTAs)
    assert hf.hf_workspace_size(B.HF_WS_ABSORB, 1, 12, 0, 93600, 128, 0, 0) == 12 * 12 * (128 * 128 + 128) * 4
    with pytest.raises(hf.HfError):
        hf.hf_workspace_size(B.HF_WS_SELECT, 1, 1, 64, 256, 96, 32, 2)
    with pytest.raises(hf.HfError):
        hf.hf_workspace_size(B.HF_WS_SELECT, 1, 1, 64, 256, 64, 32, 9)
    with pytest.raises(hf.HfError):
        hf.hf_workspace_size(7, 1, 1, 64, 256, 64, 32, 2)


def _sel(**kw):
    a = dict(Q=A, K=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, scores=None, ws=A, ws_bytes=1 << 20)
    a.update(kw)
    return hf.lib().hf_select_blocks(a["Q"], a["K"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["block"], a["r"],
                                     a["idx"], a["scores"], a["ws"], a["ws_bytes"], None)


def test_select_validation():
    assert _sel(d=96) == B.HF_ERR_UNSUPPORTED
    assert _sel(block=48) == B.HF_ERR_UNSUPPORTED
    assert _sel(r=0) == B.HF_ERR_INVALID_ARG
    assert _sel(r=9) == B.HF_ERR_INVALID_ARG
    assert _sel(Nk=0) == B.HF_ERR_INVALID_ARG
    assert _sel(B=0) == B.HF_ERR_INVALID_ARG
    assert _sel(Q=None) == B.HF_ERR_INVALID_ARG
    assert _sel(Q=A + 2) == B.HF_ERR_ALIGNMENT
    assert _sel(scores=A + 4) == B.HF_ERR_ALIGNMENT
    assert _sel(ws=None) == B.HF_ERR_WORKSPACE
    assert _sel(ws_bytes=100) == B.HF_ERR_WORKSPACE
    assert _sel(Nq=0) == B.HF_OK  # empty query chunk: nothing to launch


def _state(Bn=1, H=1, d=64):
    st = B.HfStateC()
    st.B, st.H, st.d, st.S, st.z, st.S_split, st.n_absorbed = Bn, H, d, A, A, A, 0
    return st


def _fwd(st=None, **kw):
    a = dict(Q=A, K=A, V=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, scale=0.0, O=A)
    a.update(kw)
    st = st or _state()
    return hf.lib().hf_hybrid_attn_fwd(a["Q"], a["K"], a["V"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"],
                                       a["block"], a["r"], a["idx"], ctypes.byref(st), a["scale"], a["O"],
                                       None, 0, None)


def test_attention_validation():
    assert _fwd(d=32) == B.HF_ERR_UNSUPPORTED
    assert _fwd(block=16) == B.HF_ERR_UNSUPPORTED
    assert _fwd(r=9) == B.HF_ERR_INVALID_ARG
    assert _fwd(st=_state(H=2)) == B.HF_ERR_INVALID_ARG
    assert _fwd(st=_state(d=128)) == B.HF_ERR_INVALID_ARG
    assert _fwd(scale=float("nan")) == B.HF_ERR_INVALID_ARG
    assert _fwd(scale=float("inf")) == B.HF_ERR_INVALID_ARG
    assert _fwd(V=None) == B.HF_ERR_INVALID_ARG
    assert _fwd(O=A + 8) == B.HF_ERR_ALIGNMENT
    assert _fwd(idx=A + 4) == B.HF_ERR_ALIGNMENT
    assert _fwd(Nq=0) == B.HF_OK
    assert hf.lib().hf_hybrid_attn_fwd(A, A, A, 1, 1, 64, 256, 64, 32, 2, A, None, 0.0, A, None, 0, None) \
        == B.HF_ERR_INVALID_ARG


def test_state_and_absorb_validation():
    lib = hf.lib()
    st = B.HfStateC()
    assert lib.hf_state_init(None, 1, 1, 64, A, A, A, None) == B.HF_ERR_INVALID_ARG
    assert lib.hf_state_init(ctypes.byref(st), 1, 1, 32, A, A, A, None) == B.HF_ERR_UNSUPPORTED
    assert lib.hf_state_init(ctypes.byref(st), 1, 1, 64, A + 4, A, A, None) == B.HF_ERR_ALIGNMENT
    assert lib.hf_state_init(ctypes.byref(st), 1, 1, 64, A, A, A + 8, None) == B.HF_ERR_ALIGNMENT
    assert lib.hf_state_init(ctypes.byref(st), 1, 1, 64, A, A, None, None) == B.HF_ERR_INVALID_ARG
    assert lib.hf_state_init(ctypes.byref(st), 0, 1, 64, A, A, A, None) == B.HF_ERR_INVALID_ARG
    s = _state()
    s.S_split = None
    assert lib.hf_absorb_evicted(ctypes.byref(s), A, A, 100, A, 1 << 30, None) == B.HF_ERR_INVALID_ARG
    assert _fwd(st=s) == B.HF_ERR_INVALID_ARG
    s = _state()
    assert lib.hf_absorb_evicted(ctypes.byref(s), A, A, -1, A, 1 << 30, None) == B.HF_ERR_INVALID_ARG
    assert lib.hf_absorb_evicted(ctypes.byref(s), A, A, 0, None, 0, None) == B.HF_OK
    assert s.n_absorbed == 0
    assert lib.hf_absorb_evicted(ctypes.byref(s), A, A, 100, A, 16, None) == B.HF_ERR_WORKSPACE
    assert lib.hf_absorb_evicted(ctypes.byref(s), A + 2, A, 100, A, 1 << 30, None) == B.HF_ERR_ALIGNMENT
    assert lib.hf_absorb_evicted(None, A, A, 100, A, 1 << 30, None) == B.HF_ERR_INVALID_ARG


def test_debug_injection_arguments():
    assert hf.lib().hf_debug_inject_timeout(9, 1, 1000) == B.HF_ERR_INVALID_ARG
    assert hf.lib().hf_debug_inject_timeout(2, -1, 1000) == B.HF_ERR_INVALID_ARG
    assert hf.lib().hf_debug_inject_timeout(0, 0, 0) == B.HF_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "libhf.so"))
    with pytest.raises(ImportError):
        B.lib()


def _sel2(**kw):
    a = dict(Q=A, K=A, B=1, H=1, Nq=64, Nk=1000, d=64, block=32, r=4, T=100, nf=2, idx=A, frames=None, scores=None,
             ws=A, ws_bytes=1 << 20)
    a.update(kw)
    return hf.lib().hf_select_blocks_two_stage(a["Q"], a["K"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["block"],
                                               a["r"], a["T"], a["nf"], a["idx"], a["frames"], a["scores"], a["ws"],
                                               a["ws_bytes"], None)


def test_select_two_stage_validation():
    assert _sel2(T=16) == B.HF_ERR_INVALID_ARG      # frames shorter than a block
    assert _sel2(nf=0) == B.HF_ERR_INVALID_ARG
    assert _sel2(nf=11) == B.HF_ERR_INVALID_ARG     # W = 10
    assert _sel2(r=0) == B.HF_ERR_INVALID_ARG
    assert _sel2(r=33) == B.HF_ERR_INVALID_ARG      # nKB = 32
    assert _sel2(d=96) == B.HF_ERR_UNSUPPORTED
    assert _sel2(Nk=4097 * 32, T=64) == B.HF_ERR_UNSUPPORTED  # nKB > 4096
    assert _sel2(Q=None) == B.HF_ERR_INVALID_ARG
    assert _sel2(frames=A + 4) == B.HF_ERR_ALIGNMENT
    assert _sel2(ws_bytes=100) == B.HF_ERR_WORKSPACE
    assert _sel2(Nq=0) == B.HF_OK
    n = hf.hf_workspace_size(B.HF_WS_SELECT_TWO_STAGE, 1, 12, 4680, 32760, 128, 128, 64)
    assert n == 12 * 37 * 128 * 4 + 12 * 256 * 128 * 4 * 4


def _kp(**kw):
    kp = B.HfKpoolC()
    a = dict(B=1, H=2, d=64, G=8, cap=64, sums=A)
    a.update(kw)
    rc = hf.lib().hf_kpool_init(ctypes.byref(kp), a["B"], a["H"], a["d"], a["G"], a["cap"], a["sums"])
    return rc, kp


def test_kpool_validation():
    assert _kp()[0] == B.HF_OK
    rc, kp = _kp(G=16, cap=100)
    assert rc == B.HF_OK and (kp.n_gran, kp.head, kp.granule, kp.capacity) == (0, 0, 16, 100)
    assert _kp(G=3)[0] == B.HF_ERR_INVALID_ARG
    assert _kp(G=256)[0] == B.HF_ERR_INVALID_ARG
    assert _kp(cap=0)[0] == B.HF_ERR_INVALID_ARG
    assert _kp(sums=None)[0] == B.HF_ERR_INVALID_ARG
    assert _kp(d=32)[0] == B.HF_ERR_UNSUPPORTED
    assert _kp(sums=A + 4)[0] == B.HF_ERR_ALIGNMENT
    L = hf.lib()
    _, kp = _kp()
    # errors leave the cache unchanged; none of these reaches a launch
    assert L.hf_kpool_push(ctypes.byref(kp), A, 12, 0, None) == B.HF_ERR_INVALID_ARG   # not whole granules
    assert L.hf_kpool_push(ctypes.byref(kp), A, 0, 8, None) == B.HF_ERR_INVALID_ARG    # evicts more than the window
    assert L.hf_kpool_push(ctypes.byref(kp), A, 65 * 8, 0, None) == B.HF_ERR_INVALID_ARG  # over capacity
    assert L.hf_kpool_push(ctypes.byref(kp), None, 8, 0, None) == B.HF_ERR_INVALID_ARG
    assert L.hf_kpool_push(ctypes.byref(kp), A + 2, 8, 0, None) == B.HF_ERR_ALIGNMENT
    assert (kp.n_gran, kp.head) == (0, 0)
    # evicting only is host bookkeeping: the ring head moves, wrapping at the capacity
    kp.n_gran, kp.head = 40, 50
    assert L.hf_kpool_push(ctypes.byref(kp), None, 0, 20 * 8, None) == B.HF_OK
    assert (kp.n_gran, kp.head) == (20, (50 + 20) % 64)


def test_select_cached_validation():
    L = hf.lib()
    _, kp = _kp()

    def sel(kp_, **kw):
        a = dict(Q=A, Nq=64, block=32, r=2, idx=A, scores=None, ws=A, ws_bytes=1 << 20)
        a.update(kw)
        return L.hf_select_blocks_cached(a["Q"], ctypes.byref(kp_), a["Nq"], a["block"], a["r"], a["idx"],
                                         a["scores"], a["ws"], a["ws_bytes"], None)
    assert sel(kp) == B.HF_ERR_INVALID_ARG            # empty window
    kp.n_gran = 32                                    # 256 key tokens: 8 blocks of 32
    assert sel(kp, Nq=0) == B.HF_OK
    assert sel(kp, r=9) == B.HF_ERR_INVALID_ARG
    assert sel(kp, block=48) == B.HF_ERR_UNSUPPORTED
    _, kp16 = _kp(G=64)
    kp16.n_gran = 4
    assert sel(kp16, block=32) == B.HF_ERR_INVALID_ARG  # the granule does not divide the block
    assert sel(kp, Q=A + 2) == B.HF_ERR_ALIGNMENT
    assert sel(kp, ws_bytes=100) == B.HF_ERR_WORKSPACE
    kp.head = 64
    assert sel(kp) == B.HF_ERR_INVALID_ARG            # a corrupted head


def test_select_cached_push_validation():
    """The fused push + cached selection checks both halves before anything runs: an error
    from either leaves the cache unchanged."""
    L = hf.lib()
    _, kp = _kp()
    kp.n_gran, kp.head = 32, 60   # 256 key tokens: 8 blocks of 32, the window wrapping the ring

    def call(**kw):
        a = dict(Q=A, K=A, n=64, ev=64, Nq=64, block=32, r=2, idx=A, ws=A, ws_bytes=1 << 20)
        a.update(kw)
        return L.hf_select_blocks_cached_push(a["Q"], ctypes.byref(kp), a["K"], a["n"], a["ev"], a["Nq"],
                                              a["block"], a["r"], a["idx"], None, a["ws"], a["ws_bytes"], None)
    assert call(n=12) == B.HF_ERR_INVALID_ARG              # the push: not whole granules
    assert call(n=41 * 8) == B.HF_ERR_INVALID_ARG          # the push: over capacity (32 - 8 + 41 > 64)
    assert call(K=A + 2) == B.HF_ERR_ALIGNMENT              # the push: unaligned keys
    assert call(r=9) == B.HF_ERR_INVALID_ARG                # the select: r above the window's 8 blocks
    assert call(ev=0, r=11) == B.HF_ERR_INVALID_ARG         # ... and above 10 blocks after a push of 64
    assert call(block=48) == B.HF_ERR_UNSUPPORTED
    assert call(Q=A + 2) == B.HF_ERR_ALIGNMENT
    assert call(ws_bytes=100) == B.HF_ERR_WORKSPACE
    assert call(n=0, ev=256) == B.HF_ERR_INVALID_ARG        # the window left empty
    assert (kp.n_gran, kp.head) == (32, 60)
    # evicting only, with no queries, is the push's host bookkeeping alone
    assert call(K=None, n=0, ev=64, Nq=0) == B.HF_OK
    assert (kp.n_gran, kp.head) == (24, (60 + 8) % 64)


def test_kpool_binding_checks_shapes_before_any_call():
    """The Python binding rejects mismatched tensors on the host (no device needed)."""
    import torch

    kp = hf.HfKpool(torch.empty(0))
    kp.c.B, kp.c.H, kp.c.d, kp.c.granule, kp.c.capacity = 1, 2, 64, 8, 16
    with pytest.raises(ValueError):
        hf.hf_kpool_push(kp, torch.empty(1, 3, 8, 64, dtype=torch.bfloat16))   # wrong head count
    with pytest.raises(ValueError):
        hf.hf_kpool_push(kp, torch.empty(1, 2, 8, 32, dtype=torch.bfloat16))   # wrong d
    with pytest.raises(ValueError):
        hf.hf_kpool_init(torch.empty(2, 16, 64), 8)                             # not [B,H,cap,d]
    with pytest.raises(ValueError):
        hf.hf_kpool_init(torch.empty(1, 2, 16, 64), 8)                          # a CPU tensor
    assert kp.n_tokens == 0


def test_binding_checks_every_tensor_shape_before_any_call():
    """Every tensor the binding hands to the library is checked against the shapes that
    Q (or the cache) implies, on the host, before a pointer is taken: a mismatched
    buffer would otherwise be read or written past its end on the device."""
    import torch

    bf = torch.bfloat16
    Q = torch.empty(1, 2, 100, 64, dtype=bf)
    K = torch.empty(1, 2, 300, 64, dtype=bf)          # nQB = 4, nKB = 10 at block 32
    i32 = lambda *s: torch.empty(*s, dtype=torch.int32)  # noqa: E731
    with pytest.raises(ValueError, match="K must be"):
        hf.hf_select_blocks(Q, torch.empty(1, 3, 300, 64, dtype=bf), 32, 2)
    with pytest.raises(ValueError, match="K must be"):
        hf.hf_select_blocks(Q, torch.empty(1, 2, 300, 128, dtype=bf), 32, 2)
    with pytest.raises(ValueError, match="idx_out"):
        hf.hf_select_blocks(Q, K, 32, 2, idx_out=i32(1, 2, 3, 2))
    with pytest.raises(ValueError, match="scores_out"):
        hf.hf_select_blocks(Q, K, 32, 2, idx_out=i32(1, 2, 4, 2), scores_out=torch.empty(1, 2, 4, 9))
    with pytest.raises(ValueError, match="idx_out"):
        hf.hf_select_blocks_two_stage(Q, K, 32, 2, 100, 2, idx_out=i32(1, 2, 4, 3))
    with pytest.raises(ValueError, match="frames_out"):
        hf.hf_select_blocks_two_stage(Q, K, 32, 2, 100, 2, frames_out=i32(1, 2, 4, 3))
    with pytest.raises(ValueError, match="K must be"):
        hf.hf_select_blocks_noalloc(Q, torch.empty(2, 2, 300, 64, dtype=bf), 32, 2, i32(1, 2, 4, 2))
    with pytest.raises(ValueError, match="idx_out"):
        hf.hf_select_blocks_noalloc(Q, K, 32, 2, i32(1, 2, 4, 3))
    with pytest.raises(ValueError, match="scores_out"):
        hf.hf_select_blocks_noalloc(Q, K, 32, 2, i32(1, 2, 4, 2), scores_out=torch.empty(1, 2, 4, 11))
    # attention: V, idx, O and the state against Q and K
    st = hf.HfState(torch.empty(0), torch.empty(0), torch.empty(0, dtype=torch.uint8))
    st.c.B, st.c.H, st.c.d = 1, 2, 64
    V = torch.empty_like(K)
    idx = i32(1, 2, 4, 2)
    with pytest.raises(ValueError, match="V must"):
        hf.hf_hybrid_attn_fwd(Q, K, torch.empty(1, 2, 299, 64, dtype=bf), 32, 2, idx, st)
    with pytest.raises(ValueError, match="idx must"):
        hf.hf_hybrid_attn_fwd(Q, K, V, 32, 2, i32(1, 2, 4, 3), st)
    with pytest.raises(ValueError, match="O must"):
        hf.hf_hybrid_attn_fwd(Q, K, V, 32, 2, idx, st, O=torch.empty(1, 2, 99, 64, dtype=bf))
    st.c.H = 3
    with pytest.raises(ValueError, match="state"):
        hf.hf_hybrid_attn_fwd(Q, K, V, 32, 2, idx, st)
    # the cached selection: Q against the cache
    kp = hf.HfKpool(torch.empty(0))
    kp.c.B, kp.c.H, kp.c.d, kp.c.granule, kp.c.capacity, kp.c.n_gran = 1, 2, 64, 8, 64, 32
    with pytest.raises(ValueError, match="cache"):
        hf.hf_select_blocks_cached(torch.empty(1, 2, 100, 128, dtype=bf), kp, 32, 2)
    with pytest.raises(ValueError, match="idx_out"):
        hf.hf_select_blocks_cached(Q, kp, 32, 2, idx_out=i32(1, 2, 4, 1))


def test_fused_attention_absorb_validation():
    """hf_hybrid_attn_fwd_absorb checks both halves' arguments before any launch."""
    L = hf.lib()

    def call(st=None, **kw):
        a = dict(Q=A, K=A, V=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, scale=0.0, O=A, Kev=A, Vev=A,
                 n=100, ws=A, ws_bytes=1 << 30)
        a.update(kw)
        st = st or _state()
        return L.hf_hybrid_attn_fwd_absorb(a["Q"], a["K"], a["V"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"],
                                           a["block"], a["r"], a["idx"], ctypes.byref(st), a["scale"], a["O"],
                                           a["Kev"], a["Vev"], a["n"], a["ws"], a["ws_bytes"], None)
    assert call(r=9) == B.HF_ERR_INVALID_ARG            # attention argument
    assert call(st=_state(H=2)) == B.HF_ERR_INVALID_ARG
    assert call(O=A + 8) == B.HF_ERR_ALIGNMENT
    assert call(Kev=None) == B.HF_ERR_INVALID_ARG       # absorption argument
    assert call(Vev=A + 2) == B.HF_ERR_ALIGNMENT
    assert call(n=-1) == B.HF_ERR_INVALID_ARG
    assert call(ws=None) == B.HF_ERR_WORKSPACE
    assert call(ws_bytes=16) == B.HF_ERR_WORKSPACE
    st = _state()
    assert call(st=st, Nq=0, n=0, Kev=None, Vev=None, ws=None) == B.HF_OK   # nothing to do
    assert st.n_absorbed == 0


def test_rope_validation():
    """The RoPE entry points reject an invalid or missing rope before any launch."""
    L = hf.lib()

    def sel(rope, **kw):
        a = dict(Q=A, K=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, ws=A, ws_bytes=1 << 20)
        a.update(kw)
        return L.hf_select_blocks_rope(a["Q"], a["K"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["block"], a["r"],
                                       ctypes.byref(rope) if rope is not None else None, a["idx"], None, a["ws"],
                                       a["ws_bytes"], None)

    def fwd(rope, **kw):
        a = dict(Q=A, K=A, V=A, B=1, H=1, Nq=64, Nk=256, d=64, block=32, r=2, idx=A, O=A)
        a.update(kw)
        st = _state()
        return L.hf_hybrid_attn_fwd_rope(a["Q"], a["K"], a["V"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"],
                                         a["block"], a["r"], a["idx"], ctypes.byref(st), 0.0,
                                         ctypes.byref(rope) if rope is not None else None, a["O"], None, 0, None)

    good = hf.hf_rope(16, 64, 3, 3)   # window 256 keys = 4 frames of 64; a 1-frame chunk at frame 3
    for call in (sel, fwd):
        assert call(good, Nq=0) == B.HF_OK
        assert call(None) == B.HF_ERR_INVALID_ARG
        assert call(hf.hf_rope(15, 64, 3, 3)) == B.HF_ERR_INVALID_ARG    # odd d_t
        assert call(hf.hf_rope(66, 64, 3, 3)) == B.HF_ERR_INVALID_ARG    # d_t > d
        assert call(hf.hf_rope(16, 16, 3, 3)) == B.HF_ERR_INVALID_ARG    # frames shorter than a block
        assert call(hf.hf_rope(16, 64, 64, 3)) == B.HF_ERR_INVALID_ARG   # cap > 63
        assert call(hf.hf_rope(16, 64, 3, 4)) == B.HF_ERR_INVALID_ARG    # the chunk past the window
        assert call(hf.hf_rope(16, 64, 3, 3, base=1.0)) == B.HF_ERR_INVALID_ARG
        assert call(hf.hf_rope(16, 64, 3, 3), r=9) == B.HF_ERR_INVALID_ARG
