"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Inputs are the seeded bf16 tensors of ``hybrid_sparse_linear_hf_b200.inputs`` drawn on
the CPU; the oracle sees them widened exactly to float64. Tolerances (tests/parity.py):
masks bit-exact except near-ties (pooled scores within 1e-4), outputs max-abs 2e-2 and
rel-L2 5e-3, the fp32 state rel-L2 1e-5. Output parity is checked against the oracle
run on the GPU's own kept-block lists, so a legal tie swap never confounds it.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import hybrid_sparse_linear_hf_b200 as hf
from hybrid_sparse_linear_hf_b200.inputs import WORKLOADS, Workload, draw_step_inputs, frame_structured
from tests.parity import (assert_masks_match, assert_output_close, assert_state_close, f64, SCORE_ABS)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed, B, H, N, d, tpf=64, w=0.0):
    g = torch.Generator().manual_seed(seed)
    return frame_structured(g, B, H, N, d, tpf, w)


def _run_select(Q, K, block, r):
    nQB, nKB = -(-Q.shape[2] // block), -(-K.shape[2] // block)
    scores = torch.empty(Q.shape[0], Q.shape[1], nQB, nKB, dtype=torch.float32, device=DEV)
    idx = hf.hf_select_blocks(Q.to(DEV), K.to(DEV), block, r, scores_out=scores)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), scores.cpu().numpy().astype(np.float64)


def _state_from(K_ev, V_ev, d):
    B, H = K_ev.shape[:2]
    S = torch.empty(B, H, d, d, dtype=torch.float32, device=DEV)
    z = torch.empty(B, H, d, dtype=torch.float32, device=DEV)
    st = hf.hf_state_init(S, z)
    hf.hf_absorb_evicted(st, K_ev.to(DEV), V_ev.to(DEV))
    torch.cuda.synchronize()
    return st


def _check_status():
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_OK, f"device status {rc} word {word:#x}"


# --------------------------------------------------------------------------- select
@pytest.mark.parametrize("B,H,Nq,Nk,d,block,r", [
    (1, 1, 64, 256, 64, 32, 2),        # the tiny workload's shape
    (1, 2, 100, 300, 64, 32, 5),       # ragged query and key tails
    (2, 3, 257, 1000, 128, 128, 3),    # ragged, several heads and batches
    (1, 4, 128, 640, 128, 64, 10),
    (1, 2, 33, 129, 128, 128, 2),      # 1-token key tail
    (1, 1, 64, 4096, 64, 32, 128),     # many key blocks
    (1, 2, 300, 2000, 128, 128, 16),   # r = nKB
    (1, 1, 40, 131072, 128, 128, 64),  # 1024 key blocks: static + dynamic shared memory > 48 KB
])
def test_select_matches_oracle(B, H, Nq, Nk, d, block, r):
    Q = _gen(1, B, H, Nq, d, w=0.5)
    K = _gen(2, B, H, Nk, d, w=0.5)
    idx, scores = _run_select(Q, K, block, r)
    oidx, osc = oracle.select_blocks(f64(Q), f64(K), block, r)
    assert np.abs(scores - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, r)
    _check_status()


@pytest.mark.parametrize("d,nKB", [(128, 384), (128, 385), (64, 768), (64, 769)])
def test_select_staged_boundary(d, nKB):
    """Either side of the largest key-block count whose means (nKB x d fp32) are staged in
    shared memory (192 KB): the staged scoring kernel on transposed means, and the plain one
    on row-major means, against the oracle; the last key block is partial."""
    block, r = 128, 40
    Nk = (nKB - 1) * block + 57
    Q = _gen(11, 1, 2, 3 * block + 5, d, w=0.5)
    K = _gen(12, 1, 2, Nk, d, w=0.5)
    idx, scores = _run_select(Q, K, block, r)
    oidx, osc = oracle.select_blocks(f64(Q), f64(K), block, r)
    assert np.abs(scores - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, r)
    _check_status()


def test_select_ties_lower_index():
    """Duplicated key blocks produce exactly equal pooled scores: the lower index wins."""
    d, block = 64, 32
    base = _gen(3, 1, 1, 4 * block, d)
    K = torch.cat([base, base], dim=2)  # block 4+i duplicates block i
    Q = _gen(4, 1, 1, 2 * block, d)
    for r in range(1, 9):
        idx, scores = _run_select(Q, K, block, r)
        oidx, osc = oracle.select_blocks(f64(Q), f64(K), block, r)
        assert np.array_equal(idx, oidx), (r, idx, oidx)
        for row in idx.reshape(-1, r):
            for J in row:
                if J >= 4:
                    assert J - 4 in row


@pytest.mark.parametrize("nKB,r", [(256, 1), (256, 64), (256, 255), (256, 256), (200, 37), (300, 64), (300, 299)])
def test_select_scores_differing_in_low_bits(nKB, r):
    """Pooled scores 1 + j 2^-20 (exact in fp32: query rows (1, 1, 0, ...), key block J's rows
    (1, j_J 2^-20, 0, ...)), so the order is decided by the low bytes of the keys, with
    every value of j repeated: the kept blocks are the r largest j, the lower J first among
    equal ones, exactly."""
    d, block = 128, 32
    g = torch.Generator().manual_seed(nKB + r)
    j = torch.randint(0, 64, (nKB,), generator=g) * 4 + torch.randint(0, 2, (nKB,), generator=g)
    K = torch.zeros(1, 2, nKB * block, d)
    K[..., 0] = 1.0
    K[0, 0, :, 1] = (j.double() * 2.0 ** -20).repeat_interleave(block).float()
    K[0, 1, :, 1] = (j.flip(0).double() * 2.0 ** -20).repeat_interleave(block).float()
    Q = torch.zeros(1, 2, 2 * block, d)
    Q[..., :2] = 1.0
    Q, K = Q.bfloat16(), K.bfloat16()
    assert torch.equal(K[0, 0, ::block, 1].double(), j.double() * 2.0 ** -20)  # exact in bf16
    idx, scores = _run_select(Q, K, block, r)
    for h, jj in ((0, j), (1, j.flip(0))):
        assert np.array_equal(scores[0, h, 0], (1.0 + jj.double() * 2.0 ** -20).float().numpy())
        order = sorted(range(nKB), key=lambda J: (-int(jj[J]), J))
        want = np.sort(np.array(order[:r], dtype=np.int32))
        for I in range(2):
            assert np.array_equal(idx[0, h, I], want), (h, I)


def _split_bytes(S):
    """The state's split copy from S [B,H,d,d] fp32: per (b, h) the hi tile bf16(S), then the
    lo tile bf16(S - hi), each d/64 chunks of 64 columns n, a chunk d rows k of 128 bytes,
    16-byte group g of row k at position g ^ (k % 8)."""
    B, H, d, _ = S.shape
    hi = S.to(torch.bfloat16)
    lo = (S - hi.float()).to(torch.bfloat16)
    k = torch.arange(d).view(d, 1)
    pos = torch.arange(8).view(1, 8)
    g_at = pos ^ (k % 8)  # group stored at position pos of row k
    tiles = []
    for t in (hi, lo):
        x = t.reshape(B * H, d, d // 64, 8, 8)                                   # [bh][k][c][g][e]
        x = x[:, torch.arange(d).view(d, 1, 1), torch.arange(d // 64).view(1, -1, 1),
              g_at.view(d, 1, 8)]                                              # [bh][k][c][pos][e]
        tiles.append(x.permute(0, 2, 1, 3, 4).reshape(B * H, d * d))           # [bh][c][k][pos][e]
    return torch.stack(tiles, dim=1).reshape(-1).view(torch.uint8)


@pytest.mark.parametrize("d", [64, 128])
def test_state_split_follows_S(d):
    """The split copy kept beside the state equals bf16 hi / lo of S in the readout layout,
    byte for byte: zero after hf_state_init, then after absorptions (separate and fused)."""
    B, H = 1, 3
    S = torch.empty(B, H, d, d, device=DEV)
    z = torch.empty(B, H, d, device=DEV)
    st = hf.hf_state_init(S, z)
    torch.cuda.synchronize()
    assert not st.S_split.any()
    for seed, n in ((1, 300), (2, 64), (3, 1000)):
        hf.hf_absorb_evicted(st, _gen(seed, B, H, n, d, w=0.5).to(DEV), _gen(seed + 10, B, H, n, d).to(DEV))
        torch.cuda.synchronize()
        assert torch.equal(st.S_split.cpu(), _split_bytes(st.S.cpu())), (seed, n)
    Q = _gen(7, B, H, 128, d).to(DEV)
    K = _gen(8, B, H, 512, d).to(DEV)
    V = _gen(9, B, H, 512, d).to(DEV)
    idx = hf.hf_select_blocks(Q, K, 128, 2)
    hf.hf_hybrid_attn_fwd_absorb(Q, K, V, 128, 2, idx, st, K[:, :, :256].contiguous(), V[:, :, :256].contiguous())
    torch.cuda.synchronize()
    _check_status()
    assert torch.equal(st.S_split.cpu(), _split_bytes(st.S.cpu()))


# --------------------------------------------------------------------------- absorb
@pytest.mark.parametrize("B,H,n,d", [(1, 1, 192, 64), (1, 2, 1000, 128), (2, 3, 77, 128), (1, 12, 4680, 128),
                                     (1, 1, 1, 64), (1, 40, 130, 64),
                                     (1, 148, 4000, 128)])  # one slice per head: 63 tiles per CTA
def test_absorb_matches_oracle(B, H, n, d):
    K_ev = _gen(5, B, H, n, d, w=0.5)
    V_ev = _gen(6, B, H, n, d, w=0.5)
    st = _state_from(K_ev, V_ev, d)
    S_o, z_o = oracle.absorb_batch(f64(K_ev), f64(V_ev))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    assert st.n_absorbed == n
    _check_status()


def test_absorb_deterministic_and_incremental():
    d = 128
    K_ev = _gen(7, 1, 3, 3000, d, w=0.5)
    V_ev = _gen(8, 1, 3, 3000, d, w=0.5)
    a = _state_from(K_ev, V_ev, d)
    b = _state_from(K_ev, V_ev, d)
    assert torch.equal(a.S, b.S) and torch.equal(a.z, b.z), "absorption must be bit-reproducible"
    # incremental in uneven pieces == oracle batch
    S = torch.empty(1, 3, d, d, device=DEV)
    z = torch.empty(1, 3, d, device=DEV)
    st = hf.hf_state_init(S, z)
    for lo, hi in [(0, 1), (1, 65), (65, 1000), (1000, 3000)]:
        hf.hf_absorb_evicted(st, K_ev[:, :, lo:hi].contiguous().to(DEV), V_ev[:, :, lo:hi].contiguous().to(DEV))
    torch.cuda.synchronize()
    S_o, z_o = oracle.absorb_batch(f64(K_ev), f64(V_ev))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    _check_status()


# --------------------------------------------------------------------------- attention
def _attn_case(B, H, Nq, Nk, d, block, r, n_state, seed=10, w=0.5, scale=0.0):
    Q = _gen(seed, B, H, Nq, d, w=w)
    K = _gen(seed + 1, B, H, Nk, d, w=w)
    V = _gen(seed + 2, B, H, Nk, d, w=w)
    K_ev = _gen(seed + 3, B, H, n_state, d, w=w)
    V_ev = _gen(seed + 4, B, H, n_state, d, w=w)
    if n_state:
        st = _state_from(K_ev, V_ev, d)
    else:
        S = torch.empty(B, H, d, d, device=DEV)
        z = torch.empty(B, H, d, device=DEV)
        st = hf.hf_state_init(S, z)
    idx = hf.hf_select_blocks(Q.to(DEV), K.to(DEV), block, r)
    O = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), block, r, idx, st, scale=scale)
    torch.cuda.synchronize()
    _check_status()
    return Q, K, V, st, idx.cpu().numpy(), O


@pytest.mark.parametrize("B,H,Nq,Nk,d,block,r,n_state", [
    (1, 1, 64, 256, 64, 32, 2, 192),        # the tiny workload's shape
    (1, 2, 300, 1000, 128, 128, 3, 500),    # ragged query tail (44 rows) and key tail (104)
    (1, 2, 200, 700, 128, 64, 4, 300),
    (1, 2, 100, 300, 128, 32, 3, 64),
    (1, 3, 130, 900, 64, 128, 5, 129),
    (1, 2, 96, 400, 64, 64, 7, 0),          # empty state: O = sparse term
    (2, 2, 256, 1024, 128, 128, 8, 256),    # r = nKB: dense window attention
    (1, 1, 128, 129, 128, 128, 2, 10),      # 1-token key tail
])
def test_attention_matches_oracle(B, H, Nq, Nk, d, block, r, n_state):
    Q, K, V, st, idx, O = _attn_case(B, H, Nq, Nk, d, block, r, n_state)
    want = oracle.hybrid_attention(f64(Q), f64(K), f64(V), idx, f64(st.S), f64(st.z), block)
    assert_output_close(f64(O), want)


def test_attention_dense_equals_window_attention_plus_readout():
    """Keeping every block equals dense sliding-window attention plus the readout."""
    B, H, Nq, Nk, d, block = 1, 2, 64, 256, 64, 32
    Q, K, V, st, idx, O = _attn_case(B, H, Nq, Nk, d, block, 8, 192, seed=20, w=0.0)
    want = oracle.dense_swa(f64(Q), f64(K), f64(V)) + oracle.linear_readout(f64(Q), f64(st.S), f64(st.z))
    assert_output_close(f64(O), want)


def test_attention_custom_scale_and_unsorted_idx():
    B, H, Nq, Nk, d, block, r = 1, 2, 128, 512, 128, 64, 3
    Q, K, V, st, idx, O = _attn_case(B, H, Nq, Nk, d, block, r, 100, seed=30, scale=0.05)
    want = oracle.hybrid_attention(f64(Q), f64(K), f64(V), idx, f64(st.S), f64(st.z), block, scale=0.05)
    assert_output_close(f64(O), want)
    # reversed index order gives the same result
    ridx = torch.from_numpy(np.ascontiguousarray(idx[..., ::-1])).to(DEV)
    O2 = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), block, r, ridx, st, scale=0.05)
    torch.cuda.synchronize()
    assert_output_close(f64(O2), want)


def test_attention_bad_index_is_skipped_and_flagged():
    B, H, Nq, Nk, d, block, r = 1, 1, 64, 256, 64, 32, 3
    Q, K, V, st, idx, O = _attn_case(B, H, Nq, Nk, d, block, r, 64, seed=40)
    bad = idx.copy()
    bad[0, 0, 0, 1] = 99   # out of range: skipped
    bad[0, 0, 1, 0] = -1
    O2 = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), block, r, torch.from_numpy(bad).to(DEV), st)
    rc, word = hf.hf_query_status()
    assert rc == hf.HF_ERR_DEVICE_BAD_INDEX, (rc, hex(word))
    assert hf.hf_query_status()[0] == hf.HF_OK  # cleared
    for I, keep in [(0, [idx[0, 0, 0, 0], idx[0, 0, 0, 2]]), (1, [idx[0, 0, 1, 1], idx[0, 0, 1, 2]])]:
        kidx = np.zeros((1, 1, 2, 2), dtype=np.int32)
        kidx[0, 0, I] = keep
        want = oracle.hybrid_attention_tile(f64(Q), f64(K), f64(V), kidx, f64(st.S), f64(st.z), block, 0, 0, I)
        assert_output_close(f64(O2)[0, 0, I * block:(I + 1) * block], want)


def test_empty_inputs_are_noops():
    d = 64
    S = torch.empty(1, 1, d, d, device=DEV)
    z = torch.empty(1, 1, d, device=DEV)
    st = hf.hf_state_init(S, z)
    e = torch.empty(1, 1, 0, d, dtype=torch.bfloat16, device=DEV)
    hf.hf_absorb_evicted(st, e, e)
    K = _gen(1, 1, 1, 64, d).to(DEV)
    idx = torch.empty(1, 1, 0, 1, dtype=torch.int32, device=DEV)
    hf.hf_select_blocks(e, K, 32, 1, idx_out=idx)
    O = hf.hf_hybrid_attn_fwd(e, K, K, 32, 1, idx, st)
    torch.cuda.synchronize()
    assert O.numel() == 0 and float(S.abs().sum()) == 0.0 and st.n_absorbed == 0
    _check_status()


# --------------------------------------------------------------------------- workloads
def test_tiny_workload_step():
    wl = WORKLOADS["tiny"]
    x = draw_step_inputs(wl)
    Q, K, V, K_ev, V_ev = (x[k] for k in ("Q", "K", "V", "K_ev", "V_ev"))
    st = _state_from(K_ev, V_ev, wl.d)
    idx, scores = _run_select(Q, K, wl.block, wl.r)
    oidx, osc = oracle.select_blocks(f64(Q), f64(K), wl.block, wl.r)
    assert_masks_match(idx, oidx, osc, wl.r)
    O = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), wl.block, wl.r, torch.from_numpy(idx).to(DEV), st)
    torch.cuda.synchronize()
    S_o, z_o = oracle.absorb_batch(f64(K_ev), f64(V_ev))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    want = oracle.hybrid_attention(f64(Q), f64(K), f64(V), idx, S_o, z_o, wl.block)
    assert_output_close(f64(O), want)
    _check_status()


@pytest.mark.parametrize("keep", [1.0, 0.5, 0.25, 0.125])
def test_sparsity_sweep_tiny(keep):
    wl = WORKLOADS["tiny"].with_keep(keep)
    x = draw_step_inputs(wl)
    Q, K, V, K_ev, V_ev = (x[k] for k in ("Q", "K", "V", "K_ev", "V_ev"))
    st = _state_from(K_ev, V_ev, wl.d)
    idx = hf.hf_select_blocks(Q.to(DEV), K.to(DEV), wl.block, wl.r)
    O = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), wl.block, wl.r, idx, st)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    oidx, osc = oracle.select_blocks(f64(Q), f64(K), wl.block, wl.r)
    assert_masks_match(idx, oidx, osc, wl.r)
    want = oracle.hybrid_attention(f64(Q), f64(K), f64(V), idx, f64(st.S), f64(st.z), wl.block)
    assert_output_close(f64(O), want)
    if keep == 1.0:
        dense = oracle.dense_swa(f64(Q), f64(K), f64(V)) + oracle.linear_readout(f64(Q), f64(st.S), f64(st.z))
        assert_output_close(f64(O), dense)
    _check_status()


def test_streaming_300_steps():
    """300 chunk steps at the tiny shape; each step evicts 3 fresh frames into the state.
    The fp32 state is checked against a float64 batch recompute at steps 10, 100, 300,
    and the step output against the oracle at the same steps."""
    wl = WORKLOADS["tiny"]
    d = wl.d
    S = torch.empty(1, 1, d, d, device=DEV)
    z = torch.empty(1, 1, d, device=DEV)
    st = hf.hf_state_init(S, z)
    ev_k, ev_v = [], []
    for t in range(1, 301):
        x = draw_step_inputs(wl, seed=10000 + t, n_evicted=wl.Ne_step)
        Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
        idx = hf.hf_select_blocks(Qd, Kd, wl.block, wl.r)
        O = hf.hf_hybrid_attn_fwd(Qd, Kd, Vd, wl.block, wl.r, idx, st)
        if t in (10, 100, 300):
            torch.cuda.synchronize()
            S_before, z_before = f64(st.S), f64(st.z)
            want = oracle.hybrid_attention(f64(x["Q"]), f64(x["K"]), f64(x["V"]), idx.cpu().numpy(),
                                           S_before, z_before, wl.block)
            assert_output_close(f64(O), want, what=f"O at step {t}")
        hf.hf_absorb_evicted(st, x["K_ev"].to(DEV), x["V_ev"].to(DEV))
        ev_k.append(x["K_ev"])
        ev_v.append(x["V_ev"])
        if t in (10, 100, 300):
            torch.cuda.synchronize()
            S_o, z_o = oracle.absorb_batch(f64(torch.cat(ev_k, 2)), f64(torch.cat(ev_v, 2)))
            assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    assert st.n_absorbed == 300 * wl.Ne_step
    _check_status()


def test_streaming_832x480_20_steps():
    """20 chunk steps at the 832x480 shape, each evicting 3 fresh frames (4680 tokens per
    head) into the state; at the end the state of two heads against a float64 batch
    recompute, and one step's sampled query blocks against the oracle."""
    wl = WORKLOADS["832x480"]
    d = wl.d
    S = torch.empty(wl.B, wl.H, d, d, device=DEV)
    z = torch.empty(wl.B, wl.H, d, device=DEV)
    st = hf.hf_state_init(S, z)
    heads = (0, wl.H - 1)
    ev_k, ev_v = [], []
    for t in range(1, 21):
        g = torch.Generator().manual_seed(10000 + t)
        K_ev = frame_structured(g, wl.B, wl.H, wl.Ne_step, d, wl.tokens_per_frame, wl.w)
        V_ev = frame_structured(g, wl.B, wl.H, wl.Ne_step, d, wl.tokens_per_frame, wl.w)
        if t == 20:
            # the last step's attention reads the state of the first 19 steps
            x = draw_step_inputs(wl, seed=20000, n_evicted=1)
            Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
            idx = hf.hf_select_blocks(Qd, Kd, wl.block, wl.r)
            O = hf.hf_hybrid_attn_fwd(Qd, Kd, Vd, wl.block, wl.r, idx, st)
            torch.cuda.synchronize()
            S19, z19 = f64(st.S), f64(st.z)
            Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
            Og = f64(O)
            for (b, h, I) in _sample_tiles(wl, 3, seed=2):
                lo, hi = I * wl.block, min((I + 1) * wl.block, wl.Nq)
                want = oracle.hybrid_attention_tile(Q64, K64, V64, idx.cpu().numpy(), S19, z19, wl.block, b, h, I)
                assert_output_close(Og[b, h, lo:hi], want, what=f"O tile {(b, h, I)} at step 20")
        hf.hf_absorb_evicted(st, K_ev.to(DEV), V_ev.to(DEV))
        ev_k.append(K_ev[:, list(heads)])
        ev_v.append(V_ev[:, list(heads)])
    torch.cuda.synchronize()
    _check_status()
    assert st.n_absorbed == 20 * wl.Ne_step
    S_o, z_o = oracle.absorb_batch(f64(torch.cat(ev_k, 2)), f64(torch.cat(ev_v, 2)))
    assert_state_close(f64(st.S[:, list(heads)]), f64(st.z[:, list(heads)]), S_o, z_o)


def _check_every_tile(Og, Q64, K64, V64, idx, S64, z64, block, heads, what="O"):
    """Every query block of the given heads against the oracle, tile by tile (each tile at
    the output tolerances on its own)."""
    Nq = Q64.shape[2]
    n = 0
    for b in range(Q64.shape[0]):
        for h in heads:
            sl = (slice(b, b + 1), slice(h, h + 1))
            want = oracle.hybrid_attention(Q64[sl], K64[sl], V64[sl], idx[sl], S64[sl], z64[sl], block)
            for I, (lo, hi) in enumerate(oracle.block_ranges(Nq, block)):
                assert_output_close(Og[b, h, lo:hi], want[0, 0, lo:hi], what=f"{what} tile {(b, h, I)}")
                n += 1
    return n


def _sample_tiles(wl, n, seed=0):
    rng = np.random.default_rng(seed)
    tiles = {(0, h, int(rng.integers(0, wl.nQB))) for h in rng.integers(0, wl.H, size=n)}
    tiles.add((0, wl.H - 1, wl.nQB - 1))  # the partial last query block
    tiles.add((0, 0, 0))
    return sorted(tiles)


@pytest.mark.parametrize("name", ["832x480"])
def test_full_size_workload_every_tile(name):
    """The full 832x480-shaped step in the bench's launch configuration: every mask, the
    whole state, and the output of every one of the 444 query tiles against the oracle."""
    wl = WORKLOADS[name]
    x = draw_step_inputs(wl)
    Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
    st = _state_from(x["K_ev"], x["V_ev"], wl.d)
    nKB = wl.nKB
    scores = torch.empty(wl.B, wl.H, wl.nQB, nKB, device=DEV)
    idx_t = hf.hf_select_blocks(Qd, Kd, wl.block, wl.r, scores_out=scores)
    O = hf.hf_hybrid_attn_fwd(Qd, Kd, Vd, wl.block, wl.r, idx_t, st)
    torch.cuda.synchronize()
    _check_status()
    idx = idx_t.cpu().numpy()
    Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
    oidx, osc = oracle.select_blocks(Q64, K64, wl.block, wl.r)
    assert np.abs(scores.cpu().numpy() - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, wl.r)
    S_o, z_o = oracle.absorb_batch(f64(x["K_ev"]), f64(x["V_ev"]))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    Og = f64(O)
    n = _check_every_tile(Og, Q64, K64, V64, idx, f64(st.S), f64(st.z), wl.block, range(wl.H))
    assert n == wl.B * wl.H * wl.nQB


def test_1280x720_workload_every_tile_of_four_heads():
    """The 1280x720-shaped step (40 heads, 10800 query x 43200 key tokens, block 128, r 68):
    every mask, every query block of four heads (first, last and two between) and sampled
    query blocks of the others against the oracle. The state holds 2 evicted frames here
    (the attention reads S and z the same way whatever they absorbed; the 120-frame build
    is checked on two heads below)."""
    wl = WORKLOADS["1280x720"]
    x = draw_step_inputs(wl, n_evicted=2 * wl.tokens_per_frame)
    Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
    st = _state_from(x["K_ev"], x["V_ev"], wl.d)
    scores = torch.empty(wl.B, wl.H, wl.nQB, wl.nKB, device=DEV)
    idx_t = hf.hf_select_blocks(Qd, Kd, wl.block, wl.r, scores_out=scores)
    O = hf.hf_hybrid_attn_fwd(Qd, Kd, Vd, wl.block, wl.r, idx_t, st)
    torch.cuda.synchronize()
    _check_status()
    idx = idx_t.cpu().numpy()
    Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
    oidx, osc = oracle.select_blocks(Q64, K64, wl.block, wl.r)
    assert np.abs(scores.cpu().numpy() - osc).max() <= SCORE_ABS
    assert_masks_match(idx, oidx, osc, wl.r)
    S_o, z_o = oracle.absorb_batch(f64(x["K_ev"]), f64(x["V_ev"]))
    assert_state_close(f64(st.S), f64(st.z), S_o, z_o)
    Og = f64(O)
    heads = (0, 13, 26, wl.H - 1)
    n = _check_every_tile(Og, Q64, K64, V64, idx, f64(st.S), f64(st.z), wl.block, heads)
    assert n == 4 * wl.nQB
    for (b, h, I) in _sample_tiles(wl, 6, seed=1):
        lo, hi = I * wl.block, min((I + 1) * wl.block, wl.Nq)
        want = oracle.hybrid_attention_tile(Q64, K64, V64, idx, S_o, z_o, wl.block, b, h, I)
        assert_output_close(Og[b, h, lo:hi], want, what=f"O tile {(b, h, I)}")


def test_1280x720_state_build_sampled_heads():
    """The 1280x720 state build as the bench would run it: 40 heads x 120 frames (432 000
    tokens per head, 3 slices of 2250 tiles per head, so long per-CTA accumulations),
    drawn on the device; two heads checked against the oracle."""
    wl = WORKLOADS["1280x720"]
    g = torch.Generator(device=DEV).manual_seed(wl.seed + 5000)
    K = frame_structured(g, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, DEV)
    V = frame_structured(g, wl.B, wl.H, wl.Ne_state, wl.d, wl.tokens_per_frame, wl.w, DEV)
    st = _state_from(K, V, wl.d)
    _check_status()
    for h in (0, wl.H - 1):
        S_o, z_o = oracle.absorb_batch(f64(K[:, h:h + 1]), f64(V[:, h:h + 1]))
        assert_state_close(f64(st.S[:, h:h + 1]), f64(st.z[:, h:h + 1]), S_o, z_o)
    del K, V


@pytest.mark.parametrize("tail", [128, 50])
@pytest.mark.parametrize("k2,k3", [(40.0, 70.0), (26.0, 30.0)])
def test_attention_online_rescale_mixed_rows(tail, k2, k3):
    """Even query rows meet much larger scores in later blocks while odd rows do not:
    every warp mixes both cases. With (40, 70) the even rows' logits jump by ~15 and ~27
    (log2 units) over the first blocks' (their running max must be raised twice, O
    rescaled); with (26, 30) by ~10 and ~11.5, large p values the running max may keep.
    With a tail of 50 the block that raises the max the most is the partial last one,
    whose padding columns must stay masked when its exponentials are taken again."""
    d, block, Nq, Nk = 128, 128, 256, 3 * 128 + tail
    g = torch.Generator().manual_seed(77)
    Q = torch.randn(1, 2, Nq, d, generator=g) * 0.3
    Q[:, :, 0::2, 0] = 3.0
    K = torch.randn(1, 2, Nk, d, generator=g) * 0.3
    V = torch.randn(1, 2, Nk, d, generator=g)
    K[:, :, 2 * block:3 * block, 0] = k2   # block 2: scores ~3 k2 for even rows
    K[:, :, 3 * block:4 * block, 0] = k3   # block 3: scores ~3 k3 for even rows
    Q, K, V = Q.bfloat16(), K.bfloat16(), V.bfloat16()
    S = torch.empty(1, 2, d, d, device=DEV)
    z = torch.empty(1, 2, d, device=DEV)
    st = hf.hf_state_init(S, z)
    hf.hf_absorb_evicted(st, _gen(1, 1, 2, 100, d).to(DEV), _gen(2, 1, 2, 100, d).to(DEV))
    for order in ([0, 1, 2, 3], [3, 2, 1, 0], [1, 3, 0, 2]):
        idx = torch.tensor(order, dtype=torch.int32).repeat(1, 2, 2, 1).contiguous()
        O = hf.hf_hybrid_attn_fwd(Q.to(DEV), K.to(DEV), V.to(DEV), block, 4, idx.to(DEV), st)
        torch.cuda.synchronize()
        _check_status()
        want = oracle.hybrid_attention(f64(Q), f64(K), f64(V), idx.numpy(), f64(st.S), f64(st.z), block)
        assert_output_close(f64(O), want, what=f"O order {order}")


def test_bench_step_sequence_on_device_drawn_inputs():
    """The bench's loop (select -> hybrid attention -> absorb of the step's evicted
    frames, back to back without host syncs) on inputs drawn by the device generator,
    every query tile of the last step checked against the oracle."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, seed=123, n_evicted=wl.Ne_step, device=DEV)
    S = torch.empty(wl.B, wl.H, wl.d, wl.d, device=DEV)
    z = torch.empty(wl.B, wl.H, wl.d, device=DEV)
    st = hf.hf_state_init(S, z)
    gen = torch.Generator(device=DEV).manual_seed(5)
    bk = frame_structured(gen, wl.B, wl.H, 20 * wl.tokens_per_frame, wl.d, wl.tokens_per_frame, wl.w, device=DEV)
    bv = frame_structured(gen, wl.B, wl.H, 20 * wl.tokens_per_frame, wl.d, wl.tokens_per_frame, wl.w, device=DEV)
    hf.hf_absorb_evicted(st, bk, bv)
    idx = torch.empty(wl.B, wl.H, wl.nQB, wl.r, dtype=torch.int32, device=DEV)
    O = torch.empty_like(x["Q"])
    for _ in range(4):
        hf.hf_select_blocks(x["Q"], x["K"], wl.block, wl.r, idx_out=idx)
        S_before, z_before = st.S.clone(), st.z.clone()
        hf.hf_hybrid_attn_fwd(x["Q"], x["K"], x["V"], wl.block, wl.r, idx, st, O=O)
        hf.hf_absorb_evicted(st, x["K_ev"], x["V_ev"])
    torch.cuda.synchronize()
    _check_status()
    Q64, K64, V64 = f64(x["Q"]), f64(x["K"]), f64(x["V"])
    idx_h = idx.cpu().numpy()
    Og = f64(O)
    n = _check_every_tile(Og, Q64, K64, V64, idx_h, f64(S_before), f64(z_before), wl.block, range(wl.H))
    assert n == wl.B * wl.H * wl.nQB


def test_absorb_beside_next_selection_equals_sequential_steps():
    """A step's absorption on a second stream beside the next step's selection (which does
    not read the state), the next attention waiting for it, gives step after step
    bit-identically the outputs and the state of the sequential select -> attention ->
    absorb: the calls are safe on any stream, their workspaces included."""
    wl = WORKLOADS["832x480"]
    x = draw_step_inputs(wl, seed=321, n_evicted=wl.Ne_step, device=DEV)
    Q, K, V, K_ev, V_ev = x["Q"], x["K"], x["V"], x["K_ev"], x["V_ev"]
    states, outs = [], []
    for _ in range(2):
        S = torch.empty(wl.B, wl.H, wl.d, wl.d, device=DEV)
        z = torch.empty(wl.B, wl.H, wl.d, device=DEV)
        states.append(hf.hf_state_init(S, z))
        outs.append([])
    stream, side = torch.cuda.current_stream(), torch.cuda.Stream()
    absorbed = torch.cuda.Event()
    idx = torch.empty(wl.B, wl.H, wl.nQB, wl.r, dtype=torch.int32, device=DEV)
    idx2 = torch.empty_like(idx)
    for k in range(4):
        # sequential
        hf.hf_select_blocks(Q, K, wl.block, wl.r, idx_out=idx)
        outs[0].append(hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx, states[0]))
        hf.hf_absorb_evicted(states[0], K_ev, V_ev)
        # overlapped: step k absorbs step k-1's frames beside its selection
        side.wait_stream(stream)
        if k > 0:
            hf.hf_absorb_evicted(states[1], K_ev, V_ev, stream=side)
        absorbed.record(side)
        hf.hf_select_blocks(Q, K, wl.block, wl.r, idx_out=idx2)
        stream.wait_event(absorbed)
        outs[1].append(hf.hf_hybrid_attn_fwd(Q, K, V, wl.block, wl.r, idx2, states[1]))
    side.wait_stream(stream)
    hf.hf_absorb_evicted(states[1], K_ev, V_ev, stream=side)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    _check_status()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)
    assert torch.equal(states[0].S, states[1].S) and torch.equal(states[0].z, states[1].z)
    assert torch.equal(states[0].S_split, states[1].S_split)


# --------------------------------------------------------------------------- fused step
@pytest.mark.parametrize("B,H,Nq,Nk,d,block,r,n_state,n_ev", [
    (1, 1, 64, 256, 64, 32, 2, 192, 192),       # the tiny workload's shape
    (1, 3, 300, 1000, 128, 128, 3, 500, 777),   # ragged tails, evicted tokens not a multiple of 64
    (2, 2, 200, 700, 64, 64, 4, 64, 1),         # a single evicted token
    (1, 12, 4680, 32760, 128, 128, 64, 1560, 4680),  # the 832x480 step
])
def test_fused_attention_absorb_equals_separate_calls(B, H, Nq, Nk, d, block, r, n_state, n_ev):
    """hf_hybrid_attn_fwd_absorb gives bit-identically the O of hf_hybrid_attn_fwd (state
    before the absorption) and the state of hf_absorb_evicted afterwards; both agree with
    the oracle."""
    g = torch.Generator().manual_seed(B * 1000 + Nq + n_ev)
    Q, K, V, K0, V0, Ke, Ve = (frame_structured(g, B, H, n, d, 64, 0.5) for n in (Nq, Nk, Nk, n_state, n_state,
                                                                                  n_ev, n_ev))
    Qd, Kd, Vd, Ked, Ved = (t.to(DEV) for t in (Q, K, V, Ke, Ve))
    st_a = _state_from(K0, V0, d)
    st_b = _state_from(K0, V0, d)
    S0, z0 = f64(st_a.S), f64(st_a.z)
    idx = hf.hf_select_blocks(Qd, Kd, block, r)
    O_a = hf.hf_hybrid_attn_fwd(Qd, Kd, Vd, block, r, idx, st_a)
    hf.hf_absorb_evicted(st_a, Ked, Ved)
    O_b = hf.hf_hybrid_attn_fwd_absorb(Qd, Kd, Vd, block, r, idx, st_b, Ked, Ved)
    torch.cuda.synchronize()
    _check_status()
    assert torch.equal(O_a, O_b), "fused O differs from the separate attention call"
    assert torch.equal(st_a.S, st_b.S) and torch.equal(st_a.z, st_b.z), "fused state differs"
    assert st_b.n_absorbed == n_state + n_ev
    S_o, z_o = oracle.absorb(S0, z0, f64(Ke), f64(Ve))
    assert_state_close(f64(st_b.S), f64(st_b.z), S_o, z_o)
    idx_h = idx.cpu().numpy()
    heads = range(H) if H <= 3 else (0, H - 1)
    _check_every_tile(f64(O_b), f64(Q), f64(K), f64(V), idx_h, S0, z0, block, heads, what="fused O")


def test_streaming_832x480_fused_steps():
    """20 chunk steps at the 832x480 shape through the fused call, back to back on one
    stream (each step's absorption overlapping the attention's tail and the next step's
    selection queued behind it): the final state against a float64 batch recompute on two
    heads, and every query tile of the last step's output against the oracle run on the
    state of the 19 steps before it."""
    wl = WORKLOADS["832x480"]
    d = wl.d
    S = torch.empty(wl.B, wl.H, d, d, device=DEV)
    z = torch.empty(wl.B, wl.H, d, device=DEV)
    st = hf.hf_state_init(S, z)
    heads = (0, wl.H - 1)
    x = draw_step_inputs(wl, seed=20001, n_evicted=1)
    Qd, Kd, Vd = x["Q"].to(DEV), x["K"].to(DEV), x["V"].to(DEV)
    idx = hf.hf_select_blocks(Qd, Kd, wl.block, wl.r)
    O = torch.empty_like(Qd)
    ev_k, ev_v = [], []
    snap = None
    for t in range(1, 21):
        g = torch.Generator().manual_seed(30000 + t)
        K_ev = frame_structured(g, wl.B, wl.H, wl.Ne_step, d, wl.tokens_per_frame, wl.w)
        V_ev = frame_structured(g, wl.B, wl.H, wl.Ne_step, d, wl.tokens_per_frame, wl.w)
        if t == 20:
            snap = (st.S.clone(), st.z.clone())
        hf.hf_hybrid_attn_fwd_absorb(Qd, Kd, Vd, wl.block, wl.r, idx, st, K_ev.to(DEV), V_ev.to(DEV), O=O)
        ev_k.append(K_ev[:, list(heads)])
        ev_v.append(V_ev[:, list(heads)])
    torch.cuda.synchronize()
    _check_status()
    assert st.n_absorbed == 20 * wl.Ne_step
    S_o, z_o = oracle.absorb_batch(f64(torch.cat(ev_k, 2)), f64(torch.cat(ev_v, 2)))
    assert_state_close(f64(st.S[:, list(heads)]), f64(st.z[:, list(heads)]), S_o, z_o)
    n = _check_every_tile(f64(O), f64(x["Q"]), f64(x["K"]), f64(x["V"]), idx.cpu().numpy(), f64(snap[0]),
                          f64(snap[1]), wl.block, range(wl.H), what="O at step 20")
    assert n == wl.H * wl.nQB
