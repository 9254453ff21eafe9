"""Pins of the fp64 oracle against things other than itself.

Each ``check_*`` takes an oracle namespace (the real module, or a copy with a
planted mistake) and raises AssertionError when the oracle disagrees with:
hand-derived worked examples (tests/golden/hand_examples.json), brute-force
enumeration, closed forms, invariants, or a library routine (torch float64).
``tests/test_oracle_pins.py`` runs them on the real oracle and checks that every
planted mistake is caught by at least one of them.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _as4(x):
    """[N, d] -> [1, 1, N, d] float64."""
    return np.asarray(x, dtype=np.float64)[None, None]


# ---------------------------------------------------------------------------
# phi
# ---------------------------------------------------------------------------
def check_phi_library(o):
    """phi = torch's elu + 1 (float64) on a grid spanning both branches and 0."""
    x = np.concatenate([np.linspace(-20, 20, 4001), [0.0, -0.0, 1e-300, -1e-300, 88.0, -700.0]])
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    got = o.phi(x)
    # elu(x) + 1 = (exp(x) - 1) + 1 carries ~1e-16 absolute cancellation error for x < 0
    assert np.allclose(got, ref, rtol=1e-15, atol=4e-16), "phi != elu + 1"
    neg = x < -1.0
    assert np.allclose(got[neg], np.exp(x[neg]), rtol=1e-15, atol=0.0), "phi(x<=0) != exp(x)"
    assert np.all(got > 0.0), "phi must be positive"


# ---------------------------------------------------------------------------
# pooling and selection
# ---------------------------------------------------------------------------
def check_pool_by_hand(o):
    """Block means over valid rows, written out with python loops on a ragged case."""
    rng = np.random.default_rng(5)
    X = rng.integers(-4, 5, size=(1, 2, 7, 3)).astype(np.float64)
    block = 3
    got = o.pool_blocks(X, block)
    assert got.shape == (1, 2, 3, 3)
    for h in range(2):
        for t, (lo, hi) in enumerate([(0, 3), (3, 6), (6, 7)]):
            for c in range(3):
                s = 0.0
                for i in range(lo, hi):
                    s += X[0, h, i, c]
                assert abs(got[0, h, t, c] - s / (hi - lo)) < 1e-14


def check_selection_golden(o):
    g = _golden()["selection"]
    Q, K, block = _as4(g["Q"]), _as4(g["K"]), g["block"]
    s = o.block_scores(Q, K, block)[0, 0, 0]
    assert np.allclose(s, g["scores"], atol=1e-15, rtol=0), f"scores {s}"
    for r, want in g["idx_by_r"].items():
        idx, _ = o.select_blocks(Q, K, block, int(r))
        assert idx[0, 0, 0].tolist() == want, f"r={r}: {idx[0, 0, 0].tolist()} != {want}"


def _brute_force_topr(s, r):
    """The unique size-r set M with: for j in M, j' not in M, s_j > s_j' or (s_j == s_j' and j < j')."""
    n = len(s)
    found = []
    for M in itertools.combinations(range(n), r):
        Ms = set(M)
        ok = all((s[j] > s[jj]) or (s[j] == s[jj] and j < jj)
                 for j in M for jj in range(n) if jj not in Ms)
        if ok:
            found.append(list(M))
    assert len(found) == 1, f"expected exactly one dominant subset, got {found}"
    return found[0]


def check_selection_bruteforce(o):
    """Brute force over all C(nKB, r) subsets, integer scores so that ties are common."""
    rng = np.random.default_rng(11)
    nKB, d = 8, 4
    for trial in range(12):
        # one 1-token query block q = e0 and 1-token key blocks with k[0] = score:
        # pooled score s_J = k_J[0] exactly.
        sc = rng.integers(-3, 4, size=nKB).astype(np.float64)
        Q = np.zeros((1, 1, 1, d))
        Q[0, 0, 0, 0] = 1.0
        K = rng.normal(size=(1, 1, nKB, d))
        K[0, 0, :, 0] = sc
        for r in range(1, nKB + 1):
            idx, s = o.select_blocks(Q, K, 1, r)
            assert np.array_equal(s[0, 0, 0], sc)
            assert idx[0, 0, 0].tolist() == _brute_force_topr(sc.tolist(), r), (trial, r)


def check_selection_ties_constructed(o):
    """Duplicated key blocks give exactly equal pooled scores: the lower index wins."""
    rng = np.random.default_rng(3)
    block, d = 4, 8
    base = rng.normal(size=(6, block, d))
    # key blocks 0..11 where block 6+i duplicates block i
    Kb = np.concatenate([base, base], axis=0)
    K = Kb.reshape(1, 1, 12 * block, d)
    Q = rng.normal(size=(1, 1, 2 * block, d))
    _, s = o.select_blocks(Q, K, block, 1)
    for I in range(2):
        for r in range(1, 13):
            idx, _ = o.select_blocks(Q, K, block, r)
            got = idx[0, 0, I].tolist()
            assert got == _brute_force_topr(s[0, 0, I].tolist(), r)
            # with duplicates, a kept upper copy implies its lower twin is kept
            for J in got:
                if J >= 6:
                    assert J - 6 in got


def check_selection_output_form(o):
    rng = np.random.default_rng(9)
    Q = rng.normal(size=(2, 3, 70, 16))
    K = rng.normal(size=(2, 3, 150, 16))
    idx, s = o.select_blocks(Q, K, 32, 3)
    assert idx.shape == (2, 3, 3, 3) and idx.dtype == np.int32
    assert s.shape == (2, 3, 3, 5)
    assert np.all(np.diff(idx, axis=-1) > 0), "kept blocks must be ascending and distinct"
    assert idx.min() >= 0 and idx.max() < 5


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def check_attention_golden(o):
    g = _golden()["attention"]
    Q, K, V = _as4(g["Q"]), _as4(g["K"]), _as4(g["V"])
    idx = np.asarray(g["idx"], dtype=np.int32)[None, None, None, :]
    got = o.sparse_attention(Q, K, V, idx, g["block"])[0, 0, 0]
    assert np.allclose(got, g["O"], atol=1e-12, rtol=0), f"{got} != {g['O']}"


def check_attention_dense_equivalence(o):
    """With every block kept the sparse term equals dense attention: the oracle's own
    dense form and torch's float64 scaled_dot_product_attention."""
    rng = np.random.default_rng(21)
    B, H, Nq, Nk, d, block = 1, 2, 45, 100, 16, 16  # ragged query and key tails
    Q, K, V = (rng.normal(size=(B, H, n, d)) for n in (Nq, Nk, Nk))
    nKB = -(-Nk // block)
    idx, _ = o.select_blocks(Q, K, block, nKB)
    assert idx[0, 0, 0].tolist() == list(range(nKB))
    sp = o.sparse_attention(Q, K, V, idx, block)
    dn = o.dense_swa(Q, K, V)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V)).numpy()
    assert np.allclose(sp, ref, atol=1e-12, rtol=0), np.abs(sp - ref).max()
    assert np.allclose(dn, ref, atol=1e-12, rtol=0), np.abs(dn - ref).max()


def check_attention_subset_library(o):
    """A proper subset of blocks equals torch SDPA over exactly those keys."""
    rng = np.random.default_rng(22)
    Nq, Nk, d, block = 20, 77, 8, 8
    Q, K, V = (rng.normal(size=(1, 1, n, d)) for n in (Nq, Nk, Nk))
    keep = [1, 4, 9]  # block 9 is the 5-token partial tail
    idx = np.tile(np.asarray(keep, dtype=np.int32), (1, 1, 3, 1))
    toks = np.concatenate([np.arange(J * block, min((J + 1) * block, Nk)) for J in keep])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K[:, :, toks]), torch.from_numpy(V[:, :, toks])).numpy()
    got = o.sparse_attention(Q, K, V, idx, block)
    assert np.allclose(got, ref, atol=1e-12, rtol=0)


def check_attention_identical_keys(o):
    """Identical keys in the kept blocks give uniform weights: O = mean of their v."""
    rng = np.random.default_rng(23)
    Nq, Nk, d, block = 8, 32, 4, 8
    Q = rng.normal(size=(1, 1, Nq, d))
    K = np.tile(rng.normal(size=(1, 1, 1, d)), (1, 1, Nk, 1))
    V = rng.normal(size=(1, 1, Nk, d))
    idx = np.asarray([[[[0, 3]]]], dtype=np.int32)
    got = o.sparse_attention(Q, K, V, idx, block)
    want = np.concatenate([V[0, 0, 0:8], V[0, 0, 24:32]]).mean(axis=0)
    assert np.allclose(got[0, 0], want[None, :], atol=1e-13)


# ---------------------------------------------------------------------------
# readout and absorption
# ---------------------------------------------------------------------------
def check_absorb_readout_golden(o):
    g = _golden()["absorb_readout"]
    S, z = o.absorb_batch(_as4(g["K_ev"]), _as4(g["V_ev"]))
    assert np.allclose(S[0, 0], g["S"], atol=1e-14, rtol=0), S[0, 0]
    assert np.allclose(z[0, 0], g["z"], atol=1e-14, rtol=0), z[0, 0]
    got = o.linear_readout(_as4(g["Q"]), S, z)[0, 0]
    assert np.allclose(got, g["O_lin"], atol=1e-13, rtol=0), got


def check_absorb_incremental_equals_batch(o):
    rng = np.random.default_rng(31)
    B, H, d = 2, 3, 16
    Ks = [rng.normal(size=(B, H, n, d)) for n in (5, 1, 17, 64)]
    Vs = [rng.normal(size=(B, H, n, d)) for n in (5, 1, 17, 64)]
    S = np.zeros((B, H, d, d))
    z = np.zeros((B, H, d))
    for k, v in zip(Ks, Vs):
        S, z = o.absorb(S, z, k, v)
    Sb, zb = o.absorb_batch(np.concatenate(Ks, axis=2), np.concatenate(Vs, axis=2))
    assert np.allclose(S, Sb, atol=1e-12, rtol=0) and np.allclose(z, zb, atol=1e-12, rtol=0)
    assert np.all(z > 0), "z is a sum of positive features"
    assert S.shape == (B, H, d, d) and z.shape == (B, H, d), "state size independent of tokens"


def check_absorb_single_token(o):
    """One token: S = phi(k) v^T, z = phi(k), phi written out branch by branch."""
    k = np.array([0.5, -1.25, 0.0, 2.0])
    v = np.array([1.0, -2.0, 3.0, 0.25])
    ph = np.array([1.5, math.exp(-1.25), 1.0, 3.0])
    S, z = o.absorb_batch(_as4([k]), _as4([v]))
    assert np.allclose(S[0, 0], np.outer(ph, v), atol=1e-15, rtol=0)
    assert np.allclose(z[0, 0], ph, atol=1e-15, rtol=0)


def check_readout_closed_forms(o):
    """Single-token state: O_lin = v * a / (a + 1e-6) with a = phi(q).phi(k).
    Empty state: O_lin = 0."""
    rng = np.random.default_rng(41)
    d = 8
    k = rng.normal(size=d)
    v = rng.normal(size=d)
    q = rng.normal(size=(5, d))
    S, z = o.absorb_batch(_as4([k]), _as4([v]))
    got = o.linear_readout(_as4(q), S, z)[0, 0]
    pk = np.where(k > 0, k + 1, np.exp(np.minimum(k, 0)))
    pq = np.where(q > 0, q + 1, np.exp(np.minimum(q, 0)))
    a = pq @ pk
    assert np.allclose(got, (a / (a + 1e-6))[:, None] * v[None, :], atol=1e-14, rtol=0)
    zero = o.linear_readout(_as4(q), np.zeros((1, 1, d, d)), np.zeros((1, 1, d)))
    assert np.all(zero == 0.0)


def check_hybrid_sum(o):
    """O = O_s + O_lin; with an empty state O = O_s."""
    rng = np.random.default_rng(51)
    Q, K, V = (rng.normal(size=(1, 2, n, 8)) for n in (16, 40, 40))
    idx, _ = o.select_blocks(Q, K, 8, 2)
    S, z = o.absorb_batch(rng.normal(size=(1, 2, 30, 8)), rng.normal(size=(1, 2, 30, 8)))
    hyb = o.hybrid_attention(Q, K, V, idx, S, z, 8)
    assert np.allclose(hyb, o.sparse_attention(Q, K, V, idx, 8) + o.linear_readout(Q, S, z), atol=1e-14)
    empty = o.hybrid_attention(Q, K, V, idx, np.zeros((1, 2, 8, 8)), np.zeros((1, 2, 8)), 8)
    assert np.allclose(empty, o.sparse_attention(Q, K, V, idx, 8), atol=0, rtol=0)
    tile = o.hybrid_attention_tile(Q, K, V, idx, S, z, 8, 0, 1, 1)
    assert np.allclose(tile, hyb[0, 1, 8:16], atol=1e-14)


# ---------------------------------------------------------------------------
# two-stage (frame, then block) selection
# ---------------------------------------------------------------------------
def check_two_stage_golden(o):
    g = _golden()["two_stage_selection"]
    Q, block, T = _as4(g["Q"]), g["block"], g["tokens_per_frame"]
    for case in g["cases"]:
        K = _as4(case["K"])
        f = o.frame_scores(Q, K, block, T)[0, 0, 0]
        assert np.allclose(f, case["frame_scores"], atol=1e-15, rtol=0), f"frame scores {f}"
        s = o.block_scores(Q, K, block)[0, 0, 0]
        assert np.allclose(s, case["block_scores"], atol=1e-15, rtol=0), f"block scores {s}"
        for e in case["expect"]:
            idx, frames, _, _ = o.select_blocks_two_stage(Q, K, block, e["r"], T, e["n_frames"])
            assert frames[0, 0, 0].tolist() == e["frames"], (e, frames[0, 0, 0].tolist())
            assert idx[0, 0, 0].tolist() == e["idx"], (e, idx[0, 0, 0].tolist())


def check_two_stage_all_frames_is_one_stage(o):
    """Keeping every frame makes every block a candidate: the one-stage selection."""
    rng = np.random.default_rng(21)
    Q = rng.standard_normal((1, 2, 70, 8))
    K = rng.standard_normal((1, 2, 333, 8))
    block, T = 16, 50
    W = -(-333 // T)
    for r in (1, 5, 21):
        idx2, _, _, _ = o.select_blocks_two_stage(Q, K, block, r, T, W)
        idx1, _ = o.select_blocks(Q, K, block, r)
        assert np.array_equal(idx1, idx2), f"r={r}"


def check_two_stage_frames_are_blocks(o):
    """With frames of one block each and r frames kept, the frames are the top-r blocks."""
    rng = np.random.default_rng(22)
    Q = rng.standard_normal((1, 1, 64, 4))
    K = rng.standard_normal((1, 1, 200, 4))
    block, r = 16, 4
    idx2, frames, _, _ = o.select_blocks_two_stage(Q, K, block, r, block, r)
    idx1, _ = o.select_blocks(Q, K, block, r)
    assert np.array_equal(idx1, idx2)
    assert np.array_equal(frames, idx1)


def _two_stage_brute(q_tokens, k_tokens, block, T, n_frames, r):
    """Independent statement with python lists and sets: integer-valued inputs, exact means."""
    qm = [sum(col) / len(q_tokens) for col in zip(*q_tokens)]
    Nk = len(k_tokens)
    frames = [list(range(w * T, min((w + 1) * T, Nk))) for w in range(-(-Nk // T))]
    blocks = [list(range(J * block, min((J + 1) * block, Nk))) for J in range(-(-Nk // block))]
    mean = lambda toks: [sum(k_tokens[t][c] for t in toks) / len(toks) for c in range(len(qm))]  # noqa: E731
    dot = lambda a, b: sum(x * y for x, y in zip(a, b))  # noqa: E731
    fs = [dot(qm, mean(fr)) for fr in frames]
    kept = sorted(sorted(range(len(frames)), key=lambda w: (-fs[w], w))[:n_frames])
    kept_tokens = set(t for w in kept for t in frames[w])
    cand = [J for J, toks in enumerate(blocks) if kept_tokens.intersection(toks)]
    bs = {J: dot(qm, mean(blocks[J])) for J in range(len(blocks))}
    ranked = sorted(cand, key=lambda J: (-bs[J], J))
    others = sorted((J for J in range(len(blocks)) if J not in cand), key=lambda J: (-bs[J], J))
    return kept, sorted((ranked + others)[:r])


def check_two_stage_bruteforce(o):
    rng = np.random.default_rng(23)
    for trial in range(12):
        d = int(rng.integers(1, 4))
        block = int(rng.integers(2, 6))
        T = int(rng.integers(block, 3 * block + 2))
        Nk = int(rng.integers(2 * T, 5 * T))
        Nq = int(rng.integers(1, 2 * block + 1))
        Q = rng.integers(-2, 3, size=(1, 1, Nq, d)).astype(np.float64)
        K = rng.integers(-2, 3, size=(1, 1, Nk, d)).astype(np.float64)
        W = -(-Nk // T)
        n_frames = int(rng.integers(1, W + 1))
        r = int(rng.integers(1, -(-Nk // block) + 1))  # may exceed the candidates: filled
        idx, frames, _, _ = o.select_blocks_two_stage(Q, K, block, r, T, n_frames)
        for I in range(-(-Nq // block)):
            qt = Q[0, 0, I * block:min((I + 1) * block, Nq)].tolist()
            kept, want = _two_stage_brute(qt, K[0, 0].tolist(), block, T, n_frames, r)
            assert frames[0, 0, I].tolist() == kept, (trial, I, frames[0, 0, I].tolist(), kept)
            assert idx[0, 0, I].tolist() == want, (trial, I, idx[0, 0, I].tolist(), want)


# ---------------------------------------------------------------------------
# chunk-aware growth (per-chunk keep schedule)
# ---------------------------------------------------------------------------
def check_schedule_golden(o):
    for case in _golden()["keep_schedule"]["cases"]:
        r, s, beta = o.keep_schedule(case["nKB"], case["s_base"], case["s_target"])
        assert r.tolist() == case["r"], (r.tolist(), case["r"])
        assert np.allclose(s, case["s"], atol=1e-6), (s, case["s"])
        assert abs(beta - case["beta"]) < 1e-6, beta


def _feasible_cases(seed, count):
    """Random window sizes (a window filling up, then full), target and s_base with beta >= 0."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        n = int(rng.integers(2, 14))
        full = int(rng.integers(4, 300))
        fill = int(rng.integers(1, 8))
        nKB = [max(1, (full * min(i + 1, fill)) // fill) for i in range(n)]
        t = float(rng.uniform(0.05, 0.9))
        flat = 1.0 - ((1.0 - t) * sum(nKB) - nKB[0]) / sum(nKB[1:])  # s_base with beta = 0
        if not (0.0 <= flat < 0.97):
            continue
        s_base = float(rng.uniform(flat, min(0.99, flat + 0.3)))
        out.append((nKB, s_base, t, flat))
    return out


def check_schedule_budget_and_rounding(o):
    for nKB, s_base, t, _ in _feasible_cases(31, 40):
        try:
            r, s, beta = o.keep_schedule(nKB, s_base, t)
        except ValueError:
            continue  # some s_i below 0: rejected, checked elsewhere
        assert s[0] == 0.0 and r[0] == nKB[0], "the first chunk attends densely"
        kept = sum((1.0 - s[i]) * nKB[i] for i in range(len(nKB)))
        assert abs(kept - (1.0 - t) * sum(nKB)) <= 1e-9 * sum(nKB), "FLOP budget"
        assert all(s[i] <= s[i + 1] + 1e-15 for i in range(1, len(nKB) - 1)), "sparsity grows with i"
        for i, k in enumerate(nKB):
            x = (1.0 - s[i]) * k
            assert 1 <= r[i] <= k
            assert r[i] >= min(x, k) - 1e-9 and (r[i] == 1 or r[i] - 1 < x + 1e-9), (i, x, r[i])


def check_schedule_two_chunks(o):
    """With one sparse chunk, it keeps exactly what the dense first chunk leaves of the budget."""
    for a, b, t, s_base in ((3, 9, 0.4, 0.9), (37, 256, 0.75, 0.95), (1, 1, 0.25, 0.7), (5, 50, 0.6, 0.7)):
        r, s, beta = o.keep_schedule([a, b], s_base, t)
        s1 = 1.0 - ((1.0 - t) * (a + b) - a) / b
        assert abs(s[1] - s1) < 1e-12 and abs(beta - (s_base - s1)) < 1e-12, (s, beta, s1)
        assert r[1] == min(max(math.ceil((1.0 - s1) * b - 1e-12), 1), b)


def check_schedule_noise_scale(o):
    """Later chunks' sparsity gaps to s_base follow 1/sqrt(i): chunk 4 has half chunk 1's
    gap, chunk 9 a third; at the flat s_base (beta = 0) every later chunk has s_base; beta
    agrees with a bisection on the budget."""
    nKB = [20] + [40] * 11
    t = 0.6
    flat = 1.0 - ((1.0 - t) * sum(nKB) - nKB[0]) / sum(nKB[1:])
    _, s, beta = o.keep_schedule(nKB, flat + 0.2, t)
    g = (flat + 0.2) - s
    assert beta > 0 and abs(g[4] / g[1] - 0.5) < 1e-12 and abs(g[9] / g[1] - 1.0 / 3.0) < 1e-12, g
    _, s, beta = o.keep_schedule(nKB, flat + 1e-9, t)  # just above: rounding decides beta's sign at flat
    assert 0.0 <= beta < 1e-8 and np.allclose(s[1:], flat, atol=1e-8)
    # beta by bisection on the budget residual, independent of the closed form
    s_base = flat + 0.1
    lo, hi = 0.0, 1.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        kept = nKB[0] + sum((1.0 - s_base + mid / math.sqrt(i)) * nKB[i] for i in range(1, len(nKB)))
        lo, hi = (mid, hi) if kept < (1.0 - t) * sum(nKB) else (lo, mid)
    _, _, beta = o.keep_schedule(nKB, s_base, t)
    assert abs(beta - lo) < 1e-12, (beta, lo)


def check_schedule_rejects(o):
    def rejected(*a):
        try:
            o.keep_schedule(*a)
        except ValueError:
            return True
        return False
    assert rejected([10, 10], 0.2, 0.5), "s_base below the flat value needs beta < 0"
    assert rejected([], 0.5, 0.5) and rejected([4, 0], 0.5, 0.5)
    assert rejected([4, 4], 1.0, 0.5) and rejected([4, 4], 0.5, -0.1)
    assert rejected([100, 1], 0.99, 0.9), "the budget leaves the later chunk nothing (s_1 >= 1)"
    r, s, _ = o.keep_schedule([7], 0.5, 0.9)
    assert r.tolist() == [7] and s.tolist() == [0.0], "a single chunk is dense"


# ---------------------------------------------------------------------------
# capped relative temporal RoPE
# ---------------------------------------------------------------------------
def check_rope_positions_golden(o):
    """Temporal indices of hand-worked cases (frames, offsets from the newest frame, cap)."""
    for c in _golden()["rope"]["positions"]:
        got = o.rope_positions(c["n_tokens"], c["tokens_per_frame"], c["frame0"], c["n_frames"], c["cap"])
        assert got.tolist() == c["p"], (c, got.tolist())


def check_rope_rotation_closed_form(o):
    """One token, d = 6, d_t = 4, base 100, index 3: pair 0 turns by 3 rad, pair 1 by
    3 * 100**(-1/2) = 0.3 rad (cos/sin from math), dims 4, 5 untouched."""
    x = [1.0, 2.0, 3.0, 4.0, 5.0, 6.0]
    got = o.rope_rotate(_as4([x]), [3], 4, base=100.0)[0, 0, 0]
    c0, s0, c1, s1 = math.cos(3.0), math.sin(3.0), math.cos(0.3), math.sin(0.3)
    want = [1 * c0 - 2 * s0, 1 * s0 + 2 * c0, 3 * c1 - 4 * s1, 3 * s1 + 4 * c1, 5.0, 6.0]
    assert np.allclose(got, want, rtol=0, atol=1e-14), (got, want)


def check_rope_complex_form(o):
    """The same rotation written with complex numbers: pair (x[2i], x[2i+1]) is
    x[2i] + 1j x[2i+1], multiplied by exp(1j p theta_i), theta_i = base**(-2i/d_t)."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((1, 2, 9, 12))
    pos = rng.integers(0, 40, size=9)
    d_t = 8
    got = o.rope_rotate(X, pos, d_t)
    zc = X[..., 0:d_t:2] + 1j * X[..., 1:d_t:2]
    theta = 10000.0 ** (-np.arange(d_t // 2) * 2.0 / d_t)
    zc = zc * np.exp(1j * pos[:, None] * theta[None, :])
    want = X.copy()
    want[..., 0:d_t:2] = zc.real
    want[..., 1:d_t:2] = zc.imag
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def check_rope_norm_inverse_relative(o):
    """A rotation keeps every token's norm, the index -p undoes the index p, and the
    product of two turned vectors depends only on the difference of their indices."""
    rng = np.random.default_rng(12)
    X = rng.standard_normal((1, 1, 7, 16))
    pos = rng.integers(0, 30, size=7)
    Y = o.rope_rotate(X, pos, 10)
    assert np.allclose(np.linalg.norm(Y, axis=-1), np.linalg.norm(X, axis=-1), rtol=1e-13)
    assert np.allclose(o.rope_rotate(Y, -pos, 10), X, atol=1e-12)
    q, k = X[0, 0, 0], X[0, 0, 1]
    for pq, pk, sh in [(5, 2, 7), (0, 9, 3), (4, 4, 11)]:
        a = o.rope_rotate(_as4([q]), [pq], 10)[0, 0, 0] @ o.rope_rotate(_as4([k]), [pk], 10)[0, 0, 0]
        b = o.rope_rotate(_as4([q]), [pq + sh], 10)[0, 0, 0] @ o.rope_rotate(_as4([k]), [pk + sh], 10)[0, 0, 0]
        assert abs(a - b) < 1e-12, (pq, pk, sh, a, b)


def check_rope_cap_and_identity(o):
    """Frames at least `cap` frames old sit at index 0 (unturned); with cap 0 or d_t 0
    the turned step equals the plain one; the selection ranks blocks by the means of the
    turned tokens."""
    rng = np.random.default_rng(13)
    T, W, C, d, block = 8, 5, 2, 8, 8
    Q = rng.standard_normal((1, 1, C * T, d))
    K = rng.standard_normal((1, 1, W * T, d))
    V = rng.standard_normal((1, 1, W * T, d))
    S = np.abs(rng.standard_normal((1, 1, d, d)))
    z = np.abs(rng.standard_normal((1, 1, d)))
    rope = {"d_t": 4, "tokens_per_frame": T, "cap": 2, "q_frame0": W - C}
    Qr, Kr = o.rope_qk(Q, K, rope)
    # by hand: the chunk's frames are window frames 3, 4 (offsets 1, 0: indices 1, 2); the
    # window's frames 0..4 have offsets 4..0, indices 0, 0, 0, 1, 2
    assert np.allclose(Qr, o.rope_rotate(Q, [1] * T + [2] * T, 4), atol=1e-14)
    assert np.allclose(Kr, o.rope_rotate(K, [0] * (3 * T) + [1] * T + [2] * T, 4), atol=1e-14)
    old = slice(0, (W - 2) * T)  # frames 0..2 are >= 2 frames older than the newest
    assert np.array_equal(Kr[:, :, old], K[:, :, old])
    assert not np.allclose(Kr[:, :, (W - 1) * T:], K[:, :, (W - 1) * T:])
    idx = np.tile(np.arange(3, dtype=np.int32), (1, 1, 2, 1))
    for ident in ({"d_t": 0}, {"cap": 0}):
        r2 = dict(rope, **ident)
        assert np.allclose(o.hybrid_attention_rope(Q, K, V, idx, S, z, block, r2),
                           o.hybrid_attention(Q, K, V, idx, S, z, block), atol=1e-13)
    # the sparse branch alone sees the turn; the linear branch reads the raw q
    Qr, Kr = o.rope_qk(Q, K, rope)
    got = o.hybrid_attention_rope(Q, K, V, idx, S, z, block, rope)
    assert np.allclose(got - o.linear_readout(Q, S, z), o.sparse_attention(Qr, Kr, V, idx, block), atol=1e-13)
    # turned keys of the first frame (index 0) and raw ones give the same readout of a
    # state built from them (the linear branch of evicted frames)
    S1, z1 = o.absorb_batch(K[:, :, :T], V[:, :, :T])
    S2, z2 = o.absorb_batch(Kr[:, :, :T], V[:, :, :T])
    assert np.array_equal(S1, S2) and np.array_equal(z1, z2)
    # selection by brute force over the means of the turned tokens
    s = Qr.reshape(1, 1, C * T // block, block, d).mean(3) @ np.swapaxes(
        Kr.reshape(1, 1, W * T // block, block, d).mean(3), -1, -2)
    idx_o, s_o = o.select_blocks_rope(Q, K, block, 2, rope)
    assert np.allclose(s_o, s, atol=1e-12)
    for I in range(2):
        assert idx_o[0, 0, I].tolist() == sorted(_brute_force_topr(s[0, 0, I], 2))


ALL_CHECKS = [
    check_phi_library, check_pool_by_hand, check_selection_golden, check_selection_bruteforce,
    check_selection_ties_constructed, check_selection_output_form, check_attention_golden,
    check_attention_dense_equivalence, check_attention_subset_library,
    check_attention_identical_keys, check_absorb_readout_golden,
    check_absorb_incremental_equals_batch, check_absorb_single_token,
    check_readout_closed_forms, check_hybrid_sum, check_two_stage_golden,
    check_two_stage_all_frames_is_one_stage, check_two_stage_frames_are_blocks,
    check_two_stage_bruteforce, check_schedule_golden, check_schedule_budget_and_rounding,
    check_schedule_two_chunks, check_schedule_noise_scale, check_schedule_rejects,
    check_rope_positions_golden, check_rope_rotation_closed_form, check_rope_complex_form,
    check_rope_norm_inverse_relative, check_rope_cap_and_identity,
]
