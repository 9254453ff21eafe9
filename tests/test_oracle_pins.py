"""The fp64 oracle against its pins, and planted mistakes against the pins.

CPU only. A planted mistake lives in a private copy of the oracle module loaded
for the test; the real oracle is never modified.
"""
import importlib.util
import os

import numpy as np
import pytest

import oracle
import oracle.hf_oracle as real_oracle
from tests import oracle_pins as pins

ORACLE_PATH = os.path.abspath(real_oracle.__file__)


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(real_oracle)


def _fresh_copy(name):
    spec = importlib.util.spec_from_file_location(f"_oracle_mutant_{name}", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_phi_no_plus_one(m):
    m.phi = lambda x: np.where(np.asarray(x) > 0, np.asarray(x, float), np.exp(np.minimum(x, 0.0)))


def _mut_phi_exp(m):
    m.phi = lambda x: np.exp(np.asarray(x, float))


def _mut_readout_no_eps(m):
    def f(Q, S, z):
        ph = m.phi(Q)
        return (ph @ np.asarray(S, float)) / (ph @ np.asarray(z, float)[..., :, None])
    m.linear_readout = f


def _mut_readout_transposed(m):
    def f(Q, S, z):
        ph = m.phi(Q)
        return (ph @ np.swapaxes(np.asarray(S, float), -1, -2)) / (ph @ np.asarray(z, float)[..., :, None] + 1e-6)
    m.linear_readout = f


def _mut_readout_no_phi_q(m):
    def f(Q, S, z):
        q = np.asarray(Q, float)
        return (q @ np.asarray(S, float)) / (q @ np.asarray(z, float)[..., :, None] + 1e-6)
    m.linear_readout = f


def _mut_select_ties_high(m):
    orig_lexsort = np.lexsort

    class _NP:
        def __getattr__(self, k):
            return getattr(np, k)

        @staticmethod
        def lexsort(keys):
            a, b = keys
            return orig_lexsort((-a, b))
    m.np = _NP()


def _mut_select_bottom(m):
    orig = m.block_scores
    m.block_scores = lambda Q, K, block: -orig(Q, K, block)


def _mut_pool_sum(m):
    def f(X, block):
        X = np.asarray(X, float)
        B, H, N, d = X.shape
        out = np.empty((B, H, -(-N // block), d))
        for t, (lo, hi) in enumerate(m.block_ranges(N, block)):
            out[:, :, t] = X[:, :, lo:hi].sum(axis=2)
        return out
    m.pool_blocks = f


def _mut_attention_no_scale(m):
    m.default_scale = lambda d: 1.0


def _mut_attention_sqrt_d(m):
    m.default_scale = lambda d: float(np.sqrt(d))


def _mut_attention_all_keys(m):
    m._selected_tokens = lambda kept, Nk, block: np.arange(Nk)


def _mut_absorb_transposed(m):
    def f(S, z, K_ev, V_ev):
        pk = m.phi(K_ev)
        v = np.asarray(V_ev, float)
        return np.asarray(S, float) + np.swapaxes(v, -1, -2) @ pk, np.asarray(z, float) + pk.sum(axis=-2)
    m.absorb = f


def _mut_absorb_z_raw(m):
    def f(S, z, K_ev, V_ev):
        pk = m.phi(K_ev)
        v = np.asarray(V_ev, float)
        return (np.asarray(S, float) + np.swapaxes(pk, -1, -2) @ v,
                np.asarray(z, float) + np.asarray(K_ev, float).sum(axis=-2))
    m.absorb = f


def _mut_hybrid_difference(m):
    def f(Q, K, V, idx, S, z, block, scale=None):
        return m.sparse_attention(Q, K, V, idx, block, scale) - m.linear_readout(Q, S, z)
    m.hybrid_attention = f


def _mut_two_stage_inside_only(m):
    def f(kept_frames, Nk, block, tokens_per_frame):
        frames = m.frame_ranges(Nk, tokens_per_frame)
        return np.asarray([J for J, (lo, hi) in enumerate(m.block_ranges(Nk, block))
                           if any(frames[int(w)][0] <= lo and hi <= frames[int(w)][1] for w in kept_frames)],
                          dtype=np.int64)
    m.candidate_blocks = f


def _mut_two_stage_ignore_frames(m):
    m.candidate_blocks = lambda kept, Nk, block, T: np.arange(-(-Nk // block))


def _mut_pool_frames_sum(m):
    def f(K, T):
        K = np.asarray(K, float)
        B, H, N, d = K.shape
        return np.stack([K[:, :, lo:hi].sum(axis=2) for lo, hi in m.frame_ranges(N, T)], axis=2)
    m.pool_frames = f


def _mut_two_stage_frame_ties_high(m):
    def f(Q, K, block, r, T, n_frames):
        # frame ranking with equal scores broken towards the higher frame index
        fs = m.frame_scores(Q, K, block, T)
        s = m.block_scores(Q, K, block)
        B, H, nQB, nKB = s.shape
        W = fs.shape[-1]
        idx = np.empty((B, H, nQB, r), dtype=np.int32)
        frames = np.empty((B, H, nQB, n_frames), dtype=np.int32)
        for b in range(B):
            for h in range(H):
                for I in range(nQB):
                    kept = np.sort(np.lexsort((-np.arange(W), -fs[b, h, I]))[:n_frames])
                    frames[b, h, I] = kept
                    is_cand = np.zeros(nKB, dtype=bool)
                    is_cand[m.candidate_blocks(kept, np.asarray(K).shape[2], block, T)] = True
                    idx[b, h, I] = np.sort(np.lexsort((np.arange(nKB), -s[b, h, I], ~is_cand))[:r])
        return idx, frames, s, fs
    m.select_blocks_two_stage = f


def _mut_two_stage_no_fill(m):
    orig = m.select_blocks_two_stage

    def f(Q, K, block, r, T, n_frames):
        idx, frames, s, fs = orig(Q, K, block, r, T, n_frames)
        Nk = np.asarray(K).shape[2]
        for b, h, I in np.ndindex(*idx.shape[:3]):
            cand = set(m.candidate_blocks(frames[b, h, I], Nk, block, T).tolist())
            keep = [J for J in idx[b, h, I].tolist() if J in cand]
            idx[b, h, I] = np.asarray((keep + [keep[-1]] * r)[:r])  # short lists padded
        return idx, frames, s, fs
    m.select_blocks_two_stage = f


def _mut_schedule_alpha_linear(m):
    # alpha_i = 1/i instead of 1/sqrt(i)
    import math as math_mod

    class _Math:
        def __getattr__(self, k):
            return getattr(math_mod, k)

        @staticmethod
        def sqrt(x):
            return float(x) if x >= 1 else math_mod.sqrt(x)
    m.math = _Math()


def _mut_schedule_first_chunk_sparse(m):
    orig = m.keep_schedule

    def f(nKB, s_base, s_target):
        r, s, beta = orig(nKB, s_base, s_target)
        s = s.copy()
        s[0] = s_base - beta  # the formula applied to the first chunk too
        r = r.copy()
        r[0] = max(1, int(np.ceil((1.0 - s[0]) * nKB[0])))
        return r, s, beta
    m.keep_schedule = f


def _mut_schedule_floor(m):
    orig = m.keep_schedule

    def f(nKB, s_base, s_target):
        r, s, beta = orig(nKB, s_base, s_target)
        r = np.array([min(max(int(np.floor((1.0 - s[i]) * nKB[i])), 1), nKB[i]) for i in range(len(nKB))])
        return r, s, beta
    m.keep_schedule = f


def _mut_schedule_budget_on_chunks(m):
    # the target read as a per-chunk sparsity for the later chunks only (dense chunk not counted)
    orig = m.keep_schedule

    def f(nKB, s_base, s_target):
        total = float(sum(nKB))
        t2 = 1.0 - (1.0 - s_target) * (total - nKB[0]) / total if len(nKB) > 1 else s_target
        return orig(nKB, s_base, t2)
    m.keep_schedule = f


def _mut_rope_sign(m):
    orig = m.rope_rotate
    m.rope_rotate = lambda X, positions, d_t, base=m.ROPE_BASE: orig(X, -np.asarray(positions), d_t, base)


def _mut_rope_half_pairs(m):
    def f(X, positions, d_t, base=m.ROPE_BASE):
        X = np.asarray(X, dtype=np.float64).copy()
        pos = np.asarray(positions, dtype=np.float64)
        h = d_t // 2
        for i in range(h):
            ang = pos * base ** (-2.0 * i / d_t)
            a, b = X[..., i].copy(), X[..., i + h].copy()
            X[..., i] = a * np.cos(ang) - b * np.sin(ang)
            X[..., i + h] = a * np.sin(ang) + b * np.cos(ang)
        return X
    m.rope_rotate = f


def _mut_rope_uncapped(m):
    def f(n_tokens, tokens_per_frame, frame0, n_frames, cap):
        return np.array([frame0 + t // tokens_per_frame for t in range(n_tokens)], dtype=np.int64)
    m.rope_positions = f


def _mut_rope_frequency(m):
    orig = m.rope_rotate

    def f(X, positions, d_t, base=m.ROPE_BASE):
        return orig(X, positions, 2 * d_t, base) if d_t else orig(X, positions, d_t, base)
    m.rope_rotate = f


def _mut_rope_turned_readout(m):
    def f(Q, K, V, idx, S, z, block, rope, scale=None):
        Qr, Kr = m.rope_qk(Q, K, rope)
        return m.sparse_attention(Qr, Kr, V, idx, block, scale) + m.linear_readout(Qr, S, z)
    m.hybrid_attention_rope = f


def _mut_rope_query_frames(m):
    orig = m.rope_qk
    m.rope_qk = lambda Q, K, rope: orig(Q, K, dict(rope, q_frame0=0))


MUTANTS = [
    _mut_phi_no_plus_one, _mut_phi_exp, _mut_readout_no_eps, _mut_readout_transposed,
    _mut_readout_no_phi_q, _mut_select_ties_high, _mut_select_bottom, _mut_pool_sum,
    _mut_attention_no_scale, _mut_attention_sqrt_d, _mut_attention_all_keys,
    _mut_absorb_transposed, _mut_absorb_z_raw, _mut_hybrid_difference, _mut_two_stage_inside_only,
    _mut_two_stage_ignore_frames, _mut_pool_frames_sum, _mut_two_stage_frame_ties_high, _mut_two_stage_no_fill,
    _mut_schedule_alpha_linear, _mut_schedule_first_chunk_sparse, _mut_schedule_floor,
    _mut_schedule_budget_on_chunks, _mut_rope_sign, _mut_rope_half_pairs, _mut_rope_uncapped,
    _mut_rope_frequency, _mut_rope_turned_readout, _mut_rope_query_frames,
]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__[5:])
def test_planted_mistake_is_caught(mutate):
    m = _fresh_copy(mutate.__name__)
    mutate(m)
    failures = []
    for check in pins.ALL_CHECKS:
        try:
            check(m)
        except (AssertionError, ValueError, IndexError):
            failures.append(check.__name__)
    assert failures, f"no pin caught the planted mistake {mutate.__name__}"


def test_oracle_package_exports():
    for name in oracle.__all__:
        assert hasattr(oracle, name)
