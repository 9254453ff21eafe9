"""fp64 CPU oracle of the hybrid attention chunk step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA path and imports nothing
from the package.

Every function is a plain, literal statement of the definition it cites, in
float64 numpy, on inputs that the caller widens exactly from bf16. A library
matmul is used as a step where the definition is a matrix product; there is no
blocking, fusion or reordering beyond what the definitions state.

Sources (page title, then the section used):
  [HF-de]  "Long-Horizon Streaming Video Generation via Hybrid Attention with
           Decoupled Distillation", German technical summary (gist.science),
           §2 Methodik, A. Hybride Aufmerksamkeitsmechanismen.
  [HF-abs] the same title, English abstract (arxivdaily.com).
  [HF-pt]  the same title, Portuguese technical summary (gist.science),
           §2 Metodologia, A. Mecanismo de Atenção Híbrida.
  [LF]     "Light Forcing: Accelerating Autoregressive Video Diffusion via
           Sparse Attention", German technical summary (gist.science),
           §2.2 Hierarchische Spärliche Attention (token compression by mean
           pooling at block and frame level; per-query-block selection; the
           two-stage mask selection: frames first by frame-level compressed keys,
           then blocks within the selected frames); §2.1 Chunk-bewusstes
           Wachstum (dense first chunk, sparsity s_i = s_base - alpha_i beta for
           the later chunks, beta set by a FLOP budget).
  [HF-de] §2 C and [HF-pt] §2 B.2 (relative RoPE: the largest temporal RoPE
           index is capped, in training and inference alike, and positions are
           expressed as relative offsets).

The pages give the structure (a compact KV state absorbing evicted tokens
through a linear attention function; Top-K block-sparse attention inside the
window; output = sum of both) but no formulas. The step's specification fixes
the open parts, and this oracle follows them:
  * phi(x) = elu(x) + 1, i.e. x + 1 for x > 0 and exp(x) otherwise;
  * flat key/query blocks of ``block`` tokens over the flattened sequence, the
    last block possibly partial;
  * pooled block score s_IJ = mean(q in I) . mean(k in J), unscaled;
  * each query block keeps its top-r key blocks, ties to the lower index,
    emitted in ascending order;
  * sparse softmax attention over the valid tokens of the kept blocks with
    scale 1/sqrt(d), no causal mask inside the window;
  * linear readout phi(q) S / (phi(q) . z + 1e-6);
  * state update S += phi(K)^T V, z += sum_t phi(k_t).

Parity pins: each function is checked in ``tests/test_oracle_pins.py`` against
closed forms, brute force, library routines and hand-derived fixtures; none is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

READOUT_EPS = 1e-6

__all__ = [
    "READOUT_EPS", "phi", "block_ranges", "pool_blocks", "block_scores",
    "select_blocks", "frame_ranges", "pool_frames", "frame_scores", "candidate_blocks",
    "select_blocks_two_stage", "sparse_attention_tile", "sparse_attention", "linear_readout",
    "hybrid_attention", "hybrid_attention_tile", "absorb", "absorb_batch",
    "dense_swa", "default_scale", "keep_schedule", "ROPE_BASE", "rope_positions", "rope_rotate", "rope_qk",
    "select_blocks_rope", "hybrid_attention_rope", "hybrid_attention_rope_tile",
]


def _f64(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    return a


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(d) (textbook attention; the pages give none)."""
    return 1.0 / math.sqrt(d)


def phi(x) -> np.ndarray:
    """Feature map of the linear temporal attention: elu(x) + 1.

    elu(x) = x for x > 0 and exp(x) - 1 otherwise, so phi(x) = x + 1 (x > 0),
    exp(x) (x <= 0); phi > 0 everywhere. [HF-de] §2A (linear attention function);
    the map itself is the specification's choice.
    """
    x = _f64(x)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def block_ranges(n: int, block: int) -> list[tuple[int, int]]:
    """Token ranges [t*block, min((t+1)*block, n)) of the ceil(n/block) blocks."""
    return [(t * block, min((t + 1) * block, n)) for t in range(-(-n // block))]


def pool_blocks(X, block: int) -> np.ndarray:
    """Mean of the valid tokens of every block: [B,H,N,d] -> [B,H,ceil(N/block),d].

    [LF] §2.2: query and key tokens are compressed by mean pooling at block level.
    """
    X = _f64(X)
    B, H, N, d = X.shape
    out = np.empty((B, H, -(-N // block), d), dtype=np.float64)
    for t, (lo, hi) in enumerate(block_ranges(N, block)):
        out[:, :, t, :] = X[:, :, lo:hi, :].mean(axis=2)
    return out


def block_scores(Q, K, block: int) -> np.ndarray:
    """s[b,h,I,J] = pooled(Q)[I] . pooled(K)[J] (unscaled), [B,H,nQB,nKB]."""
    Qp = pool_blocks(Q, block)
    Kp = pool_blocks(K, block)
    return Qp @ np.swapaxes(Kp, -1, -2)


def select_blocks(Q, K, block: int, r: int):
    """Top-r key blocks of every query block.

    For each (b, h, I), the key blocks J are ordered by decreasing s_IJ, equal
    scores by increasing J; the first r are kept and returned in ascending J.
    [HF-de] §2A (only the most important, Top-K, blocks are computed);
    [LF] §2.2 (selection per query block from pooled scores).

    Returns (idx int32 [B,H,nQB,r], scores float64 [B,H,nQB,nKB]).
    """
    s = block_scores(Q, K, block)
    B, H, nQB, nKB = s.shape
    if not 1 <= r <= nKB:
        raise ValueError(f"r={r} outside [1, {nKB}]")
    idx = np.empty((B, H, nQB, r), dtype=np.int32)
    order_key = np.arange(nKB)
    for b in range(B):
        for h in range(H):
            for I in range(nQB):
                # lexsort sorts by the last key first: -s descending score, then J.
                order = np.lexsort((order_key, -s[b, h, I]))
                idx[b, h, I] = np.sort(order[:r])
    return idx, s


def frame_ranges(n: int, tokens_per_frame: int) -> list[tuple[int, int]]:
    """Token ranges [w*T, min((w+1)*T, n)) of the ceil(n/T) frames of a window."""
    return block_ranges(n, tokens_per_frame)


def pool_frames(K, tokens_per_frame: int) -> np.ndarray:
    """Mean of the valid tokens of every frame: [B,H,N,d] -> [B,H,ceil(N/T),d].

    [LF] §2.2: key tokens are also compressed by mean pooling at frame level.
    """
    return pool_blocks(K, tokens_per_frame)


def frame_scores(Q, K, block: int, tokens_per_frame: int) -> np.ndarray:
    """f[b,h,I,w] = pooled(Q, blocks)[I] . pooled(K, frames)[w] (unscaled), [B,H,nQB,W]."""
    Qp = pool_blocks(Q, block)
    Kf = pool_frames(K, tokens_per_frame)
    return Qp @ np.swapaxes(Kf, -1, -2)


def candidate_blocks(kept_frames, Nk: int, block: int, tokens_per_frame: int) -> np.ndarray:
    """Key blocks whose token range intersects the token range of a kept frame (sorted)."""
    frames = frame_ranges(Nk, tokens_per_frame)
    out = []
    for J, (lo, hi) in enumerate(block_ranges(Nk, block)):
        if any(lo < frames[int(w)][1] and frames[int(w)][0] < hi for w in kept_frames):
            out.append(J)
    return np.asarray(out, dtype=np.int64)


def select_blocks_two_stage(Q, K, block: int, r: int, tokens_per_frame: int, n_frames: int):
    """Two-stage (frame, then block) top-r selection for every query block.

    [LF] §2.2, "Zweistufige Maskenauswahl": for each query block the frames are
    ranked by the frame-level compressed keys and a small set is kept; the blocks
    within the kept frames are then ranked by the block-level compressed keys.
    Readings: the n_frames frames of largest f_Iw are kept (equal scores: lower w
    first); a key block lies within the kept frames when any of its tokens does; of
    those candidate blocks the r of largest s_IJ are kept (equal scores: lower J
    first) and returned in ascending J. Should fewer than r blocks touch the kept
    frames (a short last frame), every candidate is kept and the remaining places go
    to the best other blocks in the same order.

    Returns (idx int32 [B,H,nQB,r], frames int32 [B,H,nQB,n_frames] ascending,
    block scores float64 [B,H,nQB,nKB], frame scores float64 [B,H,nQB,W]).
    """
    s = block_scores(Q, K, block)
    f = frame_scores(Q, K, block, tokens_per_frame)
    B, H, nQB, nKB = s.shape
    W = f.shape[-1]
    Nk = np.asarray(K).shape[2]
    if not 1 <= n_frames <= W:
        raise ValueError(f"n_frames={n_frames} outside [1, {W}]")
    if not 1 <= r <= nKB:
        raise ValueError(f"r={r} outside [1, {nKB}]")
    idx = np.empty((B, H, nQB, r), dtype=np.int32)
    frames = np.empty((B, H, nQB, n_frames), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for I in range(nQB):
                order = np.lexsort((np.arange(W), -f[b, h, I]))
                kept = np.sort(order[:n_frames])
                frames[b, h, I] = kept
                cand = candidate_blocks(kept, Nk, block, tokens_per_frame)
                is_cand = np.zeros(nKB, dtype=bool)
                is_cand[cand] = True
                # candidates first, then by decreasing score, then by increasing J
                order = np.lexsort((np.arange(nKB), -s[b, h, I], ~is_cand))
                idx[b, h, I] = np.sort(order[:r])
    return idx, frames, s, f


def _selected_tokens(kept_blocks, Nk: int, block: int) -> np.ndarray:
    ranges = block_ranges(Nk, block)
    return np.concatenate([np.arange(*ranges[int(J)]) for J in kept_blocks])


def sparse_attention_tile(Q, K, V, idx, block: int, b: int, h: int, I: int,
                          scale: float | None = None) -> np.ndarray:
    """Softmax attention of query block I over the valid tokens of its kept blocks.

    O_i = sum_j softmax_j(scale * q_i . k_j) v_j, j over the tokens of the key
    blocks idx[b,h,I]; exact softmax (max-subtracted), not an online one.
    [HF-de] §2A (block-sparse attention inside the local window);
    [HF-pt] §2A.2.
    Returns [L_I, d] float64.
    """
    Q = np.asarray(Q)
    K = np.asarray(K)
    V = np.asarray(V)
    d = Q.shape[-1]
    scale = default_scale(d) if scale is None else float(scale)
    lo, hi = block_ranges(Q.shape[2], block)[I]
    q = _f64(Q[b, h, lo:hi])
    toks = _selected_tokens(idx[b, h, I], K.shape[2], block)
    k = _f64(K[b, h, toks])
    v = _f64(V[b, h, toks])
    a = scale * (q @ k.T)
    m = a.max(axis=1, keepdims=True)
    p = np.exp(a - m)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def sparse_attention(Q, K, V, idx, block: int, scale: float | None = None) -> np.ndarray:
    """Sparse term O_s for all query blocks, [B,H,Nq,d] float64."""
    B, H, Nq, d = np.shape(Q)
    out = np.empty((B, H, Nq, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for I, (lo, hi) in enumerate(block_ranges(Nq, block)):
                out[b, h, lo:hi] = sparse_attention_tile(Q, K, V, idx, block, b, h, I, scale)
    return out


def linear_readout(Q, S, z) -> np.ndarray:
    """Linear term O_lin = phi(q)^T S / (phi(q) . z + 1e-6).

    Q [..., N, d], S [..., d, d] (S[k, n] = sum_t phi(k_t)[k] v_t[n]), z [..., d].
    [HF-de] §2A and [HF-abs] (compact key-value state read by linear attention);
    the normalised form with 1e-6 is the specification's.
    """
    ph = phi(Q)
    S = _f64(S)
    z = _f64(z)
    num = ph @ S
    den = (ph @ z[..., :, None]) + READOUT_EPS
    return num / den


def hybrid_attention_tile(Q, K, V, idx, S, z, block: int, b: int, h: int, I: int,
                          scale: float | None = None) -> np.ndarray:
    """Output rows of query block I: O = O_s + O_lin ([HF-de] §2A Kombination; [HF-pt] §2A)."""
    lo, hi = block_ranges(np.shape(Q)[2], block)[I]
    o_s = sparse_attention_tile(Q, K, V, idx, block, b, h, I, scale)
    o_l = linear_readout(np.asarray(Q)[b, h, lo:hi], np.asarray(S)[b, h], np.asarray(z)[b, h])
    return o_s + o_l


def hybrid_attention(Q, K, V, idx, S, z, block: int, scale: float | None = None) -> np.ndarray:
    """O = sparse term + linear term for every query, [B,H,Nq,d] float64."""
    return sparse_attention(Q, K, V, idx, block, scale) + linear_readout(Q, S, z)


def absorb(S, z, K_ev, V_ev):
    """State after absorbing evicted tokens: S + phi(K)^T V, z + sum_t phi(k_t).

    S [B,H,d,d], z [B,H,d], K_ev/V_ev [B,H,Ne,d]. [HF-de] §2A (evicted frames are
    aggregated into the compact state by a linear attention function);
    [HF-abs] (incremental absorption of evicted tokens); [HF-pt] §2A.1.
    Returns new (S, z); the inputs are not modified.
    """
    pk = phi(K_ev)
    v = _f64(V_ev)
    return _f64(S) + np.swapaxes(pk, -1, -2) @ v, _f64(z) + pk.sum(axis=-2)


def absorb_batch(K_ev, V_ev):
    """State built in one go from an empty state (S = 0, z = 0)."""
    B, H, _, d = np.shape(K_ev)
    return absorb(np.zeros((B, H, d, d)), np.zeros((B, H, d)), K_ev, V_ev)


def dense_swa(Q, K, V, scale: float | None = None) -> np.ndarray:
    """Dense sliding-window attention: softmax(scale * Q K^T) V over all window keys.

    [HF-de] §1 (SWA with KV caching), the dense case the block-sparse form replaces.
    """
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    scale = default_scale(Q.shape[-1]) if scale is None else float(scale)
    a = scale * (Q @ np.swapaxes(K, -1, -2))
    a = a - a.max(axis=-1, keepdims=True)
    p = np.exp(a)
    return (p @ V) / p.sum(axis=-1, keepdims=True)


def keep_schedule(nKB, s_base: float, s_target: float):
    """Chunk-aware growth: the sparsity of every chunk of a video and its kept key blocks.

    [LF] §2.1: the first chunk attends densely; a later chunk i gets the sparsity ratio
    s_i = s_base - alpha_i * beta, where alpha_i follows the noise scale 1/sqrt(T) and beta
    is set so that the FLOPs of all chunks meet a target sparsity ratio, so that earlier
    chunks keep more and later ones less.
    Readings (the page gives no constants): T is the chunk's position i >= 1, so
    alpha_i = 1/sqrt(i); a chunk's dense attention FLOPs are proportional to the key blocks of
    its window, nKB[i] (every chunk has the same queries); the budget is
        sum_i (1 - s_i) nKB[i] = (1 - s_target) sum_i nKB[i];
    chunk i keeps r_i = clamp(ceil((1 - s_i) nKB[i]), 1, nKB[i]) blocks. A single chunk is
    dense whatever the target. A schedule whose beta would be negative (sparsity falling
    with i) or whose s_i would leave [0, 1) is rejected with ValueError.
    Returns (r int64 [n], s float64 [n], beta).
    """
    nKB = [int(x) for x in nKB]
    n = len(nKB)
    if n < 1 or min(nKB) < 1:
        raise ValueError("every chunk needs at least one key block")
    if not (0.0 <= s_base < 1.0 and 0.0 <= s_target < 1.0):
        raise ValueError("sparsity ratios lie in [0, 1)")
    s = np.zeros(n)
    beta = 0.0
    if n > 1:
        alpha = np.array([1.0 / math.sqrt(i) for i in range(1, n)])
        later = np.array(nKB[1:], dtype=np.float64)
        # nKB[0] + sum_{i>=1} (1 - s_base + alpha_i beta) nKB[i] = (1 - s_target) sum_i nKB[i]
        budget = (1.0 - s_target) * float(sum(nKB))
        beta = (budget - nKB[0] - (1.0 - s_base) * later.sum()) / float((alpha * later).sum())
        if beta < 0.0:
            raise ValueError("the budget needs sparsity falling with the chunk index (beta < 0)")
        s[1:] = s_base - alpha * beta
        if np.any(s < 0.0) or np.any(s >= 1.0):
            raise ValueError("a chunk's sparsity leaves [0, 1)")
    r = np.array([min(max(math.ceil((1.0 - s[i]) * nKB[i]), 1), nKB[i]) for i in range(n)], dtype=np.int64)
    return r, s, beta


# ---------------------------------------------------------------------------
# capped relative temporal RoPE ([HF-de] §2 C; [HF-pt] §2 B.2)
# ---------------------------------------------------------------------------
# Readings (the pages name the technique and nothing else): the temporal part of a
# rotary embedding acts on the first d_t dimensions of a head, as consecutive pairs
# (2i, 2i+1) turned by the angle p * base**(-2i/d_t) (the textbook RoPE frequencies,
# base 10000); the spatial parts of a video RoPE do not depend on time and are left to
# the model. A token's temporal index p counts from its frame's offset to the newest
# frame of the window, delta, capped at P: p = P - min(delta, P), so the newest frame
# sits at P and every frame P or more frames old at 0 (the index never exceeds P
# however long the video). The rotation applies to q and k of the softmax branch, and
# so to the tokens the block selection pools; the linear branch reads the raw q and k
# (evicted frames are older than the window, i.e. at index 0 where the rotation is the
# identity once P does not exceed the window).
ROPE_BASE = 10000.0


def rope_positions(n_tokens: int, tokens_per_frame: int, frame0: int, n_frames: int, cap: int) -> np.ndarray:
    """Temporal index of each of n_tokens consecutive tokens whose first token lies in
    window frame frame0 (frames of tokens_per_frame tokens; the window holds n_frames
    frames, the newest being n_frames - 1): p = cap - min(delta, cap) with
    delta = (n_frames - 1) - frame. int64 [n_tokens]."""
    p = np.empty(n_tokens, dtype=np.int64)
    for t in range(n_tokens):
        frame = frame0 + t // tokens_per_frame
        delta = (n_frames - 1) - frame
        p[t] = cap - min(delta, cap)
    return p


def rope_rotate(X, positions, d_t: int, base: float = ROPE_BASE) -> np.ndarray:
    """X [..., N, d] with the pairs (2i, 2i+1), i < d_t/2, of token n turned by the angle
    positions[n] * base**(-2i/d_t); the other dimensions unchanged."""
    X = _f64(X).copy()
    pos = np.asarray(positions, dtype=np.float64)
    for i in range(d_t // 2):
        ang = pos * base ** (-2.0 * i / d_t)
        c, s = np.cos(ang), np.sin(ang)
        a = X[..., 2 * i].copy()
        b = X[..., 2 * i + 1].copy()
        X[..., 2 * i] = a * c - b * s
        X[..., 2 * i + 1] = a * s + b * c
    return X


def rope_qk(Q, K, rope: dict):
    """Q and K of a chunk step turned by their temporal indices. rope: d_t,
    tokens_per_frame, cap, q_frame0 (window frame of Q's first token), base. K is the
    window (its first token starts frame 0); the window holds ceil(Nk / tokens_per_frame)
    frames."""
    T = int(rope["tokens_per_frame"])
    Nq, Nk = np.shape(Q)[2], np.shape(K)[2]
    W = -(-Nk // T)
    base = float(rope.get("base", ROPE_BASE))
    pq = rope_positions(Nq, T, int(rope["q_frame0"]), W, int(rope["cap"]))
    pk = rope_positions(Nk, T, 0, W, int(rope["cap"]))
    return rope_rotate(Q, pq, int(rope["d_t"]), base), rope_rotate(K, pk, int(rope["d_t"]), base)


def select_blocks_rope(Q, K, block: int, r: int, rope: dict):
    """select_blocks on the turned Q and K (the selection pools the tokens the softmax
    branch attends with)."""
    Qr, Kr = rope_qk(Q, K, rope)
    return select_blocks(Qr, Kr, block, r)


def hybrid_attention_rope(Q, K, V, idx, S, z, block: int, rope: dict, scale: float | None = None) -> np.ndarray:
    """Sparse term on the turned Q and K plus the linear term on the raw Q."""
    Qr, Kr = rope_qk(Q, K, rope)
    return sparse_attention(Qr, Kr, V, idx, block, scale) + linear_readout(Q, S, z)


def hybrid_attention_rope_tile(Q, K, V, idx, S, z, block: int, rope: dict, b: int, h: int, I: int,
                               scale: float | None = None) -> np.ndarray:
    """Output rows of query block I of hybrid_attention_rope."""
    Qr, Kr = rope_qk(np.asarray(Q)[b:b + 1, h:h + 1], np.asarray(K)[b:b + 1, h:h + 1], rope)
    lo, hi = block_ranges(np.shape(Q)[2], block)[I]
    o_s = sparse_attention_tile(Qr, Kr, np.asarray(V)[b:b + 1, h:h + 1], np.asarray(idx)[b:b + 1, h:h + 1],
                                block, 0, 0, I, scale)
    o_l = linear_readout(np.asarray(Q)[b, h, lo:hi], np.asarray(S)[b, h], np.asarray(z)[b, h])
    return o_s + o_l
