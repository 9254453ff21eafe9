/*
 * hf.h - C ABI of the hybrid attention chunk step (B200, sm_100a).
 *
 * The step is the attention of "Hybrid Forcing": for each new chunk of query tokens
 * the output is the SUM of
 *   (1) block-sparse softmax attention over the local sliding window of cached
 *       frames, restricted to the top-r key blocks of every query block, and
 *   (2) a linear-attention readout of a compact key-value state (S, z) that has
 *       absorbed the tokens of every frame evicted from the window.
 * Sources: "Long-Horizon Streaming Video Generation via Hybrid Attention with
 * Decoupled Distillation" - German technical summary, section 2 A (linear temporal
 * attention over a compact KV state; Top-K block-sparse SWA; output = sum), English
 * abstract (state absorbs evicted tokens incrementally), Portuguese technical summary
 * section 2 A.1/A.2; "Light Forcing: Accelerating Autoregressive Video Diffusion via
 * Sparse Attention" - German technical summary, section 2.2 (mean-pooled block
 * scores, selection per query block).
 *
 * Fixed readings of the open details:
 *   phi(x) = elu(x) + 1 evaluated in fp32;
 *   blocks are `block` consecutive tokens of the flattened sequence, the last block of
 *   a sequence may be partial (its padding is excluded from pooling and masked);
 *   score(I, J) = mean(q in I) . mean(k in J), unscaled, fp32;
 *   each query block keeps the r best key blocks, ties to the lower index, listed in
 *   ascending order;
 *   sparse term: softmax(scale * q.k) over the valid tokens of the kept blocks,
 *   scale = 1/sqrt(d) unless given, no causal mask inside the window;
 *   linear term: phi(q)^T S / (phi(q) . z + 1e-6);
 *   state update: S += phi(K)^T V, z += sum_t phi(k_t).
 *
 * Conventions for every call
 *   - Tensors are dense row-major [B][H][N][d] (d innermost), bf16 unless stated.
 *   - Every pointer is a DEVICE pointer of the current CUDA device unless stated, and
 *     must be 16-byte aligned (TMA requirement).
 *   - Supported: d in {64, 128}; block in {32, 64, 128}; 1 <= r <= nKB.
 *   - The caller owns every buffer, including workspaces (size from
 *     hf_workspace_size). The library allocates no device memory. Its only state is
 *     one 32-bit device error word per GPU, read by hf_query_status, and the fixed
 *     scratch array of hf_select_blocks_noalloc.
 *   - All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Argument errors are returned before anything is launched; a failed
 *     launch returns HF_ERR_CUDA. A kernel that gives up on an internal wait (bounded,
 *     about one second) records HF_ERR_DEVICE_TIMEOUT in the device error word
 *     instead of hanging; hf_query_status reports it.
 *   - Calls on one stream are ordered; calls whose buffers overlap must not run
 *     concurrently on different streams. Kernels are launched with programmatic
 *     stream serialisation: a kernel may be scheduled while the previous kernel of its
 *     stream finishes its last CTAs, and waits for it on the device before reading
 *     anything; stream order is kept for every caller-visible buffer.
 */
#ifndef HF_H_
#define HF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HF_API __attribute__((visibility("default")))
#else
#define HF_API
#endif

/* bfloat16 bit pattern (1 sign, 8 exponent, 7 mantissa bits). */
typedef uint16_t hf_bf16;

typedef enum hf_status {
  HF_OK = 0,
  HF_ERR_INVALID_ARG = 1,     /* null pointer, bad size, r outside [1, nKB], ...      */
  HF_ERR_UNSUPPORTED = 2,     /* d or block outside the supported set                 */
  HF_ERR_ALIGNMENT = 3,       /* a pointer is not 16-byte aligned                     */
  HF_ERR_WORKSPACE = 4,       /* workspace missing or smaller than hf_workspace_size  */
  HF_ERR_CUDA = 5,            /* a CUDA runtime/driver call or a launch failed        */
  HF_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up on an internal wait (device word)   */
  HF_ERR_DEVICE_BAD_INDEX = 7 /* hf_hybrid_attn_fwd met a block index outside [0,nKB) */
} hf_status;

/* Compact key-value state of the linear temporal attention, one per (b, h):
 *   S[b][h][k][n] = sum over absorbed tokens t of phi(k_t)[k] * v_t[n]   (fp32, d x d)
 *   z[b][h][k]    = sum over absorbed tokens t of phi(k_t)[k]           (fp32, d)
 * S and z are caller-owned device buffers of B*H*d*d and B*H*d floats. S_split is a
 * caller-owned device buffer of HF_STATE_SPLIT_BYTES(B, H, d) bytes (16-byte aligned)
 * that the library keeps equal to S split into two bf16 terms, hi = bf16(S) and
 * lo = bf16(S - hi) (round to nearest even), in the layout the hybrid attention's
 * readout MMAs read: per (b, h) the hi tile, then the lo tile, each d/64 chunks of 64
 * columns n, a chunk d rows k of 128 bytes, the 16-byte group g of row k stored at
 * position g ^ (k % 8). It changes with S (hf_state_init, hf_absorb_evicted and the fused
 * calls); a caller that writes S itself leaves it stale. n_absorbed is a host-side count
 * of tokens absorbed per head (bookkeeping only; the kernels do not read it). The state's
 * size does not depend on how many tokens it has absorbed. */
typedef struct hf_state {
  int B, H, d;
  float* S;
  float* z;
  void* S_split;
  long long n_absorbed;
} hf_state;

/* Bytes of a state's S_split buffer: two bf16 d x d tiles per (b, h). */
#define HF_STATE_SPLIT_BYTES(B, H, d) ((size_t)(B) * (size_t)(H) * 4u * (size_t)(d) * (size_t)(d))

/* Workspace kinds for hf_workspace_size. */
enum { HF_WS_SELECT = 1, HF_WS_ATTN = 2, HF_WS_ABSORB = 3, HF_WS_SELECT_TWO_STAGE = 4 };

/* Bytes of device workspace the call `which` needs (0 = none; NULL may be passed).
 * For HF_WS_ABSORB pass the number of evicted tokens as Nk (Nq, block, r ignored).
 * Returns (size_t)-1 for arguments the call would reject. Host-only, no CUDA call. */
HF_API size_t hf_workspace_size(int which, int B, int H, int Nq, int Nk, int d, int block, int r);

/* Bind S_dev / z_dev / S_split_dev to *st and zero them (stream-ordered memsets): the
 * empty state. Errors: HF_ERR_INVALID_ARG (st/S_dev/z_dev/S_split_dev NULL, B/H < 1),
 * HF_ERR_UNSUPPORTED (d), HF_ERR_ALIGNMENT, HF_ERR_CUDA. */
HF_API hf_status hf_state_init(hf_state* st, int B, int H, int d, float* S_dev, float* z_dev, void* S_split_dev,
                               void* stream);

/* Absorb n_tokens evicted tokens per (b, h) into the state:
 *   S += phi(K_ev)^T V_ev, z += sum_t phi(K_ev[t])   (K_ev, V_ev: [B][H][n_tokens][d])
 * Source: Hybrid Forcing, German technical summary section 2 A (evicted frames are
 * aggregated into the compact state by a linear attention function); English abstract.
 * phi is evaluated in fp32; phi(K)^T V runs on the tensor cores with phi(K) split
 * into two bf16 terms (hi + lo) and fp32 accumulation; the per-head reduction is
 * deterministic (same inputs -> bit-identical state). n_tokens == 0 is a no-op.
 * st->n_absorbed += n_tokens on success. ws: HF_WS_ABSORB bytes.
 * Errors: HF_ERR_INVALID_ARG, HF_ERR_ALIGNMENT, HF_ERR_WORKSPACE, HF_ERR_CUDA. */
HF_API hf_status hf_absorb_evicted(hf_state* st, const hf_bf16* K_ev, const hf_bf16* V_ev, int n_tokens,
                                   void* ws, size_t ws_bytes, void* stream);

/* Top-r key-block selection for every query block.
 *   nQB = ceil(Nq/block), nKB = ceil(Nk/block)
 *   score[b][h][I][J] = mean(Q rows of block I) . mean(K rows of block J)   (fp32)
 *   idx_out[b][h][I][0..r) = the r blocks J of largest score, ties to the lower J,
 *                            in ascending order                           (int32)
 * Sources: Light Forcing, German technical summary section 2.2 (mean pooling at block
 * level, selection per query block); Hybrid Forcing, German technical summary
 * section 2 A (Top-K blocks). Q: [B][H][Nq][d], K: [B][H][Nk][d].
 * scores_out: optional [B][H][nQB][nKB] fp32 (NULL to skip). NaN scores rank last.
 * Nq == 0 is a no-op. ws: HF_WS_SELECT bytes.
 * Errors: HF_ERR_INVALID_ARG (Nk < 1, r outside [1, nKB], NULL), HF_ERR_UNSUPPORTED,
 * HF_ERR_ALIGNMENT, HF_ERR_WORKSPACE, HF_ERR_CUDA. */
HF_API hf_status hf_select_blocks(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk, int d,
                                  int block, int r, int32_t* idx_out, float* scores_out, void* ws,
                                  size_t ws_bytes, void* stream);

/* Two-stage top-r key-block selection: frames first, then blocks within the kept frames.
 *   frames: runs of tokens_per_frame tokens of the window (the last may be partial),
 *           W = ceil(Nk / tokens_per_frame); tokens_per_frame >= block
 *   f[b][h][I][w] = mean(Q rows of block I) . mean(K rows of frame w)            (fp32)
 *   frames_out[b][h][I][0..n_frames) = the n_frames frames of largest f, ties to the
 *                                      lower w, ascending                      (int32)
 *   candidate blocks: the key blocks with at least one token in a kept frame
 *   idx_out[b][h][I][0..r) = the r candidates of largest score (as in hf_select_blocks),
 *                            ties to the lower J, ascending; with fewer than r
 *                            candidates, every candidate and then the best other
 *                            blocks                                             (int32)
 * Source: Light Forcing, German technical summary section 2.2 (tokens compressed by mean
 * pooling at block and frame level; two-stage mask selection: a small set of frames by
 * the frame-level compressed keys, then the blocks within them by the block-level ones).
 * Q: [B][H][Nq][d], K: [B][H][Nk][d]. frames_out ([B][H][nQB][n_frames]) and scores_out
 * ([B][H][nQB][nKB], fp32 block scores) are optional (NULL to skip). The output feeds
 * hf_hybrid_attn_fwd like hf_select_blocks'. Nq == 0 is a no-op.
 * ws: HF_WS_SELECT_TWO_STAGE bytes (hf_workspace_size with the same block and r).
 * Errors: HF_ERR_INVALID_ARG (Nk < 1, r outside [1, nKB], n_frames outside [1, W],
 * tokens_per_frame < block, NULL), HF_ERR_UNSUPPORTED (d, block, nKB > 4096),
 * HF_ERR_ALIGNMENT, HF_ERR_WORKSPACE, HF_ERR_CUDA. */
HF_API hf_status hf_select_blocks_two_stage(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk,
                                            int d, int block, int r, int tokens_per_frame, int n_frames,
                                            int32_t* idx_out, int32_t* frames_out, float* scores_out, void* ws,
                                            size_t ws_bytes, void* stream);

/* Capped relative temporal RoPE of a chunk step. Source: Hybrid Forcing, German
 * technical summary section 2 C and Portuguese technical summary section 2 B.2 (the
 * largest temporal RoPE index is capped, in training and inference alike, and positions
 * are expressed as relative offsets). Readings where the pages give no numbers:
 *   - the temporal part acts on dimensions [0, d_t) of every head as consecutive pairs
 *     (2i, 2i+1), turned by the angle p * base^(-2i/d_t) (textbook RoPE frequencies);
 *   - a token's index p comes from its frame's offset delta to the newest frame of the
 *     window: p = cap - min(delta, cap) (the newest frame at cap, every frame cap or more
 *     frames old at 0);
 *   - the window K holds ceil(Nk / tokens_per_frame) frames from frame 0; Q's first
 *     token lies in window frame q_frame0 (the chunk is the window's newest frames);
 *   - the rotation applies to q and k of the softmax branch and of the block selection;
 *     the linear branch (readout and absorption) reads the raw q and k.
 * Q and K are passed unrotated; the kernels turn them on the fly. */
typedef struct hf_rope {
  int d_t;               /* rotated dimensions: even, 0 <= d_t <= min(d, 64)             */
  int tokens_per_frame;  /* >= block                                                    */
  int cap;               /* index cap P: 0 <= cap <= 63                                 */
  int q_frame0;          /* window frame of Q's first token, 0 <= q_frame0 < window frames */
  float base;            /* frequency base (10000 in the textbook form); > 1            */
} hf_rope;

/* hf_select_blocks on the turned Q and K: the block means are those of the turned tokens
 * (each block's per-frame sums turned by the frame's index). rope: see hf_rope.
 * Errors: those of hf_select_blocks, and HF_ERR_INVALID_ARG for a NULL or invalid rope. */
HF_API hf_status hf_select_blocks_rope(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk, int d,
                                       int block, int r, const hf_rope* rope, int32_t* idx_out,
                                       float* scores_out, void* ws, size_t ws_bytes, void* stream);

/* hf_hybrid_attn_fwd with the softmax branch on the turned Q and K (the readout on the raw
 * Q): O = softmax over the kept blocks of scale * (R q) . (R k), times V, plus
 * phi(q)^T S / (phi(q) . z + 1e-6). The kernel turns the Q tile and every kept K tile in
 * shared memory. ws: none. Errors: those of hf_hybrid_attn_fwd, and HF_ERR_INVALID_ARG
 * for a NULL or invalid rope. */
HF_API hf_status hf_hybrid_attn_fwd_rope(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H,
                                         int Nq, int Nk, int d, int block, int r, const int32_t* idx,
                                         const hf_state* st, float scale, const hf_rope* rope, hf_bf16* O, void* ws,
                                         size_t ws_bytes, void* stream);

/* Pooled-key cache of the sliding window: the window's keys as fp32 sums of `granule`
 * consecutive tokens, in a ring of `capacity` sums per (b, h). A chunk step sums only the
 * keys that enter the window (hf_kpool_push) and the selection pools its key blocks from
 * the sums (hf_select_blocks_cached) instead of reading the window's K: with 8-token
 * granules it reads a quarter of K's bytes. The window is the n_gran sums from ring slot
 * head on, i.e. n_gran * granule key tokens. The library updates head and n_gran; the
 * caller owns `sums` ([B][H][capacity][d] fp32, device). A push writes ring slots that
 * earlier calls may still read on the device: calls on one stream are ordered; calls on
 * different streams must be ordered by the caller. */
typedef struct hf_kpool {
  int B, H, d;
  int granule;   /* tokens per sum; divides the block size and every push / evict count */
  int capacity;  /* ring slots per (b, h) */
  int n_gran;    /* sums in the window */
  int head;      /* ring slot of the window's first sum */
  float* sums;
} hf_kpool;

/* Empty cache. granule: 1, 2, 4, ... 128 (it must also divide the block size used with
 * the cache); capacity >= 1; d in {64, 128}; sums 16-byte aligned. No device work.
 * Errors: HF_ERR_INVALID_ARG, HF_ERR_UNSUPPORTED (d), HF_ERR_ALIGNMENT. */
HF_API hf_status hf_kpool_init(hf_kpool* kp, int B, int H, int d, int granule, int capacity, float* sums_dev);

/* The window moves: first the n_evict oldest key tokens leave it, then the n_tokens of
 * K_new ([B][H][n_tokens][d] bf16, the newest keys, in order) enter it; the sums of their
 * granules are written into the ring. n_tokens and n_evict are multiples of granule,
 * n_evict at most the window, and the new window fits the capacity. Source: the sliding
 * window of Hybrid Forcing (German technical summary sections 1 and 2 A: the window keeps
 * the recent frames, the oldest leave it) with Light Forcing section 2.2's block mean
 * pooling, computed from sums that stay valid while the window moves.
 * Ordering: kp->head and kp->n_gran move on the host when the push is issued, and the
 * push's kernel overwrites the ring slots of the evicted keys. Every earlier
 * hf_select_blocks_cached on the same ring must therefore be ordered before the push on
 * the device: issue both on one stream, or make the push's stream wait on an event
 * recorded after the select. The library does not detect a violation.
 * Errors (kp unchanged): HF_ERR_INVALID_ARG, HF_ERR_ALIGNMENT, HF_ERR_CUDA. */
HF_API hf_status hf_kpool_push(hf_kpool* kp, const hf_bf16* K_new, int n_tokens, int n_evict, void* stream);

/* hf_select_blocks over the cached window: the same scores, blocks, order and outputs,
 * for the window K of Nk = n_gran * granule tokens that the pushes put into kp (the key
 * block means come from the granule sums, in fp32). block % granule == 0. ws:
 * HF_WS_SELECT bytes for (Nq, Nk). Errors: those of hf_select_blocks, and
 * HF_ERR_INVALID_ARG for an empty window or a block the granule does not divide. */
HF_API hf_status hf_select_blocks_cached(const hf_bf16* Q, const hf_kpool* kp, int Nq, int block, int r,
                                         int32_t* idx_out, float* scores_out, void* ws, size_t ws_bytes,
                                         void* stream);

/* hf_kpool_push(kp, K_new, n_tokens, n_evict) then hf_select_blocks_cached(Q, kp, ...) as
 * one call, the chunk step of the cache: the new keys' granule sums are computed in the
 * launch that pools Q (one launch fewer than the two calls). Same results, ordering rules
 * and errors as the two calls; on any error kp is unchanged and nothing is launched
 * (HF_ERR_CUDA: a launch failed, kp unchanged). Nq == 0: the push alone. */
HF_API hf_status hf_select_blocks_cached_push(const hf_bf16* Q, hf_kpool* kp, const hf_bf16* K_new, int n_tokens,
                                              int n_evict, int Nq, int block, int r, int32_t* idx_out,
                                              float* scores_out, void* ws, size_t ws_bytes, void* stream);

/* Upper bound, in bytes, of the select workspace that hf_select_blocks_noalloc can
 * serve: a call is accepted when hf_workspace_size(HF_WS_SELECT, ...) for its shapes
 * is at most this (e.g. 12 heads x 4680 query x 32760 key tokens at d = 128, block
 * 128 need 1.7 MiB; 40 heads x 10800 x 43200 need 8.3 MiB). */
#define HF_SELECT_NOALLOC_SCRATCH_BYTES (16u << 20)

/* hf_select_blocks for callers that cannot hand the library any device memory of
 * their own: same arguments, results and errors, minus the workspace. The paper has
 * no counterpart of this call; it exists for hosts that must not call cudaMalloc or
 * an allocating library around the step (an allocation may synchronise the device or
 * fail in the middle of a stream), or whose memory is owned by an allocator they
 * cannot reach. Instead of a workspace it uses a fixed scratch array that the library
 * holds in device memory, HF_SELECT_NOALLOC_SCRATCH_BYTES per device (present on
 * every device the library's kernels are loaded on, whether this call is used or not).
 *   - Shapes whose select workspace exceeds HF_SELECT_NOALLOC_SCRATCH_BYTES return
 *     HF_ERR_WORKSPACE before anything runs; use hf_select_blocks for those.
 *   - The first call in a CUDA context (the device's primary context, or whichever
 *     context is current) does a one-off set-up: it looks up the scratch's device
 *     address in that context, which may load the library's kernels there. Make that
 *     first call before any stream capture begins. The address is kept per device
 *     together with the context it belongs to, and looked up again when the current
 *     context differs (a symbol has one copy per context; after cudaDeviceReset the
 *     primary context is a new one, so the first call after a reset is again a set-up
 *     call). A failed set-up returns HF_ERR_CUDA and is retried by the next call.
 *     Arguments the call rejects are rejected before the set-up, without any CUDA call.
 *   - Nothing in the scratch needs to start at zero: every byte a call reads was
 *     written earlier in that same call.
 *   - All calls on one device share the one scratch. Two calls whose kernels overlap
 *     in time (different streams, or different host threads, without ordering between
 *     them) race on it and may return wrong blocks; calls on one stream are ordered
 *     and safe.
 *   - Device indices >= 64 return HF_ERR_UNSUPPORTED.
 * Errors: those of hf_select_blocks, with HF_ERR_WORKSPACE meaning "too large for the
 * fixed scratch". */
HF_API hf_status hf_select_blocks_noalloc(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk,
                                          int d, int block, int r, int32_t* idx_out, float* scores_out,
                                          void* stream);

/* Hybrid attention output for the query chunk:
 *   O[b][h][i] = sum_{j in kept(I(i))} softmax_j(scale * q_i . k_j) v_j
 *              + phi(q_i)^T S[b][h] / (phi(q_i) . z[b][h] + 1e-6)
 * where kept(I) are the valid tokens of the key blocks idx[b][h][I][0..r).
 * Sources: Hybrid Forcing, German technical summary section 2 A ("Kombination": output
 * = sum of the compressed global history and the sparse local interaction);
 * Portuguese technical summary section 2 A.
 * Q, O: [B][H][Nq][d]; K, V: [B][H][Nk][d] (the window); idx: [B][H][nQB][r] int32,
 * normally from hf_select_blocks (any order is accepted; an index outside [0, nKB) is
 * skipped and flagged as HF_ERR_DEVICE_BAD_INDEX in the device error word);
 * st: the state (read only). scale <= 0 selects 1/sqrt(d). O is written in bf16
 * (round to nearest even). Nq == 0 is a no-op. ws: none (HF_WS_ATTN = 0 bytes).
 * The attention uses the state as it stands: a frame must be either in the window or
 * absorbed in the state, never both.
 * Errors: HF_ERR_INVALID_ARG, HF_ERR_UNSUPPORTED, HF_ERR_ALIGNMENT, HF_ERR_CUDA. */
HF_API hf_status hf_hybrid_attn_fwd(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H,
                                    int Nq, int Nk, int d, int block, int r, const int32_t* idx,
                                    const hf_state* st, float scale, hf_bf16* O, void* ws, size_t ws_bytes,
                                    void* stream);

/* One chunk step's attention and absorption in a single call:
 *   O = hf_hybrid_attn_fwd(Q, K, V, idx, state as it stands), then
 *   state += the n_evicted tokens (K_ev, V_ev: [B][H][n_evicted][d]) as hf_absorb_evicted.
 * Source: Hybrid Forcing, German technical summary section 2 A (the output sums the
 * sparse window term and the linear term of the compact state; frames leaving the window
 * are aggregated into that state). The window of the next chunk no longer holds the
 * evicted frames, so O reads the state before their absorption and the next call's O
 * after it.
 * The absorption's partial sums (which read only K_ev and V_ev) run on the SMs that the
 * attention's last CTAs leave, while those CTAs finish; only the final slice reduction,
 * which writes S and z, waits for the whole attention. Results are bit-identical to
 * hf_hybrid_attn_fwd followed by hf_absorb_evicted on the same stream.
 * K_ev, V_ev and ws must be complete when the call is issued (written by earlier work of
 * `stream`) and must not overlap O. ws: HF_WS_ABSORB bytes for n_evicted tokens (NULL
 * when n_evicted == 0). Nq == 0 runs the absorption alone; n_evicted == 0 the attention
 * alone. st->n_absorbed += n_evicted on success.
 * Errors: those of hf_hybrid_attn_fwd and hf_absorb_evicted, checked before anything is
 * launched. */
HF_API hf_status hf_hybrid_attn_fwd_absorb(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H,
                                           int Nq, int Nk, int d, int block, int r, const int32_t* idx,
                                           hf_state* st, float scale, hf_bf16* O, const hf_bf16* K_ev,
                                           const hf_bf16* V_ev, int n_evicted, void* ws, size_t ws_bytes,
                                           void* stream);

/* Per-chunk keep schedule of chunk-aware growth (host only; no device work): the
 * sparsity ratio s[i] and the kept key blocks r[i] of every chunk i of a video, for
 * hf_select_blocks / hf_hybrid_attn_fwd of that chunk.
 *   s[0] = 0                                  (the first chunk attends densely)
 *   s[i] = s_base - beta / sqrt(i), i >= 1    (sparsity grows towards s_base)
 *   beta: sum_i (1 - s[i]) nKB[i] = (1 - s_target) sum_i nKB[i]   (the FLOP budget)
 *   r[i] = clamp(ceil((1 - s[i]) nKB[i]), 1, nKB[i])
 * Source: Light Forcing, German technical summary section 2.1 (dense first chunk;
 * s_i = s_base - alpha_i beta with alpha_i following the noise scale 1/sqrt(T); beta set
 * so that the total FLOPs meet a target sparsity ratio). Readings where the page gives
 * no constants: alpha_i = 1/sqrt(i) with the chunk's position i as T; a chunk's FLOPs
 * proportional to its window's key blocks nKB[i] (every chunk has the same queries).
 * nKB: [n_chunks] host ints >= 1 (the window of chunk i, in blocks); r_out: [n_chunks]
 * host ints (written on success only); s_out: optional [n_chunks] host doubles (NULL to
 * skip); beta_out optional. n_chunks == 1 gives the dense first chunk whatever s_target.
 * Errors (nothing written): HF_ERR_INVALID_ARG for n_chunks < 1, a NULL nKB or r_out,
 * nKB[i] < 1, s_base or s_target outside [0, 1), a budget that would need beta < 0
 * (sparsity falling with i: raise s_base) or an s[i] outside [0, 1). */
HF_API hf_status hf_keep_schedule(int n_chunks, const int* nKB, double s_base, double s_target, int* r_out,
                                  double* s_out, double* beta_out);

/* Synchronise `stream`, then read and clear the device error word of the current
 * device. Returns HF_OK, HF_ERR_DEVICE_TIMEOUT, HF_ERR_DEVICE_BAD_INDEX or HF_ERR_CUDA
 * (an asynchronous CUDA error). If detail_out is not NULL it receives the raw word
 * (high 16 bits: error tag, low 16 bits: kernel id << 8 | wait site), 0 if none. */
HF_API hf_status hf_query_status(void* stream, uint32_t* detail_out);

/* Static description of a status code. */
HF_API const char* hf_status_string(hf_status s);

/* Library version string. */
HF_API const char* hf_version(void);

/* Number of kernels this library instance has launched since it was loaded (a host-side
 * count of launches that returned without error, over all devices and streams). A
 * caller reads it before and after a region to count the library's launches there. */
HF_API unsigned long long hf_launch_count(void);

/* TEST ONLY. Makes the next `count` launches of kernel `kernel_id` (1 = select,
 * 2 = absorb, 3 = attention) skip one internal barrier arrival, so that one wait runs
 * out after `timeout_ns` nanoseconds; the kernel then records HF_ERR_DEVICE_TIMEOUT,
 * drains its own copies and MMAs, frees its tensor memory and returns. The context
 * stays usable. kernel_id 0 clears the injection. The bound of every other wait of
 * those launches is also `timeout_ns`. Host-side setting of this library instance. */
HF_API hf_status hf_debug_inject_timeout(int kernel_id, int count, unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* HF_H_ */
