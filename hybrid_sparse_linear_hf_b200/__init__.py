"""Hybrid attention chunk step (Hybrid Forcing) for NVIDIA B200 / sm_100a.

For each new chunk of query tokens the output is the sum of block-sparse softmax
attention over the top-r key blocks of the local sliding window and a linear-attention
readout of a compact key-value state that absorbs every evicted frame. The step runs in
hand-written sm_100a CUDA kernels behind the C ABI of ``include/hf.h``; this package is
the thin Python binding of that ABI (same function names) plus the seeded synthetic
input generator.
"""
from ._binding import (  # noqa: F401
    HF_ERR_ALIGNMENT, HF_ERR_CUDA, HF_ERR_DEVICE_BAD_INDEX, HF_ERR_DEVICE_TIMEOUT, HF_ERR_INVALID_ARG,
    HF_ERR_UNSUPPORTED, HF_ERR_WORKSPACE, HF_OK, HF_SELECT_NOALLOC_SCRATCH_BYTES, HF_WS_ABSORB, HF_WS_ATTN,
    HF_WS_SELECT, HF_WS_SELECT_TWO_STAGE, LIB_PATH, HfError, HfKpool, HfState, hf_absorb_evicted,
    hf_debug_inject_timeout, hf_hybrid_attn_fwd, hf_hybrid_attn_fwd_absorb, hf_hybrid_attn_fwd_rope,
    hf_keep_schedule, hf_rope, hf_select_blocks_rope, HfRopeC, hf_launch_count, hf_kpool_init, hf_kpool_push,
    hf_query_status, hf_select_blocks, hf_select_blocks_cached, hf_select_blocks_cached_push, hf_select_blocks_noalloc,
    hf_select_blocks_two_stage, hf_state_init, hf_status_string, hf_version, hf_workspace_size, lib,
)
