"""ctypes binding of ``libhf.so`` (C ABI in ``include/hf.h``), same names as the C calls.

Argument marshalling only: every step of the hybrid attention step runs in the CUDA
kernels of the library. PyTorch supplies device memory (tensors) and streams. There is
no CPU fallback: if the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhf.so")

HF_OK = 0
HF_ERR_INVALID_ARG = 1
HF_ERR_UNSUPPORTED = 2
HF_ERR_ALIGNMENT = 3
HF_ERR_WORKSPACE = 4
HF_ERR_CUDA = 5
HF_ERR_DEVICE_TIMEOUT = 6
HF_ERR_DEVICE_BAD_INDEX = 7

HF_WS_SELECT = 1
HF_WS_ATTN = 2
HF_WS_ABSORB = 3
HF_WS_SELECT_TWO_STAGE = 4

_SIZE_T_MAX = (1 << (8 * ctypes.sizeof(ctypes.c_size_t))) - 1


class HfStateC(ctypes.Structure):
    """Mirror of ``struct hf_state``."""

    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("S", ctypes.c_void_p), ("z", ctypes.c_void_p), ("S_split", ctypes.c_void_p),
                ("n_absorbed", ctypes.c_longlong)]


class HfKpoolC(ctypes.Structure):
    """Mirror of ``struct hf_kpool``."""

    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("granule", ctypes.c_int),
                ("capacity", ctypes.c_int), ("n_gran", ctypes.c_int), ("head", ctypes.c_int),
                ("sums", ctypes.c_void_p)]


class HfRopeC(ctypes.Structure):
    """Mirror of ``struct hf_rope``."""

    _fields_ = [("d_t", ctypes.c_int), ("tokens_per_frame", ctypes.c_int), ("cap", ctypes.c_int),
                ("q_frame0", ctypes.c_int), ("base", ctypes.c_float)]


def hf_rope(d_t: int, tokens_per_frame: int, cap: int, q_frame0: int, base: float = 10000.0) -> HfRopeC:
    """The temporal RoPE of a chunk step (see ``hf_rope`` in include/hf.h)."""
    return HfRopeC(int(d_t), int(tokens_per_frame), int(cap), int(q_frame0), float(base))


class HfError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {hf_status_string(status)} (status {status})")


_lib = None

_SIGNATURES = {
    "hf_workspace_size": (ctypes.c_size_t, [ctypes.c_int] * 8),
    "hf_state_init": (ctypes.c_int, [ctypes.POINTER(HfStateC), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "hf_absorb_evicted": (ctypes.c_int, [ctypes.POINTER(HfStateC), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "hf_select_blocks": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 7 +
                         [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "hf_select_blocks_two_stage": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 9 +
                                   [ctypes.c_void_p] * 4 + [ctypes.c_size_t, ctypes.c_void_p]),
    "hf_select_blocks_rope": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 7 +
                              [ctypes.POINTER(HfRopeC), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.c_size_t, ctypes.c_void_p]),
    "hf_hybrid_attn_fwd_rope": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 +
                                [ctypes.c_void_p, ctypes.POINTER(HfStateC), ctypes.c_float, ctypes.POINTER(HfRopeC),
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "hf_select_blocks_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 7 +
                                 [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "hf_hybrid_attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 +
                           [ctypes.c_void_p, ctypes.POINTER(HfStateC), ctypes.c_float, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "hf_hybrid_attn_fwd_absorb": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 +
                                  [ctypes.c_void_p, ctypes.POINTER(HfStateC), ctypes.c_float, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_size_t, ctypes.c_void_p]),
    "hf_kpool_init": (ctypes.c_int, [ctypes.POINTER(HfKpoolC)] + [ctypes.c_int] * 5 + [ctypes.c_void_p]),
    "hf_kpool_push": (ctypes.c_int, [ctypes.POINTER(HfKpoolC), ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p]),
    "hf_select_blocks_cached_push": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(HfKpoolC), ctypes.c_void_p]
                                     + [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                             ctypes.c_size_t, ctypes.c_void_p]),
    "hf_select_blocks_cached": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(HfKpoolC)] + [ctypes.c_int] * 3 +
                                [ctypes.c_void_p] * 3 + [ctypes.c_size_t, ctypes.c_void_p]),
    "hf_keep_schedule": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_double,
                                        ctypes.c_double, ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    "hf_query_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
    "hf_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hf_version": (ctypes.c_char_p, []),
    "hf_launch_count": (ctypes.c_ulonglong, []),
    "hf_debug_inject_timeout": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_ulonglong]),
}


def lib() -> ctypes.CDLL:
    """The loaded library; raises if ``libhf.so`` has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m hybrid_sparse_linear_hf_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def hf_status_string(status: int) -> str:
    return lib().hf_status_string(int(status)).decode()


def hf_version() -> str:
    return lib().hf_version().decode()


def hf_launch_count() -> int:
    """Kernels the library has launched since it was loaded (host-side count)."""
    return int(lib().hf_launch_count())


def _check(rc: int, where: str) -> None:
    if rc != HF_OK:
        raise HfError(rc, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _shape(t, shape, name: str) -> None:
    """Host-side shape check of an optional tensor argument (before any device access)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in shape)}, got {tuple(t.shape)}")


def _qkv_dims(Q: torch.Tensor, K: torch.Tensor, name_k: str = "K"):
    """(B, H, Nq, Nk, d) of a query tensor [B,H,Nq,d] and a key tensor [B,H,Nk,d]."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-D tensor [B,H,Nq,d]")
    B, H, Nq, d = Q.shape
    if not isinstance(K, torch.Tensor) or K.dim() != 4 or tuple(K.shape[:2]) != (B, H) or K.shape[3] != d:
        raise ValueError(f"{name_k} must be [B,H,Nk,d] with Q's B={B}, H={H} and d={d}, got "
                         f"{tuple(K.shape) if isinstance(K, torch.Tensor) else type(K).__name__}")
    return B, H, Nq, K.shape[2], d


class HfState:
    """Python handle of ``hf_state``: keeps S [B,H,d,d], z [B,H,d] (fp32, device) and the
    split copy of S that the library maintains (``S_split``, bytes) alive."""

    def __init__(self, S: torch.Tensor, z: torch.Tensor, S_split: torch.Tensor):
        self.S = S
        self.z = z
        self.S_split = S_split
        self.c = HfStateC()

    @property
    def n_absorbed(self) -> int:
        return int(self.c.n_absorbed)

    @property
    def shape(self):
        return (self.c.B, self.c.H, self.c.d)


class HfKpool:
    """Python handle of ``hf_kpool``: keeps the granule sums [B,H,capacity,d] (fp32,
    device) alive; ``n_tokens`` is the window length the pushes have built."""

    def __init__(self, sums: torch.Tensor):
        self.sums = sums
        self.c = HfKpoolC()

    @property
    def n_tokens(self) -> int:
        return int(self.c.n_gran) * int(self.c.granule)


def hf_workspace_size(which: int, B: int, H: int, Nq: int, Nk: int, d: int, block: int, r: int) -> int:
    n = lib().hf_workspace_size(which, B, H, Nq, Nk, d, block, r)
    if n == _SIZE_T_MAX:
        raise HfError(HF_ERR_INVALID_ARG, "hf_workspace_size")
    return int(n)


def _workspace(nbytes: int, device, ws, stream=None):
    """The caller's workspace, or a new one; a new one used on another torch stream than the
    current one is recorded on it, so that the allocator does not hand its memory out again
    before that stream's work is done."""
    if nbytes == 0:
        return None, 0
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        if isinstance(stream, torch.cuda.Stream) and stream != torch.cuda.current_stream(ws.device):
            ws.record_stream(stream)
    return ws, ws.numel() * ws.element_size()


def hf_state_init(S: torch.Tensor, z: torch.Tensor, S_split=None, stream=None) -> HfState:
    """Bind S [B,H,d,d] and z [B,H,d] (fp32) as a state and zero them. S_split: the
    library's split copy of S (uint8 [B*H*4*d*d] on S's device; allocated when None)."""
    if S.dim() != 4 or z.dim() != 3:
        raise ValueError("S must be [B,H,d,d] and z [B,H,d]")
    B, H, d, _ = S.shape
    if S_split is None:
        S_split = torch.empty(B * H * 4 * d * d, dtype=torch.uint8, device=S.device)
    if S_split.dtype != torch.uint8 or S_split.numel() < B * H * 4 * d * d:
        raise ValueError(f"S_split must be uint8 with at least {B * H * 4 * d * d} bytes")
    st = HfState(S, z, S_split)
    _check(lib().hf_state_init(ctypes.byref(st.c), B, H, d, _dev(S, torch.float32, "S"),
                               _dev(z, torch.float32, "z"), _dev(S_split, torch.uint8, "S_split"),
                               _stream(stream)), "hf_state_init")
    return st


def hf_absorb_evicted(state: HfState, K_ev: torch.Tensor, V_ev: torch.Tensor, ws=None, stream=None) -> None:
    """S += phi(K_ev)^T V_ev, z += sum phi(K_ev) for K_ev, V_ev [B,H,n,d] bf16."""
    B, H, d = state.shape
    if K_ev.shape != V_ev.shape or K_ev.dim() != 4 or tuple(K_ev.shape[:2]) != (B, H) or K_ev.shape[3] != d:
        raise ValueError("K_ev and V_ev must both be [B,H,n,d] matching the state")
    n = K_ev.shape[2]
    nbytes = hf_workspace_size(HF_WS_ABSORB, B, H, 0, n, d, 0, 0)
    ws, ws_bytes = _workspace(nbytes, K_ev.device, ws, stream)
    _check(lib().hf_absorb_evicted(ctypes.byref(state.c), _dev(K_ev, torch.bfloat16, "K_ev"),
                                   _dev(V_ev, torch.bfloat16, "V_ev"), n,
                                   ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)),
           "hf_absorb_evicted")


def hf_select_blocks(Q: torch.Tensor, K: torch.Tensor, block: int, r: int, idx_out=None, scores_out=None,
                     ws=None, stream=None) -> torch.Tensor:
    """Top-r key blocks per query block: int32 [B,H,nQB,r] (ascending)."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    if idx_out is None:
        idx_out = torch.empty(B, H, nQB, r, dtype=torch.int32, device=Q.device)
    nbytes = hf_workspace_size(HF_WS_SELECT, B, H, Nq, Nk, d, block, r)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_select_blocks(_dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), B, H, Nq, Nk, d,
                                  block, r, _dev(idx_out, torch.int32, "idx_out"),
                                  _dev(scores_out, torch.float32, "scores_out") if scores_out is not None else None,
                                  ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)),
           "hf_select_blocks")
    return idx_out


def hf_select_blocks_rope(Q: torch.Tensor, K: torch.Tensor, block: int, r: int, rope: HfRopeC, idx_out=None,
                          scores_out=None, ws=None, stream=None) -> torch.Tensor:
    """hf_select_blocks on Q and K turned by the temporal RoPE ``rope`` (``hf_rope(...)``)."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    if not isinstance(rope, HfRopeC):
        raise TypeError("rope must come from hf_rope(...)")
    if idx_out is None:
        idx_out = torch.empty(B, H, nQB, r, dtype=torch.int32, device=Q.device)
    nbytes = hf_workspace_size(HF_WS_SELECT, B, H, Nq, Nk, d, block, r)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_select_blocks_rope(_dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), B, H, Nq, Nk, d,
                                       block, r, ctypes.byref(rope), _dev(idx_out, torch.int32, "idx_out"),
                                       _dev(scores_out, torch.float32, "scores_out")
                                       if scores_out is not None else None,
                                       ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)),
           "hf_select_blocks_rope")
    return idx_out


def hf_kpool_init(sums: torch.Tensor, granule: int) -> HfKpool:
    """An empty pooled-key cache over ``sums`` [B,H,capacity,d] fp32 (device): the ring
    of the window's sums of ``granule`` consecutive key tokens."""
    if sums.dim() != 4:
        raise ValueError("sums must be [B,H,capacity,d]")
    B, H, cap, d = sums.shape
    kp = HfKpool(sums)
    _check(lib().hf_kpool_init(ctypes.byref(kp.c), B, H, d, granule, cap, _dev(sums, torch.float32, "sums")),
           "hf_kpool_init")
    return kp


def hf_kpool_push(kp: HfKpool, K_new, n_evict: int = 0, stream=None) -> None:
    """The window drops its ``n_evict`` oldest key tokens, then takes K_new [B,H,n,d] bf16
    (or None for no new keys) as its newest."""
    n = 0 if K_new is None else int(K_new.shape[2])
    if K_new is not None and (K_new.dim() != 4 or tuple(K_new.shape[:2]) != (kp.c.B, kp.c.H)
                              or K_new.shape[3] != kp.c.d):
        raise ValueError("K_new must be [B,H,n,d] matching the cache")
    _check(lib().hf_kpool_push(ctypes.byref(kp.c), _dev(K_new, torch.bfloat16, "K_new") if n > 0 else None, n,
                               int(n_evict), _stream(stream)), "hf_kpool_push")


def hf_select_blocks_cached(Q: torch.Tensor, kp: HfKpool, block: int, r: int, idx_out=None, scores_out=None,
                            ws=None, stream=None) -> torch.Tensor:
    """hf_select_blocks over the cached window (its ``kp.n_tokens`` keys)."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-D tensor [B,H,Nq,d]")
    B, H, Nq, d = Q.shape
    if (B, H, d) != (kp.c.B, kp.c.H, kp.c.d):
        raise ValueError(f"Q's (B, H, d) = {(B, H, d)} must match the cache's {(kp.c.B, kp.c.H, kp.c.d)}")
    Nk = kp.n_tokens
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    if idx_out is None:
        idx_out = torch.empty(B, H, nQB, r, dtype=torch.int32, device=Q.device)
    nbytes = hf_workspace_size(HF_WS_SELECT, B, H, Nq, max(Nk, 1), d, block, 1)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_select_blocks_cached(_dev(Q, torch.bfloat16, "Q"), ctypes.byref(kp.c), Nq, block, r,
                                         _dev(idx_out, torch.int32, "idx_out"),
                                         _dev(scores_out, torch.float32, "scores_out")
                                         if scores_out is not None else None,
                                         ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)),
           "hf_select_blocks_cached")
    return idx_out


def hf_select_blocks_cached_push(Q: torch.Tensor, kp: HfKpool, K_new, block: int, r: int, n_evict: int = 0,
                                 idx_out=None, scores_out=None, ws=None, stream=None) -> torch.Tensor:
    """hf_kpool_push(kp, K_new, n_evict) then hf_select_blocks_cached(Q, kp, ...), in one call."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-D tensor [B,H,Nq,d]")
    B, H, Nq, d = Q.shape
    if (B, H, d) != (kp.c.B, kp.c.H, kp.c.d):
        raise ValueError(f"Q's (B, H, d) = {(B, H, d)} must match the cache's {(kp.c.B, kp.c.H, kp.c.d)}")
    n = 0 if K_new is None else int(K_new.shape[2])
    if K_new is not None and (K_new.dim() != 4 or tuple(K_new.shape[:2]) != (B, H) or K_new.shape[3] != d):
        raise ValueError("K_new must be [B,H,n,d] matching the cache")
    G = int(kp.c.granule)
    Nk = (int(kp.c.n_gran) - int(n_evict) // G + n // G) * G  # the window after the push
    nQB, nKB = -(-Nq // block), -(-max(Nk, 1) // block)
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    if idx_out is None:
        idx_out = torch.empty(B, H, nQB, r, dtype=torch.int32, device=Q.device)
    nbytes = hf_workspace_size(HF_WS_SELECT, B, H, Nq, max(Nk, 1), d, block, 1)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_select_blocks_cached_push(_dev(Q, torch.bfloat16, "Q"), ctypes.byref(kp.c),
                                              _dev(K_new, torch.bfloat16, "K_new") if n > 0 else None, n,
                                              int(n_evict), Nq, block, r, _dev(idx_out, torch.int32, "idx_out"),
                                              _dev(scores_out, torch.float32, "scores_out")
                                              if scores_out is not None else None,
                                              ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)),
           "hf_select_blocks_cached_push")
    return idx_out


def hf_select_blocks_two_stage(Q: torch.Tensor, K: torch.Tensor, block: int, r: int, tokens_per_frame: int,
                               n_frames: int, idx_out=None, frames_out=None, scores_out=None, ws=None,
                               stream=None) -> torch.Tensor:
    """Two-stage top-r key blocks per query block (frames, then blocks within them):
    int32 [B,H,nQB,r] (ascending). frames_out: optional int32 [B,H,nQB,n_frames]."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(frames_out, (B, H, nQB, n_frames), "frames_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    if idx_out is None:
        idx_out = torch.empty(B, H, nQB, r, dtype=torch.int32, device=Q.device)
    nbytes = hf_workspace_size(HF_WS_SELECT_TWO_STAGE, B, H, Nq, Nk, d, block, r)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_select_blocks_two_stage(
        _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), B, H, Nq, Nk, d, block, r, tokens_per_frame,
        n_frames, _dev(idx_out, torch.int32, "idx_out"),
        _dev(frames_out, torch.int32, "frames_out") if frames_out is not None else None,
        _dev(scores_out, torch.float32, "scores_out") if scores_out is not None else None,
        ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)), "hf_select_blocks_two_stage")
    return idx_out


# Largest select workspace hf_select_blocks_noalloc serves (HF_SELECT_NOALLOC_SCRATCH_BYTES).
HF_SELECT_NOALLOC_SCRATCH_BYTES = 16 << 20


def hf_select_blocks_noalloc(Q: torch.Tensor, K: torch.Tensor, block: int, r: int, idx_out: torch.Tensor,
                             scores_out=None, stream=None) -> torch.Tensor:
    """``hf_select_blocks`` without a workspace, for hosts that cannot allocate device
    memory around the step: the library's fixed per-device scratch holds the pooled rows.
    ``idx_out`` [B,H,nQB,r] int32 is caller-provided, so nothing is allocated here either.
    The first call on a device does a one-off set-up (make it before any stream capture);
    calls on one device share the scratch, so calls that overlap in time race."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    nQB, nKB = -(-Nq // block), -(-Nk // block)
    if idx_out is None:
        raise ValueError("idx_out [B,H,nQB,r] int32 is required (nothing is allocated here)")
    _shape(idx_out, (B, H, nQB, r), "idx_out")
    _shape(scores_out, (B, H, nQB, nKB), "scores_out")
    _check(lib().hf_select_blocks_noalloc(_dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), B, H, Nq,
                                          Nk, d, block, r, _dev(idx_out, torch.int32, "idx_out"),
                                          _dev(scores_out, torch.float32, "scores_out")
                                          if scores_out is not None else None, _stream(stream)),
           "hf_select_blocks_noalloc")
    return idx_out


def hf_keep_schedule(nKB, s_base: float, s_target: float):
    """Chunk-aware growth schedule (host only): for chunk windows of ``nKB[i]`` key blocks,
    returns (r, s, beta): kept blocks per chunk (list of int, the ``r`` of that chunk's
    select and attention calls), sparsity ratios (list of float) and beta. The first chunk
    is dense; later chunks approach ``s_base`` as beta/sqrt(i) shrinks; beta makes the
    kept FLOPs equal ``1 - s_target`` of the dense ones."""
    n = len(nKB)
    kb = (ctypes.c_int * max(n, 1))(*[int(x) for x in nKB])
    r = (ctypes.c_int * max(n, 1))()
    sv = (ctypes.c_double * max(n, 1))()
    beta = ctypes.c_double(0.0)
    _check(lib().hf_keep_schedule(n, kb, float(s_base), float(s_target), r, sv, ctypes.byref(beta)),
           "hf_keep_schedule")
    return list(r)[:n], list(sv)[:n], beta.value


def hf_hybrid_attn_fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block: int, r: int,
                       idx: torch.Tensor, state: HfState, scale: float = 0.0, O=None, stream=None) -> torch.Tensor:
    """Hybrid attention output O [B,H,Nq,d] bf16 = sparse term + linear term."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    _shape(V, (B, H, Nk, d), "V")
    _shape(idx, (B, H, -(-Nq // block), r), "idx")
    _shape(O, (B, H, Nq, d), "O")
    if state.shape != (B, H, d):
        raise ValueError(f"the state's (B, H, d) = {state.shape} must match Q's {(B, H, d)}")
    if O is None:
        O = torch.empty_like(Q)
    _check(lib().hf_hybrid_attn_fwd(_dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"),
                                    _dev(V, torch.bfloat16, "V"), B, H, Nq, Nk, d, block, r,
                                    _dev(idx, torch.int32, "idx"), ctypes.byref(state.c), float(scale),
                                    _dev(O, torch.bfloat16, "O"), None, 0, _stream(stream)),
           "hf_hybrid_attn_fwd")
    return O


def hf_hybrid_attn_fwd_rope(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block: int, r: int,
                            idx: torch.Tensor, state: HfState, rope: HfRopeC, scale: float = 0.0, O=None,
                            stream=None) -> torch.Tensor:
    """hf_hybrid_attn_fwd with the softmax branch on Q and K turned by ``rope``."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    _shape(V, (B, H, Nk, d), "V")
    _shape(idx, (B, H, -(-Nq // block), r), "idx")
    _shape(O, (B, H, Nq, d), "O")
    if state.shape != (B, H, d):
        raise ValueError(f"the state's (B, H, d) = {state.shape} must match Q's {(B, H, d)}")
    if not isinstance(rope, HfRopeC):
        raise TypeError("rope must come from hf_rope(...)")
    if O is None:
        O = torch.empty_like(Q)
    _check(lib().hf_hybrid_attn_fwd_rope(_dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"),
                                         _dev(V, torch.bfloat16, "V"), B, H, Nq, Nk, d, block, r,
                                         _dev(idx, torch.int32, "idx"), ctypes.byref(state.c), float(scale),
                                         ctypes.byref(rope), _dev(O, torch.bfloat16, "O"), None, 0, _stream(stream)),
           "hf_hybrid_attn_fwd_rope")
    return O


def hf_hybrid_attn_fwd_absorb(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block: int, r: int,
                              idx: torch.Tensor, state: HfState, K_ev: torch.Tensor, V_ev: torch.Tensor,
                              scale: float = 0.0, O=None, ws=None, stream=None) -> torch.Tensor:
    """O [B,H,Nq,d] bf16 from the state as it stands, then the state absorbs K_ev, V_ev
    [B,H,n,d] bf16 (one call: the absorption's partial sums overlap the attention's last
    CTAs)."""
    B, H, Nq, Nk, d = _qkv_dims(Q, K)
    _shape(V, (B, H, Nk, d), "V")
    _shape(idx, (B, H, -(-Nq // block), r), "idx")
    _shape(O, (B, H, Nq, d), "O")
    if state.shape != (B, H, d):
        raise ValueError(f"the state's (B, H, d) = {state.shape} must match Q's {(B, H, d)}")
    if K_ev.shape != V_ev.shape or K_ev.dim() != 4 or tuple(K_ev.shape[:2]) != (B, H) or K_ev.shape[3] != d:
        raise ValueError("K_ev and V_ev must both be [B,H,n,d] matching Q")
    n = K_ev.shape[2]
    if O is None:
        O = torch.empty_like(Q)
    nbytes = hf_workspace_size(HF_WS_ABSORB, B, H, 0, n, d, 0, 0)
    ws, ws_bytes = _workspace(nbytes, Q.device, ws, stream)
    _check(lib().hf_hybrid_attn_fwd_absorb(
        _dev(Q, torch.bfloat16, "Q"), _dev(K, torch.bfloat16, "K"), _dev(V, torch.bfloat16, "V"), B, H, Nq, Nk, d,
        block, r, _dev(idx, torch.int32, "idx"), ctypes.byref(state.c), float(scale), _dev(O, torch.bfloat16, "O"),
        _dev(K_ev, torch.bfloat16, "K_ev") if n > 0 else None, _dev(V_ev, torch.bfloat16, "V_ev") if n > 0 else None,
        n, ws.data_ptr() if ws is not None else None, ws_bytes, _stream(stream)), "hf_hybrid_attn_fwd_absorb")
    return O


def hf_query_status(stream=None) -> tuple[int, int]:
    """(status, raw device error word) after synchronising the stream; clears the word."""
    detail = ctypes.c_uint32(0)
    rc = lib().hf_query_status(_stream(stream), ctypes.byref(detail))
    return int(rc), int(detail.value)


def hf_debug_inject_timeout(kernel_id: int, count: int, timeout_ns: int) -> None:
    """Test only: see ``hf_debug_inject_timeout`` in include/hf.h."""
    _check(lib().hf_debug_inject_timeout(kernel_id, count, timeout_ns), "hf_debug_inject_timeout")
