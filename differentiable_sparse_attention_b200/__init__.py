"""alpha-entmax attention (forward + backward) for NVIDIA B200, sm_100a.

A thin ctypes binding of ``libentmax_attn.so``, whose C ABI is declared in
``include/entmax_attn.h``.  This module only marshals arguments: every step of
the computation runs in the library's CUDA kernels, and there is no fallback
of any kind -- if the library is missing, the calls raise.
PyTorch provides device memory and the current CUDA stream.
"""

from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# ENTMAX_ATTN_LIB selects another build of the same library, such as the
# bounds-checked debug build libentmax_attn_bounds.so (see build.py).
LIB_PATH = os.environ.get("ENTMAX_ATTN_LIB") or os.path.join(_HERE, "libentmax_attn.so")

OK = 0
E_NULL, E_ALIGN, E_SHAPE, E_UNSUPPORTED, E_ALPHA, E_WORKSPACE, E_CUDA, E_MAXITER, E_SCRATCH = (
    -1, -2, -3, -4, -5, -6, -7, -8, -9)
NOALLOC_SCRATCH_BYTES = 8 << 20
ST_NOT_CONVERGED, ST_TIMEOUT, ST_RANGE, ST_BOUNDS = 1, 2, 4, 8
DTYPE_CODES = {torch.bfloat16: 0, torch.float32: 1}
EXPORTED = ("entmax_attn_mask_words", "entmax_attn_workspace_size", "entmax_attn_fwd",
            "entmax_attn_bwd", "entmax_attn_status", "entmax_attn_counters",
            "entmax_attn_profile", "entmax_attn_profile_read", "entmax_attn_error_string",
            "entmax_attn_fwd_noalloc", "entmax_attn_noalloc_status",
            "entmax_attn_wait_selftest")
# include/dash_route.h: the DashAttention stage-0/1 router
DASH_EXPORTED = ("dash_route_workspace_size", "dash_route_fwd")
DASH_MAX_CHUNKS = 256
COUNTER_NAMES = ("fwd_hist_tiles", "fwd_refine_tiles", "fwd_pv_tiles", "fwd_refine_passes",
                 "bwd_row_tiles", "bwd_col_tiles", "fwd_cand_overflow_tiles")
PHASE_NAMES = ("fwd", "bwd_fp16_copies", "bwd_tile_masks", "bwd_row", "bwd_col")

_lib_handle = None


class EntmaxError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what} failed with {code}: {error_string(code)}")


def _lib():
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing; build it with "
            "`python -m differentiable_sparse_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_float, c_size, vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
    lib.entmax_attn_mask_words.argtypes = [c_int, c_int]
    lib.entmax_attn_mask_words.restype = c_int
    lib.entmax_attn_workspace_size.argtypes = [c_int] * 6
    lib.entmax_attn_workspace_size.restype = c_size
    lib.entmax_attn_fwd.argtypes = ([vp, vp, vp] + [c_int] * 5 + [c_float, c_int, c_int, c_int]
                                    + [vp] * 5 + [c_size, vp])
    lib.entmax_attn_fwd.restype = c_int
    lib.entmax_attn_bwd.argtypes = ([vp] * 6 + [c_int] * 5 + [c_float, c_int, c_int]
                                    + [vp] * 4 + [c_size, vp])
    lib.entmax_attn_bwd.restype = c_int
    lib.entmax_attn_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.entmax_attn_status.restype = c_int
    lib.entmax_attn_counters.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_ulonglong), c_int]
    lib.entmax_attn_counters.restype = c_int
    lib.entmax_attn_profile.argtypes = [c_int]
    lib.entmax_attn_profile.restype = c_int
    lib.entmax_attn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), c_int]
    lib.entmax_attn_profile_read.restype = c_int
    lib.entmax_attn_fwd_noalloc.argtypes = ([vp, vp, vp] + [c_int] * 5
                                            + [c_float, c_int, c_int, c_int] + [vp] * 4)
    lib.entmax_attn_fwd_noalloc.restype = c_int
    lib.entmax_attn_noalloc_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.entmax_attn_noalloc_status.restype = c_int
    lib.entmax_attn_error_string.argtypes = [c_int]
    lib.entmax_attn_error_string.restype = ctypes.c_char_p
    lib.entmax_attn_wait_selftest.argtypes = [vp, vp, ctypes.c_ulonglong, vp]
    lib.entmax_attn_wait_selftest.restype = c_int
    lib.dash_route_workspace_size.argtypes = [c_int] * 6
    lib.dash_route_workspace_size.restype = c_size
    lib.dash_route_fwd.argtypes = ([vp, vp] + [c_int] * 6 + [c_float, c_float, c_int]
                                   + [vp] * 4 + [c_size, vp])
    lib.dash_route_fwd.restype = c_int
    _lib_handle = lib
    return lib


def error_string(code: int) -> str:
    return _lib().entmax_attn_error_string(int(code)).decode()


def mask_words(n: int, block: int) -> int:
    w = _lib().entmax_attn_mask_words(int(n), int(block))
    if w < 0:
        raise EntmaxError(w, "entmax_attn_mask_words")
    return w


def workspace_size(B: int, H: int, N: int, D: int, block: int = 128, causal: bool = True) -> int:
    return int(_lib().entmax_attn_workspace_size(B, H, N, D, block, int(bool(causal))))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(*ts):
    ref = ts[0]
    for t in ts:
        if t.dim() != 4 or t.shape != ref.shape or t.dtype != ref.dtype or not t.is_contiguous():
            raise ValueError("q, k, v (, dout) must be contiguous [B, H, N, D] tensors of one dtype")
        if t.device != ref.device or t.device.type != "cuda":
            raise ValueError("tensors must live on one CUDA device")
    if ref.dtype not in DTYPE_CODES:
        raise ValueError(f"unsupported dtype {ref.dtype}")


_MASK_DTYPES = tuple(d for d in (torch.int32, getattr(torch, "uint32", None)) if d is not None)


def _check_buf(name, t, shape, dtypes, device):
    """A caller-supplied buffer must match what the kernels write or read: the
    library only sees its pointer, so a smaller or strided buffer would be
    accessed out of bounds on the device."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    if (tuple(t.shape) != tuple(shape) or t.dtype not in dtypes or t.device != device
            or not t.is_contiguous()):
        raise ValueError(
            f"{name} must be a contiguous {'/'.join(str(d) for d in dtypes)} tensor of shape "
            f"{tuple(shape)} on {device}; got {t.dtype} {tuple(t.shape)} on {t.device}"
            f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _check_workspace(ws, device):
    if (not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or ws.dim() != 1
            or ws.device != device or not ws.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous 1-D uint8 tensor on {device}")


class FwdResult(NamedTuple):
    out: torch.Tensor
    tau: torch.Tensor
    mask: torch.Tensor
    workspace: torch.Tensor
    tau_trace: Optional[torch.Tensor]


def alloc_workspace(B, H, N, D, block=128, causal=True, device="cuda"):
    return torch.empty(workspace_size(B, H, N, D, block, causal), dtype=torch.uint8, device=device)


def default_max_iter(alpha: float) -> int:
    """Refinement cap: the closed forms (alpha 1.5 and 2) certify exactness within
    one or two steps; the power path for other alpha stops on a tolerance."""
    return 4 if float(alpha) in (1.5, 2.0) else 12


def entmax_attn_fwd(q, k, v, alpha: float = 1.5, causal: bool = True, block: int = 128,
                    max_iter=None, *, out=None, tau=None, mask=None, workspace=None,
                    trace: bool = False, stream=None) -> FwdResult:
    """alpha-entmax attention forward through ``entmax_attn_fwd``."""
    _check_qkv(q, k, v)
    max_iter = default_max_iter(alpha) if max_iter is None else int(max_iter)
    B, H, N, D = q.shape
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    tau = torch.empty((B, H, N), dtype=torch.float32, device=dev) if tau is None else tau
    mrows = (N + block - 1) // block
    if mask is None:
        mask = torch.empty((B, H, mrows, mask_words(N, block)), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, D, block, causal, dev)
    trace_t = (torch.empty((max_iter + 1, B, H, N), dtype=torch.float32, device=dev)
               if trace else None)
    _check_buf("out", out, q.shape, q.dtype, dev)
    _check_buf("tau", tau, (B, H, N), torch.float32, dev)
    _check_buf("mask", mask, (B, H, mrows, mask_words(N, block)), _MASK_DTYPES, dev)
    _check_workspace(workspace, dev)
    rc = _lib().entmax_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), B, H, N, D, DTYPE_CODES[q.dtype], float(alpha),
        int(bool(causal)), int(block), int(max_iter), _ptr(out), _ptr(tau), _ptr(mask),
        _ptr(trace_t), _ptr(workspace), workspace.numel(), _stream_ptr(stream, dev))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_fwd")
    return FwdResult(out, tau, mask, workspace, trace_t)


def entmax_attn_bwd(q, k, v, dout, tau, mask, alpha: float = 1.5, causal: bool = True,
                    block: int = 128, *, dq=None, dk=None, dv=None, workspace=None,
                    stream=None):
    """alpha-entmax attention backward through ``entmax_attn_bwd``; returns (dq, dk, dv).

    For bf16 inputs ``workspace`` must be the one the forward of the same
    inputs wrote (``Forward.workspace``): it carries the forward's g-weighted
    means of v and its fp16 copy of v."""
    _check_qkv(q, k, v, dout)
    B, H, N, D = q.shape
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        if q.dtype == torch.bfloat16:
            raise ValueError("entmax_attn_bwd: bf16 needs the forward's workspace")
        workspace = alloc_workspace(B, H, N, D, block, causal, dev)
    mrows = (N + block - 1) // block
    _check_buf("tau", tau, (B, H, N), torch.float32, dev)
    _check_buf("mask", mask, (B, H, mrows, mask_words(N, block)), _MASK_DTYPES, dev)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_buf(name, t, q.shape, q.dtype, dev)
    _check_workspace(workspace, dev)
    rc = _lib().entmax_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(tau), _ptr(mask), B, H, N, D,
        DTYPE_CODES[q.dtype], float(alpha), int(bool(causal)), int(block), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(workspace), workspace.numel(), _stream_ptr(stream, dev))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_bwd")
    return dq, dk, dv


def status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the device status bits (ST_*)."""
    word = ctypes.c_uint32(0)
    rc = _lib().entmax_attn_status(_ptr(workspace), _stream_ptr(stream, workspace.device),
                                   ctypes.byref(word))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_status")
    return int(word.value)


def noalloc_status(device=None, stream=None) -> int:
    """Synchronise the stream and return the status bits (ST_*) of the last
    entmax_attn_fwd_noalloc call on ``device`` (default: the current one)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    word = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        rc = _lib().entmax_attn_noalloc_status(_stream_ptr(stream, dev), ctypes.byref(word))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_noalloc_status")
    return int(word.value)


def counters(workspace: torch.Tensor, stream=None) -> dict:
    """Synchronise the stream and return the work counters (COUNTER_NAMES)."""
    arr = (ctypes.c_ulonglong * len(COUNTER_NAMES))()
    rc = _lib().entmax_attn_counters(_ptr(workspace), _stream_ptr(stream, workspace.device), arr,
                                     len(COUNTER_NAMES))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_counters")
    return dict(zip(COUNTER_NAMES, (int(x) for x in arr)))


def profile(enable: bool) -> None:
    """Turn per-kernel CUDA-event recording on or off for this thread."""
    rc = _lib().entmax_attn_profile(int(bool(enable)))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_profile")


def profile_read() -> dict:
    """Per-kernel milliseconds of this thread's last recorded fwd / bwd calls."""
    arr = (ctypes.c_float * len(PHASE_NAMES))()
    rc = _lib().entmax_attn_profile_read(arr, len(PHASE_NAMES))
    if rc != OK:
        raise EntmaxError(rc, "entmax_attn_profile_read")
    return dict(zip(PHASE_NAMES, (float(x) for x in arr)))


class EntmaxAttention(torch.autograd.Function):
    """autograd wrapper: O = entmax_attention(q, k, v); backward through the library."""

    @staticmethod
    def forward(ctx, q, k, v, alpha=1.5, causal=True, block=128, max_iter=None):
        r = entmax_attn_fwd(q, k, v, alpha, causal, block, max_iter)
        ctx.save_for_backward(q, k, v, r.tau, r.mask, r.workspace)
        ctx.cfg = (alpha, causal, block)
        return r.out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, tau, mask, ws = ctx.saved_tensors
        alpha, causal, block = ctx.cfg
        dq, dk, dv = entmax_attn_bwd(q, k, v, dout.contiguous(), tau, mask, alpha, causal, block,
                                     workspace=ws)
        return dq, dk, dv, None, None, None, None


def entmax_attention(q, k, v, alpha=1.5, causal=True, block=128, max_iter=None):
    return EntmaxAttention.apply(q, k, v, alpha, causal, block, max_iter)


# ------------------------------------------------------------------ DashAttention router
class RouteResult(NamedTuple):
    wbar: torch.Tensor        # float32 [B, Hkv, N, C]
    row_mask: torch.Tensor    # int32 (uint32 bits) [B, Hkv, N, ceil(C / 32)]
    block_mask: torch.Tensor  # int32 (uint32 bits) [B, Hkv, ceil(N / 128), ceil(C / 32)]
    workspace: torch.Tensor


def dash_route(q, k, chunk: int, gamma: float, alpha: float = 1.5, max_iter=None, *,
               stream=None) -> RouteResult:
    """DashAttention stages 0-1 through ``dash_route_fwd``: chunk-mean summaries
    of k, alpha-entmax routing of every query row over the complete chunks
    before its own, averaged over the query heads of each KV head (GQA).
    q: [B, Hq, N, D] bf16, k: [B, Hkv, N, D] bf16, Hq a multiple of Hkv."""
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise TypeError("dash_route: q and k must be bfloat16")
    if int(chunk) < 1:
        raise ValueError("dash_route: chunk must be at least 1")
    if not (q.is_cuda and k.is_cuda and q.is_contiguous() and k.is_contiguous()):
        raise ValueError("dash_route: q and k must be contiguous CUDA tensors")
    if q.device != k.device:
        raise ValueError("dash_route: q and k must live on one CUDA device")
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, D):
        raise ValueError("dash_route: k must be [B, Hkv, N, D] with q's B, N and D")
    max_iter = default_max_iter(alpha) if max_iter is None else int(max_iter)
    dev = q.device
    C = N // int(chunk)
    W = (C + 31) // 32
    wbar = torch.empty((B, Hkv, N, C), dtype=torch.float32, device=dev)
    row_mask = torch.empty((B, Hkv, N, W), dtype=torch.int32, device=dev)
    block_mask = torch.empty((B, Hkv, (N + 127) // 128, W), dtype=torch.int32, device=dev)
    ws_bytes = int(_lib().dash_route_workspace_size(B, Hq, Hkv, N, D, int(chunk)))
    workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    rc = _lib().dash_route_fwd(
        _ptr(q), _ptr(k), B, Hq, Hkv, N, D, int(chunk), float(gamma), float(alpha), max_iter,
        _ptr(wbar), _ptr(row_mask), _ptr(block_mask), _ptr(workspace), ws_bytes,
        _stream_ptr(stream, dev))
    if rc != OK:
        raise EntmaxError(rc, "dash_route_fwd")
    return RouteResult(wbar, row_mask, block_mask, workspace)
