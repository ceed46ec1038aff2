"""Python binding of the C ABI in ``include/fa2.h`` (ctypes; marshalling only).

Every step of the attention forward runs in the CUDA kernels of libfa2.so;
this module only checks tensor properties, allocates outputs with torch and
passes raw pointers and the current stream.  There is no fallback: if the
library is missing or a call fails, a RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
#: The in-tree build; FA2_LIBRARY may name another build of the same sources.
LIB_PATH = os.environ.get("FA2_LIBRARY") or os.path.join(_PKG_DIR, "libfa2.so")

FA2_OK, FA2_ERR_INVALID_ARG, FA2_ERR_UNSUPPORTED, FA2_ERR_CUDA, FA2_ERR_TIMEOUT = range(5)

#: Every symbol the header declares.
EXPORTS = ("fa2_fwd", "fa2_fwd_host", "fa2_fwd_host_workspace_bytes", "fa2_sync_status",
           "fa2_fwd_inject_timeout", "fa2_fwd_splitkv", "fa2_fwd_splitkv_inject_timeout", "fa2_fwd_splitkv_splits",
           "fa2_fwd_splitkv_workspace_bytes", "fa2_fwd_splitkv_static", "fa2_bwd", "fa2_bwd_workspace_bytes",
           "fa2_bwd_inject_timeout", "fa2_strerror", "fa2_last_error_detail", "fa2_version")

_lib = None

_vp, _int, _float = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_FWD_ARGS = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _float]


def load() -> ctypes.CDLL:
    """Load libfa2.so (built in-tree); raise if it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_45_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.fa2_fwd.argtypes = _FWD_ARGS + [_vp]
    lib.fa2_fwd.restype = _int
    lib.fa2_fwd_host.argtypes = _FWD_ARGS + [_vp, ctypes.c_size_t, _vp]
    lib.fa2_fwd_host.restype = _int
    lib.fa2_fwd_host_workspace_bytes.argtypes = [_int, _int, _int, _int]
    lib.fa2_fwd_host_workspace_bytes.restype = ctypes.c_size_t
    lib.fa2_sync_status.argtypes = [_vp]
    lib.fa2_sync_status.restype = _int
    lib.fa2_fwd_inject_timeout.argtypes = _FWD_ARGS + [ctypes.c_ulonglong, _vp]
    lib.fa2_fwd_inject_timeout.restype = _int
    lib.fa2_fwd_splitkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _float, _int, _vp,
                                    ctypes.c_size_t, _vp]
    lib.fa2_fwd_splitkv.restype = _int
    lib.fa2_fwd_splitkv_inject_timeout.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                                                   _float, _int, _vp, ctypes.c_size_t, ctypes.c_ulonglong, _vp]
    lib.fa2_fwd_splitkv_inject_timeout.restype = _int
    lib.fa2_fwd_splitkv_splits.argtypes = [_int] * 6
    lib.fa2_fwd_splitkv_splits.restype = _int
    lib.fa2_fwd_splitkv_workspace_bytes.argtypes = [_int] * 6
    lib.fa2_fwd_splitkv_workspace_bytes.restype = ctypes.c_size_t
    lib.fa2_fwd_splitkv_static.argtypes = [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _float,
                                           _int, _vp]
    lib.fa2_fwd_splitkv_static.restype = _int
    lib.fa2_bwd.argtypes = [_vp] * 9 + [_int] * 5 + [_float, _vp, ctypes.c_size_t, _vp]
    lib.fa2_bwd.restype = _int
    lib.fa2_bwd_workspace_bytes.argtypes = [_int] * 4
    lib.fa2_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa2_bwd_inject_timeout.argtypes = [_vp] * 9 + [_int] * 5 + [_float, _vp, ctypes.c_size_t, _int,
                                                                     ctypes.c_ulonglong, _vp]
    lib.fa2_bwd_inject_timeout.restype = _int
    lib.fa2_strerror.argtypes = [_int]
    lib.fa2_strerror.restype = ctypes.c_char_p
    lib.fa2_last_error_detail.argtypes = []
    lib.fa2_last_error_detail.restype = ctypes.c_char_p
    lib.fa2_version.argtypes = []
    lib.fa2_version.restype = _int
    _lib = lib
    return lib


class FA2Error(RuntimeError):
    def __init__(self, status: int, lib):
        self.status = status
        msg = lib.fa2_strerror(status).decode()
        detail = lib.fa2_last_error_detail().decode()
        super().__init__(f"fa2 status {status} ({msg}){': ' + detail if detail else ''}")


def _check(status: int, lib) -> None:
    if status != FA2_OK:
        raise FA2Error(status, lib)


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check_qkv(q, k, v, device: str):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, N, d], got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device.type != device:
            raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share the shape [B, H, N, d]")


def _check_buffer(name: str, t: torch.Tensor, shape, dtype, device: str) -> None:
    """A caller-provided output or workspace buffer the kernels will write."""
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _check_workspace(workspace: torch.Tensor, need: int) -> None:
    _check_buffer("workspace", workspace, None, torch.uint8, "cuda")
    if workspace.numel() < need:
        raise ValueError(f"workspace needs {need} bytes, got {workspace.numel()}")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: float | None = None,
        out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Exact attention forward on CUDA tensors.  Returns (O bf16, LSE fp32).

    Asynchronous on ``stream`` (default: torch's current stream).
    """
    lib = load()
    _check_qkv(q, k, v, "cuda")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, torch.bfloat16, "cuda")
    _check_buffer("lse", lse, (B, H, N), torch.float32, "cuda")
    st = lib.fa2_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     B, H, N, d, int(bool(causal)), float(scale), _stream_handle(stream))
    _check(st, lib)
    return out, lse


def sync_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel reported a timed-out wait."""
    lib = load()
    _check(lib.fa2_sync_status(_stream_handle(stream)), lib)


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa2_fwd_host_workspace_bytes(B, H, N, d))


def fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, scale: float | None = None,
             out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, stream=None):
    """End-to-end call on HOST tensors (pinned for full copy bandwidth).

    Copies q, k, v to the device, runs the kernel, copies O and LSE back and
    returns after they have landed (the library overlaps the copies and the
    kernels over chunks of heads).  Outputs are allocated pinned when q is.
    ``workspace`` is an optional uint8 CUDA tensor of at least
    :func:`workspace_bytes` bytes, reused across calls.
    """
    lib = load()
    _check_qkv(q, k, v, "cpu")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    _check_workspace(workspace, need)
    pinned = q.is_pinned()
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=pinned)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=pinned)
    _check_buffer("out", out, q.shape, torch.bfloat16, "cpu")
    _check_buffer("lse", lse, (B, H, N), torch.float32, "cpu")
    st = lib.fa2_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, H, N, d, int(bool(causal)), float(scale), workspace.data_ptr(),
                          workspace.numel(), _stream_handle(stream))
    _check(st, lib)
    return out, lse


def fwd_inject_timeout(q, k, v, causal=False, scale=None, timeout_ns: int = 50_000_000, stream=None):
    """Failure-path test hook: run the kernel with the Q-tile load withheld.

    Returns the status of :func:`sync_status` (expected FA2_ERR_TIMEOUT).
    """
    lib = load()
    _check_qkv(q, k, v, "cuda")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    h = _stream_handle(stream)
    st = lib.fa2_fwd_inject_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                    B, H, N, d, int(bool(causal)), float(scale), int(timeout_ns), h)
    _check(st, lib)
    return lib.fa2_sync_status(h)


def _check_q_kv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be on cuda, got {t.device}")
    B, H, Nq, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != H or k.shape[3] != d:
        raise ValueError("need q [B, H, Nq, d] and k, v [B, H, Nk, d]")
    if Nq > k.shape[2]:
        raise ValueError("need Nq <= Nk")


def splitkv_splits(B: int, H: int, Nq: int, Nk: int, d: int, n_splits: int = 0) -> int:
    """Number of key ranges fwd_splitkv uses for this shape (0 on bad sizes)."""
    return int(load().fa2_fwd_splitkv_splits(B, H, Nq, Nk, d, n_splits))


def splitkv_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int, n_splits: int = 0) -> int:
    return int(load().fa2_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, n_splits))


def fwd_splitkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                scale: float | None = None, n_splits: int = 0, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Exact attention of Nq queries (the last Nq positions) against Nk >= Nq keys.

    q: [B, H, Nq, d]; k, v: [B, H, Nk, d] (bf16, CUDA, contiguous).  The keys
    are split into ``n_splits`` ranges (0 = chosen by the library) processed
    by separate CTAs, then merged.  ``workspace`` is an optional uint8 CUDA
    tensor of at least :func:`splitkv_workspace_bytes` bytes, 256-byte aligned
    (none is needed, and the merge is skipped, when one range is used).
    Returns (O bf16 [B, H, Nq, d], LSE fp32 [B, H, Nq]).
    """
    lib = load()
    _check_q_kv(q, k, v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = splitkv_workspace_bytes(B, H, Nq, Nk, d, n_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _check_workspace(workspace, need)
    ws_ptr, ws_len = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (None, 0)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, torch.bfloat16, "cuda")
    _check_buffer("lse", lse, (B, H, Nq), torch.float32, "cuda")
    st = lib.fa2_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, H, Nq, Nk, d, int(bool(causal)), float(scale), int(n_splits),
                             ws_ptr, ws_len, _stream_handle(stream))
    _check(st, lib)
    return out, lse


def fwd_splitkv_inject_timeout(q, k, v, causal=False, scale=None, n_splits: int = 0, timeout_ns: int = 50_000_000,
                               stream=None):
    """Failure-path test hook of :func:`fwd_splitkv`: the range kernel runs
    with its query load withheld (the merge still runs when there are two or
    more key ranges).  Returns the status of :func:`sync_status` (expected
    FA2_ERR_TIMEOUT)."""
    lib = load()
    _check_q_kv(q, k, v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = splitkv_workspace_bytes(B, H, Nq, Nk, d, n_splits)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if need > 0 else None
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    h = _stream_handle(stream)
    st = lib.fa2_fwd_splitkv_inject_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                            lse.data_ptr(), B, H, Nq, Nk, d, int(bool(causal)), float(scale),
                                            int(n_splits), ws.data_ptr() if ws is not None else None,
                                            need, int(timeout_ns), h)
    _check(st, lib)
    return lib.fa2_sync_status(h)


#: Bytes of the library's own scratch array used by :func:`fwd_splitkv_static`.
SPLITKV_STATIC_SCRATCH_BYTES = 16 << 20


def fwd_splitkv_static(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                       scale: float | None = None, n_splits: int = 0, out: torch.Tensor | None = None,
                       lse: torch.Tensor | None = None, stream=None):
    """:func:`fwd_splitkv` with the partials in the library's fixed 16 MiB
    scratch array instead of a caller workspace.

    For callers that may not allocate device memory themselves.  The C entry
    point allocates nothing; this wrapper only allocates ``out`` and ``lse``
    when they are not given.  Calls that overlap on the GPU race on the shared
    scratch; the first call on a device should precede any stream capture.
    """
    lib = load()
    _check_q_kv(q, k, v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.shape, torch.bfloat16, "cuda")
    _check_buffer("lse", lse, (B, H, Nq), torch.float32, "cuda")
    st = lib.fa2_fwd_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                    B, H, Nq, Nk, d, int(bool(causal)), float(scale), int(n_splits),
                                    _stream_handle(stream))
    _check(st, lib)
    return out, lse


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa2_bwd_workspace_bytes(B, H, N, d))


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
        causal: bool = False, scale: float | None = None, dq: torch.Tensor | None = None,
        dk: torch.Tensor | None = None, dv: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
        stream=None):
    """Gradients (dQ, dK, dV) of exact attention on CUDA tensors.

    ``o`` and ``lse`` are the forward's outputs for the same q, k, v, causal
    and scale; ``dout`` is the upstream gradient of O.  Asynchronous on
    ``stream``.  ``workspace`` is an optional uint8 CUDA tensor of at least
    :func:`bwd_workspace_bytes` bytes, 256-byte aligned.
    """
    lib = load()
    _check_qkv(q, k, v, "cuda")
    _check_qkv(o, dout, q, "cuda")
    B, H, N, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, N] tensor")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = bwd_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, need)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_buffer(name, t, q.shape, torch.bfloat16, "cuda")
    st = lib.fa2_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                     dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                     workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check(st, lib)
    return dq, dk, dv


def bwd_inject_timeout(q, k, v, o, lse, dout, kernel: int, causal: bool = False, scale=None,
                       timeout_ns: int = 50_000_000, stream=None):
    """Failure-path test hook of :func:`bwd`: ``kernel`` 0 withholds the dQ
    kernel's Q/dO load, 1 the dK/dV kernel's K/V load.  Returns the status of
    :func:`sync_status` (expected FA2_ERR_TIMEOUT)."""
    lib = load()
    _check_qkv(q, k, v, "cuda")
    _check_qkv(o, dout, q, "cuda")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    h = _stream_handle(stream)
    st = lib.fa2_bwd_inject_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                    lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                    int(bool(causal)), float(scale), ws.data_ptr(), ws.numel(), int(kernel),
                                    int(timeout_ns), h)
    _check(st, lib)
    return lib.fa2_sync_status(h)
