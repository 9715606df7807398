"""Thin Python binding of liblongnet (include/longnet.h) over ctypes.

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  If the in-tree
library is missing, loading raises: there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblongnet.so")

LONGNET_OK = 0
LONGNET_ERR_INVALID_ARG = -1
LONGNET_ERR_UNSUPPORTED = -2
LONGNET_ERR_MISALIGNED = -3
LONGNET_ERR_CUDA = -4
LONGNET_ERR_DEVICE_TIMEOUT = -5
LONGNET_ERR_DEVICE_BOUNDS = -6
LONGNET_ERR_NO_DEVICE = -7
LONGNET_ERR_SCRATCH_LIMIT = -8
LONGNET_NOALLOC_SCRATCH_BYTES = 32 << 20
LONGNET_MAX_PATTERNS = 16

LONGNET_DTYPE_F32 = 0
LONGNET_DTYPE_BF16 = 1
LONGNET_DTYPE_F16 = 2
LONGNET_FLAG_QK_NORM = 1
LONGNET_FLAG_XPOS = 2

LONGNET_IMPL_AUTO = 0
LONGNET_IMPL_SIMT = 1
LONGNET_IMPL_TCGEN05 = 2
LONGNET_IMPL_SMALLSEG = 3
LONGNET_IMPL_TILES = 4
LONGNET_IMPL_PATTERNS = 5

# Every symbol include/longnet.h declares, with its ctypes signature.
_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_i64p = ctypes.POINTER(ctypes.c_int64)
SIGNATURES = {
    "longnet_dilated_attn_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                                ctypes.c_int, _i64p, _i64p, ctypes.c_int,
                                                ctypes.c_int, _vp]),
    "longnet_dilated_attn_fwd_impl": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                                     _i64, ctypes.c_int, _i64p, _i64p,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     _vp]),
    "longnet_dilated_attn_fwd_ex": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                                   _i64, ctypes.c_int, _i64p, _i64p,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, _vp]),
    "longnet_dilated_attn_fwd_part": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                                     _i64, ctypes.c_int, _i64p, _i64p,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, _i64, _i64, _i64, _i64, _vp]),
    "longnet_dilated_attn_fwd_host": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                     _i64, _i64, _i64, _i64, ctypes.c_int, _i64p, _i64p,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     _i64, _vp]),
    "longnet_fwd_workspace_bytes": (ctypes.c_int64, [_i64, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int]),
    "longnet_dilated_attn_fwd_ws": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                                   ctypes.c_int, _i64p, _i64p, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _i64,
                                                   _vp]),
    "longnet_dilated_attn_fwd_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                                        ctypes.c_int, _i64p, _i64p, ctypes.c_int,
                                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]),
    "longnet_gather_rows": (ctypes.c_int, [_vp, _i64, _vp, _i64, _vp, _i64, _vp]),
    "longnet_scatter_rows": (ctypes.c_int, [_vp, _i64, _vp, _vp, _i64, _i64, _vp]),
    "longnet_dilated_attn_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                _i64, _i64, _i64, _i64, ctypes.c_int, _i64p,
                                                _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, _vp]),
    "longnet_dilated_attn_bwd_ws": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                   _i64, _i64, _i64, _i64, ctypes.c_int, _i64p,
                                                   _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, _vp, _i64, _vp]),
    "longnet_select_impl": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.c_int, _i64p, _i64p,
                                           ctypes.c_int, ctypes.c_int]),
    "longnet_last_device_status": (ctypes.c_int, [_vp]),
    "longnet_watchdog_selftest": (ctypes.c_int, [_i64, _vp]),
    "longnet_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "longnet_version": (ctypes.c_char_p, []),
}

_lib = None


class LongNetError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} (code {code})")
        self.code = code


def load_library(path: str = LIB_PATH):
    """Load liblongnet.so; raises if it was not built (no fallback)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"liblongnet.so not built at {path}; run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().longnet_status_string(int(code)).decode()


def version() -> str:
    return load_library().longnet_version().decode()


def _patterns(patterns: Sequence[Tuple[int, int]]):
    n = len(patterns)
    w = (ctypes.c_int64 * max(n, 1))(*[int(p[0]) for p in patterns])
    r = (ctypes.c_int64 * max(n, 1))(*[int(p[1]) for p in patterns])
    return n, w, r


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LONGNET_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return LONGNET_DTYPE_BF16
    if t.dtype == torch.float16:
        return LONGNET_DTYPE_F16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


def longnet_dilated_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             out: torch.Tensor, lse: torch.Tensor | None,
                             patterns: Sequence[Tuple[int, int]], causal: bool = True,
                             impl: int = LONGNET_IMPL_AUTO, stream=None, qk_norm: bool = False) -> None:
    """Enqueue the forward on `stream` (default: torch's current stream).

    q, k, v, out: contiguous CUDA tensors [B, N, H, D] of one dtype (fp32/bf16/fp16);
    lse: contiguous fp32 [B, H, N] or None.  qk_norm: scale q and k rows to unit
    L2 norm first (LONGNET_FLAG_QK_NORM).  Raises LongNetError on a non-zero
    status.
    """
    lib = load_library()
    for t in (q, k, v, out):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("q, k, v, out must be contiguous CUDA tensors")
    if lse is not None and not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor")
    B, N, H, D = q.shape
    for t in (k, v, out):
        if tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out must share shape and dtype")
    if lse is not None and tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_fwd_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        None if lse is None else lse.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), LONGNET_FLAG_QK_NORM if qk_norm else 0, int(impl), _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_fwd")


def _flags(qk_norm: bool, xpos: bool) -> int:
    return (LONGNET_FLAG_QK_NORM if qk_norm else 0) | (LONGNET_FLAG_XPOS if xpos else 0)


def longnet_fwd_workspace_bytes(B: int, N: int, H: int, D: int, dtype: torch.dtype, qk_norm: bool = False,
                                xpos: bool = False) -> int:
    """Device workspace bytes longnet_dilated_attn_fwd_ws needs (0 without options)."""
    code = {torch.float32: LONGNET_DTYPE_F32, torch.bfloat16: LONGNET_DTYPE_BF16,
            torch.float16: LONGNET_DTYPE_F16}[dtype]
    n = load_library().longnet_fwd_workspace_bytes(B, N, H, D, code, _flags(qk_norm, xpos))
    if n < 0:
        raise LongNetError(n, "longnet_fwd_workspace_bytes")
    return int(n)


def longnet_dilated_attn_fwd_ws(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                out: torch.Tensor, lse: torch.Tensor | None,
                                patterns: Sequence[Tuple[int, int]], causal: bool,
                                workspace: torch.Tensor | None, impl: int = LONGNET_IMPL_AUTO,
                                stream=None, qk_norm: bool = False, xpos: bool = False) -> None:
    """Enqueue the prologue (qk_norm, then XPOS) into `workspace` (a CUDA
    tensor of at least longnet_fwd_workspace_bytes bytes, 256-byte aligned)
    and the forward on its result.  Tensors as in longnet_dilated_attn_fwd.
    Raises LongNetError on a non-zero status."""
    lib = load_library()
    B, N, H, D = q.shape
    for t in (q, k, v, out):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out must be contiguous CUDA tensors of one shape and dtype")
    if lse is not None and not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32
                                and tuple(lse.shape) == (B, H, N)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    if workspace is not None and not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_ptr = None if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_fwd_ws(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        None if lse is None else lse.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), _flags(qk_norm, xpos), int(impl), ws_ptr, ws_bytes, _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_fwd_ws")


def longnet_dilated_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                     out: torch.Tensor, lse: torch.Tensor | None,
                                     patterns: Sequence[Tuple[int, int]], causal: bool,
                                     impl: int = LONGNET_IMPL_AUTO, stream=None, qk_norm: bool = False,
                                     xpos: bool = False) -> None:
    """longnet_dilated_attn_fwd_ws with the library's fixed device scratch
    (LONGNET_NOALLOC_SCRATCH_BYTES per device) as the workspace: nothing is
    allocated.  Calls that may run at the same time on one device race on
    that scratch.  Raises LongNetError on a non-zero status
    (LONGNET_ERR_SCRATCH_LIMIT when the problem needs more scratch)."""
    lib = load_library()
    B, N, H, D = q.shape
    for t in (q, k, v, out):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out must be contiguous CUDA tensors of one shape and dtype")
    if lse is not None and not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32
                                and tuple(lse.shape) == (B, H, N)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        None if lse is None else lse.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), _flags(qk_norm, xpos), int(impl), _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_fwd_noalloc")


def longnet_dilated_attn_fwd_part(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  out: torch.Tensor, lse: torch.Tensor | None,
                                  patterns: Sequence[Tuple[int, int]], causal: bool,
                                  q_range: Tuple[int, int], h_range: Tuple[int, int] | None = None,
                                  impl: int = LONGNET_IMPL_AUTO, stream=None,
                                  qk_norm: bool = False) -> None:
    """Enqueue the forward for part of the output: positions q_range = (begin,
    end) and heads h_range (default all) of out and lse; the rest of out and
    lse is left as it is.  Tensors as in longnet_dilated_attn_fwd (full
    length).  Raises LongNetError on a non-zero status."""
    lib = load_library()
    B, N, H, D = q.shape
    for t in (q, k, v, out):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out must be contiguous CUDA tensors of one shape and dtype")
    if lse is not None and not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32
                                and tuple(lse.shape) == (B, H, N)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    h0, h1 = (0, H) if h_range is None else h_range
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_fwd_part(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
        None if lse is None else lse.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), LONGNET_FLAG_QK_NORM if qk_norm else 0, int(impl), int(q_range[0]),
        int(q_range[1]), int(h0), int(h1), _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_fwd_part")


def longnet_dilated_attn_fwd_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                                  out_host: torch.Tensor, lse_host: torch.Tensor | None,
                                  q_dev: torch.Tensor, k_dev: torch.Tensor, v_dev: torch.Tensor,
                                  out_dev: torch.Tensor, lse_dev: torch.Tensor | None,
                                  patterns: Sequence[Tuple[int, int]], causal: bool = True,
                                  impl: int = LONGNET_IMPL_AUTO, stream=None, qk_norm: bool = False,
                                  pieces: int = 0) -> None:
    """Enqueue the forward on host tensors (pinned for asynchronous copies):
    the work is cut into `pieces` ranges (0: the library's choice) of batches
    (B >= 2), heads (B = 1 with H >= 4, or full attention) or positions
    (B = 1, H < 4, causal), and each piece's copy in, attention and copy out
    overlap with its neighbours'.
    The *_dev tensors are the caller's device staging of the same shapes.
    Synchronise `stream` before reading out_host / lse_host.  Raises
    LongNetError on a non-zero status."""
    lib = load_library()
    B, N, H, D = q_host.shape
    for t in (q_host, k_host, v_host, out_host):
        if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, N, H, D) or t.dtype != q_host.dtype:
            raise ValueError("q_host, k_host, v_host, out_host: contiguous host tensors [B, N, H, D] of one dtype")
    for t in (q_dev, k_dev, v_dev, out_dev):
        if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, N, H, D) or t.dtype != q_host.dtype:
            raise ValueError("q_dev, k_dev, v_dev, out_dev: contiguous CUDA tensors of the host tensors' shape")
    for t, want_cuda in ((lse_host, False), (lse_dev, True)):
        if t is not None and (t.is_cuda != want_cuda or t.dtype != torch.float32 or not t.is_contiguous()
                              or tuple(t.shape) != (B, H, N)):
            raise ValueError("lse_host / lse_dev: contiguous fp32 [B, H, N] (host / CUDA)")
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_fwd_host(
        q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), out_host.data_ptr(),
        None if lse_host is None else lse_host.data_ptr(), q_dev.data_ptr(), k_dev.data_ptr(), v_dev.data_ptr(),
        out_dev.data_ptr(), None if lse_dev is None else lse_dev.data_ptr(), B, N, H, D, n, w, r,
        int(bool(causal)), _dtype_code(q_host), LONGNET_FLAG_QK_NORM if qk_norm else 0, int(impl),
        int(pieces), _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_fwd_host")


def _rows_view(t: torch.Tensor, row_elems: int):
    if not (t.is_cuda and t.is_contiguous()) or t.numel() % row_elems != 0:
        raise ValueError("row buffers must be contiguous CUDA tensors of whole rows")
    return t.numel() // row_elems


def longnet_gather_rows(src: torch.Tensor, idx: torch.Tensor, dst: torch.Tensor, row_elems: int,
                        stream=None) -> None:
    """dst row i = src row idx[i] (rows of row_elems elements of src's dtype);
    idx: int64 CUDA tensor.  Raises LongNetError on a non-zero status."""
    if idx.dtype != torch.int64 or not (idx.is_cuda and idx.is_contiguous()):
        raise ValueError("idx must be a contiguous int64 CUDA tensor")
    src_rows, dst_rows = _rows_view(src, row_elems), _rows_view(dst, row_elems)
    if dst_rows != idx.numel() or src.dtype != dst.dtype:
        raise ValueError("dst must hold one row per index, in src's dtype")
    rc = load_library().longnet_gather_rows(src.data_ptr(), src_rows, idx.data_ptr(), idx.numel(),
                                            dst.data_ptr(), row_elems * src.element_size(),
                                            _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_gather_rows")


def longnet_scatter_rows(src: torch.Tensor, idx: torch.Tensor, dst: torch.Tensor, row_elems: int,
                         stream=None) -> None:
    """dst row idx[i] = src row i; idx: int64 CUDA tensor.  Raises
    LongNetError on a non-zero status."""
    if idx.dtype != torch.int64 or not (idx.is_cuda and idx.is_contiguous()):
        raise ValueError("idx must be a contiguous int64 CUDA tensor")
    src_rows, dst_rows = _rows_view(src, row_elems), _rows_view(dst, row_elems)
    if src_rows != idx.numel() or src.dtype != dst.dtype:
        raise ValueError("src must hold one row per index, in dst's dtype")
    rc = load_library().longnet_scatter_rows(src.data_ptr(), idx.numel(), idx.data_ptr(),
                                             dst.data_ptr(), dst_rows, row_elems * src.element_size(),
                                             _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_scatter_rows")


def dilated_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 patterns: Sequence[Tuple[int, int]], causal: bool = True,
                 impl: int = LONGNET_IMPL_AUTO, want_lse: bool = True, stream=None,
                 qk_norm: bool = False, xpos: bool = False):
    """Allocate out (and lse) with torch and run the forward.  Returns (out,
    lse).  The options (qk_norm, xpos) go through the prologue pass, with a
    workspace allocated by torch, so every family (tcgen05 included) runs."""
    B, N, H, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if want_lse else None
    if qk_norm or xpos:
        ws = torch.empty(longnet_fwd_workspace_bytes(B, N, H, D, q.dtype, qk_norm, xpos),
                         dtype=torch.uint8, device=q.device)
        longnet_dilated_attn_fwd_ws(q, k, v, out, lse, patterns, causal, ws, impl, stream, qk_norm, xpos)
    else:
        longnet_dilated_attn_fwd(q, k, v, out, lse, patterns, causal, impl, stream, qk_norm)
    return out, lse


def longnet_dilated_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                             dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor,
                             patterns: Sequence[Tuple[int, int]], causal: bool = True,
                             impl: int = LONGNET_IMPL_AUTO, stream=None,
                             qk_norm: bool = False) -> None:
    """Enqueue the backward on `stream`: dq, dk, dv (fp32) receive the
    gradients of sum(dout * out).  out and lse are the forward's results for
    q, k, v (with the same qk_norm).  q, k, v, out, dout: contiguous CUDA
    [B, N, H, D] of one dtype; dq, dk, dv: contiguous fp32 [B, N, H, D]; lse
    fp32 [B, H, N].  impl: LONGNET_IMPL_AUTO, LONGNET_IMPL_SIMT or
    LONGNET_IMPL_TILES.  Raises LongNetError on a non-zero status."""
    lib = load_library()
    B, N, H, D = q.shape
    for t in (q, k, v, out, dout):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out, dout must be contiguous CUDA tensors of one shape and dtype")
    for t in (dq, dk, dv):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != torch.float32:
            raise ValueError("dq, dk, dv must be contiguous fp32 CUDA tensors [B, N, H, D]")
    if not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32
            and tuple(lse.shape) == (B, H, N)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), LONGNET_FLAG_QK_NORM if qk_norm else 0, int(impl), _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_bwd")


def longnet_dilated_attn_bwd_ws(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                                dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor,
                                patterns: Sequence[Tuple[int, int]], causal: bool,
                                workspace: torch.Tensor | None, impl: int = LONGNET_IMPL_AUTO, stream=None,
                                qk_norm: bool = False, xpos: bool = False) -> None:
    """The backward of longnet_dilated_attn_fwd_ws (out and lse from it, with
    the same options): the prologue into `workspace`, the attention's backward
    on the encoded rows, then dq and dk taken back through XPOS and the norm.
    Tensors as in longnet_dilated_attn_bwd.  Raises LongNetError on a non-zero
    status."""
    lib = load_library()
    B, N, H, D = q.shape
    for t in (q, k, v, out, dout):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != q.dtype:
            raise ValueError("q, k, v, out, dout must be contiguous CUDA tensors of one shape and dtype")
    for t in (dq, dk, dv):
        if not (t.is_cuda and t.is_contiguous()) or tuple(t.shape) != (B, N, H, D) or t.dtype != torch.float32:
            raise ValueError("dq, dk, dv must be contiguous fp32 CUDA tensors [B, N, H, D]")
    if not (lse.is_cuda and lse.is_contiguous() and lse.dtype == torch.float32
            and tuple(lse.shape) == (B, H, N)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    if workspace is not None and not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_ptr = None if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    n, w, r = _patterns(patterns)
    rc = lib.longnet_dilated_attn_bwd_ws(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, D, n, w, r, int(bool(causal)),
        _dtype_code(q), _flags(qk_norm, xpos), int(impl), ws_ptr, ws_bytes, _stream_handle(stream))
    if rc != LONGNET_OK:
        raise LongNetError(rc, "longnet_dilated_attn_bwd_ws")


def dilated_attn_bwd(q, k, v, out, lse, dout, patterns, causal: bool = True,
                     impl: int = LONGNET_IMPL_AUTO, stream=None, qk_norm: bool = False, xpos: bool = False):
    """Allocate fp32 dq, dk, dv (and, with options, the workspace) with torch
    and run the backward matching dilated_attn.  Returns (dq, dk, dv)."""
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(3))
    if qk_norm or xpos:
        B, N, H, D = q.shape
        ws = torch.empty(longnet_fwd_workspace_bytes(B, N, H, D, q.dtype, qk_norm, xpos), dtype=torch.uint8,
                         device=q.device)
        longnet_dilated_attn_bwd_ws(q, k, v, out, lse, dout.contiguous(), dq, dk, dv, patterns, causal, ws,
                                    impl, stream, qk_norm, xpos)
    else:
        longnet_dilated_attn_bwd(q, k, v, out, lse, dout.contiguous(), dq, dk, dv, patterns, causal, impl,
                                 stream)
    return dq, dk, dv


class DilatedAttnFunction(torch.autograd.Function):
    """The forward and backward entry points as one torch autograd op."""

    @staticmethod
    def forward(ctx, q, k, v, patterns, causal, qk_norm=False, xpos=False):
        out, lse = dilated_attn(q, k, v, patterns, causal, qk_norm=qk_norm, xpos=xpos)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.patterns, ctx.causal, ctx.qk_norm, ctx.xpos = list(patterns), causal, qk_norm, xpos
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = dilated_attn_bwd(q, k, v, out, lse, dout.to(q.dtype), ctx.patterns, ctx.causal,
                                      qk_norm=ctx.qk_norm, xpos=ctx.xpos)
        # autograd wants each gradient in its input's dtype
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None


def dilated_attention(q, k, v, patterns, causal: bool = True, qk_norm: bool = False, xpos: bool = False):
    """Differentiable forward: out [B, N, H, D], gradients through the backward."""
    return DilatedAttnFunction.apply(q, k, v, patterns, causal, qk_norm, xpos)


def longnet_select_impl(B: int, N: int, H: int, D: int, patterns, causal: bool, dtype) -> int:
    """Kernel family AUTO would use (>= 1) or a negative status (host only)."""
    n, w, r = _patterns(patterns)
    code = dtype if isinstance(dtype, int) else {torch.float32: LONGNET_DTYPE_F32, torch.bfloat16: LONGNET_DTYPE_BF16,
                                                 torch.float16: LONGNET_DTYPE_F16}[dtype]
    return int(load_library().longnet_select_impl(B, N, H, D, n, w, r, int(bool(causal)), code))


def longnet_last_device_status(stream=None) -> int:
    """Synchronise the stream, then read and clear this device's status word."""
    return int(load_library().longnet_last_device_status(_stream_handle(stream)))


def longnet_watchdog_selftest(limit_ns: int = 1_000_000, stream=None) -> int:
    """Launch the kernel whose barrier wait must run out (see longnet.h)."""
    return int(load_library().longnet_watchdog_selftest(int(limit_ns), _stream_handle(stream)))
