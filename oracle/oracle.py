"""ctypes wrapper around oracle.c (TEST INFRASTRUCTURE ONLY).

The C file holds the arithmetic; this wrapper only builds it with gcc, widens
inputs to float64 and passes pointers.  Nothing here is imported by the
product path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str | None = None):
    """Load liboracle.so (or another build of oracle.c given by path)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build_oracle())
    i64, dp, ip = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)
    lib.oracle_dilated_attn_fp64.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64,
                                             ctypes.c_int, ip, ip, ctypes.c_int]
    lib.oracle_dilated_attn_fp64.restype = ctypes.c_int
    lib.oracle_dilated_attn_rows_fp64.argtypes = [dp, dp, dp, i64, i64, i64, i64, ctypes.c_int,
                                                  ip, ip, ctypes.c_int, i64, ip, dp, dp]
    lib.oracle_dilated_attn_rows_fp64.restype = ctypes.c_int
    lib.oracle_dilated_attn_bwd_fp64.argtypes = [dp, dp, dp, dp, dp, dp, dp, i64, i64, i64, i64,
                                                 ctypes.c_int, ip, ip, ctypes.c_int]
    lib.oracle_dilated_attn_bwd_fp64.restype = ctypes.c_int
    lib.oracle_dilated_attn_bwd_rows_fp64.argtypes = [dp, dp, dp, dp, i64, i64, i64, i64,
                                                      ctypes.c_int, ip, ip, ctypes.c_int, i64, ip,
                                                      dp, dp, dp]
    lib.oracle_dilated_attn_bwd_rows_fp64.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    """Exact widening to a C-contiguous float64 array (bf16/fp16/fp32 -> fp64 is exact)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t))


def qk_normalize_fp64(x) -> np.ndarray:
    """Rows of x [B, N, H, D] scaled to unit L2 norm over D, x / max(|x|, 1e-12)
    (a zero row stays zero), in fp64.  The reading adopted for the qk_norm
    option of the DilatedAttention module ("LongNet" docs page, usage example):
    the option is named there, not defined; L2 normalisation of every query and
    key row is the plainest reading."""
    x = _f64(x)
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-12)


def xpos_fp64(x, downscale=False) -> np.ndarray:
    """XPOS applied to x [B, N, H, D] (D even) by absolute position n = 0..N-1,
    in fp64.  The use_xpos option is named by "LongNet论文精读" (section
    "Dilated Attention的核心参数解析") without a formula; this is the
    published XPOS definition (Sun et al., "A Length-Extrapolatable
    Transformer"), element pairs (2i, 2i+1):
        theta_i = 10000^(-2i/D)           rotation frequency of pair i
        zeta_i  = (2i + 0.4 D) / (1.4 D)  decay base of pair i
        s(n)    = zeta_i^((n - c) / 512), c = floor(N / 2)
        pair at n -> s(n) * R(n theta_i) (x_2i, x_2i+1)
    with R(a) the rotation by angle a; keys (downscale=True) use 1 / s(n).
    The centring c cancels in every query-key product; it keeps the scales
    near 1."""
    x = _f64(x)
    B, N, H, D = x.shape
    if D % 2:
        raise ValueError("XPOS needs an even head dimension")
    n = np.arange(N, dtype=np.float64)[:, None]            # [N, 1]
    i = np.arange(D // 2, dtype=np.float64)[None, :]       # [1, D/2]
    theta = 10000.0 ** (-2.0 * i / D)
    zeta = (2.0 * i + 0.4 * D) / (1.4 * D)
    s = zeta ** ((n - (N // 2)) / 512.0)                   # [N, D/2]
    if downscale:
        s = 1.0 / s
    ang = n * theta
    cos = (np.cos(ang) * s)[None, :, None, :]
    sin = (np.sin(ang) * s)[None, :, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * cos - x1 * sin
    y[..., 1::2] = x1 * cos + x0 * sin
    return y


def _prologue(q, k, qk_norm, xpos):
    """The input-side options in their order: the norm, then XPOS."""
    if qk_norm:
        q, k = qk_normalize_fp64(q), qk_normalize_fp64(k)
    if xpos:
        q, k = xpos_fp64(q), xpos_fp64(k, downscale=True)
    return q, k


def dilated_attn_fp64(q, k, v, patterns, causal=True, lib=None, qk_norm=False, xpos=False):
    """Full fp64 forward.  q, k, v: [B, N, H, D].  patterns: [(w, r), ...].
    qk_norm: normalise q and k rows first (qk_normalize_fp64); xpos: then
    apply XPOS to them (xpos_fp64).

    Returns (out [B, N, H, D] float64, lse [B, H, N] float64).
    """
    lib = lib or load_library()
    q, k, v = _f64(q), _f64(k), _f64(v)
    q, k = _prologue(q, k, qk_norm, xpos)
    B, N, H, D = q.shape
    w = np.ascontiguousarray([p[0] for p in patterns], dtype=np.int64)
    r = np.ascontiguousarray([p[1] for p in patterns], dtype=np.int64)
    out = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    rc = lib.oracle_dilated_attn_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, N, H, D,
                                      len(patterns), _ptr(w, ctypes.c_int64), _ptr(r, ctypes.c_int64),
                                      int(bool(causal)))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out, lse


def dilated_attn_rows_fp64(q, k, v, patterns, rows_bph, causal=True, lib=None, qk_norm=False,
                           xpos=False):
    """fp64 forward of selected rows only.  rows_bph: int array [n, 3] of (b, pos, h).
    qk_norm, xpos: as in dilated_attn_fp64.

    Returns (out_rows [n, D], lse_rows [n]).
    """
    lib = lib or load_library()
    q, k, v = _f64(q), _f64(k), _f64(v)
    q, k = _prologue(q, k, qk_norm, xpos)
    B, N, H, D = q.shape
    rows = np.ascontiguousarray(np.asarray(rows_bph, dtype=np.int64).reshape(-1, 3))
    w = np.ascontiguousarray([p[0] for p in patterns], dtype=np.int64)
    r = np.ascontiguousarray([p[1] for p in patterns], dtype=np.int64)
    out = np.empty((rows.shape[0], D), dtype=np.float64)
    lse = np.empty((rows.shape[0],), dtype=np.float64)
    rc = lib.oracle_dilated_attn_rows_fp64(_ptr(q), _ptr(k), _ptr(v), B, N, H, D, len(patterns),
                                           _ptr(w, ctypes.c_int64), _ptr(r, ctypes.c_int64),
                                           int(bool(causal)), rows.shape[0],
                                           _ptr(rows, ctypes.c_int64), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return out, lse


def _patterns(patterns):
    w = np.ascontiguousarray([p[0] for p in patterns], dtype=np.int64)
    r = np.ascontiguousarray([p[1] for p in patterns], dtype=np.int64)
    return w, r


def qk_normalize_bwd_fp64(x, dxhat) -> np.ndarray:
    """Chain rule through x -> x / max(|x|, 1e-12) (qk_normalize_fp64), per
    row over D: with a = 1 / max(|x|, 1e-12) and xhat = a x, the Jacobian is
    a (I - xhat xhat^T) where |x| > 1e-12 and a I elsewhere.  Returns
    the cotangent of x given dxhat, the cotangent of xhat."""
    x, dxhat = _f64(x), _f64(dxhat)
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    a = 1.0 / np.maximum(n, 1e-12)
    xhat = x * a
    proj = dxhat - xhat * (xhat * dxhat).sum(axis=-1, keepdims=True)
    return np.where(n > 1e-12, a * proj, a * dxhat)


def xpos_bwd_fp64(g, downscale=False) -> np.ndarray:
    """Chain rule through xpos_fp64: per element pair the forward is
    y = s R(n theta_i) x (s the pair's scale, its inverse for keys), a linear
    map whose transpose is s R(-n theta_i).  Returns the cotangent of x given
    g, the cotangent of y."""
    g = _f64(g)
    B, N, H, D = g.shape
    n = np.arange(N, dtype=np.float64)[:, None]
    i = np.arange(D // 2, dtype=np.float64)[None, :]
    theta = 10000.0 ** (-2.0 * i / D)
    zeta = (2.0 * i + 0.4 * D) / (1.4 * D)
    s = zeta ** ((n - (N // 2)) / 512.0)
    if downscale:
        s = 1.0 / s
    cos = (np.cos(n * theta) * s)[None, :, None, :]
    sin = (np.sin(n * theta) * s)[None, :, None, :]
    g0, g1 = g[..., 0::2], g[..., 1::2]
    x = np.empty_like(g)
    x[..., 0::2] = g0 * cos + g1 * sin
    x[..., 1::2] = g1 * cos - g0 * sin
    return x


def dilated_attn_bwd_fp64(q, k, v, dout, patterns, causal=True, lib=None, qk_norm=False, xpos=False):
    """Full fp64 backward: the gradients of sum(dout * out) with respect to
    q, k and v, where out is the forward's output.  All tensors [B, N, H, D].
    qk_norm, xpos: the forward normalised q and k rows (qk_normalize_fp64)
    and then applied XPOS (xpos_fp64) before the scores; the gradients go
    back through both, in the reverse order.

    Returns (dq, dk, dv) as float64 arrays.
    """
    if qk_norm or xpos:
        qh, kh = _prologue(q, k, qk_norm, xpos)
        dqh, dkh, dv = dilated_attn_bwd_fp64(qh, kh, v, dout, patterns, causal, lib)
        if xpos:
            dqh, dkh = xpos_bwd_fp64(dqh), xpos_bwd_fp64(dkh, downscale=True)
        if qk_norm:
            dqh, dkh = qk_normalize_bwd_fp64(q, dqh), qk_normalize_bwd_fp64(k, dkh)
        return dqh, dkh, dv
    lib = lib or load_library()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, H, D = q.shape
    w, r = _patterns(patterns)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = lib.oracle_dilated_attn_bwd_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                          _ptr(dk), _ptr(dv), B, N, H, D, len(patterns),
                                          _ptr(w, ctypes.c_int64), _ptr(r, ctypes.c_int64),
                                          int(bool(causal)))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return dq, dk, dv


def dilated_attn_bwd_rows_fp64(q, k, v, dout, patterns, rows_bph, causal=True, lib=None,
                               qk_norm=False):
    """fp64 backward of selected rows only.  rows_bph: int array [n, 3] of
    (b, pos, h).  qk_norm as in dilated_attn_bwd_fp64.  Returns (dq_rows,
    dk_rows, dv_rows), each [n, D]."""
    if qk_norm:
        rows = np.asarray(rows_bph, dtype=np.int64).reshape(-1, 3)
        qh, kh = qk_normalize_fp64(q), qk_normalize_fp64(k)
        dqh, dkh, dv = dilated_attn_bwd_rows_fp64(qh, kh, v, dout, patterns, rows, causal, lib)
        b, pos, h = rows[:, 0], rows[:, 1], rows[:, 2]
        qr, kr = _f64(q)[b, pos, h], _f64(k)[b, pos, h]
        return qk_normalize_bwd_fp64(qr, dqh), qk_normalize_bwd_fp64(kr, dkh), dv
    lib = lib or load_library()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, H, D = q.shape
    rows = np.ascontiguousarray(np.asarray(rows_bph, dtype=np.int64).reshape(-1, 3))
    w, r = _patterns(patterns)
    n = rows.shape[0]
    dq, dk, dv = (np.empty((n, D), dtype=np.float64) for _ in range(3))
    rc = lib.oracle_dilated_attn_bwd_rows_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, H, D,
                                               len(patterns), _ptr(w, ctypes.c_int64),
                                               _ptr(r, ctypes.c_int64), int(bool(causal)), n,
                                               _ptr(rows, ctypes.c_int64), _ptr(dq), _ptr(dk),
                                               _ptr(dv))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")
    return dq, dk, dv


def num_threads(lib=None) -> int:
    """OpenMP threads the oracle runs on."""
    return int((lib or load_library()).oracle_num_threads())
