"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
with guard bands around the outputs, pick sampled rows, compare with the
oracle at the tolerances the method's parity bar fixes."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from sparse_long_sequence_attn_b200 import binding as bd

# Parity bar: max-abs error 1e-4 for fp32 inputs, 2e-2 for bf16 inputs (fp32
# accumulation), lse within 1e-3.
# fp16: P, a parked partial and the output are each rounded to 11 bits, at
# most 3 * 2^-11 * max|v| ~ 7e-3 for the N(0,1) draws here; 1e-2 is allowed.
TOL_OUT = {torch.float32: 1e-4, torch.bfloat16: 2e-2, torch.float16: 1e-2}
TOL_LSE = 1e-3
GUARD = 4096  # elements of NaN guard band on each side of every output


def run_cuda(q, k, v, patterns, causal, impl, want_lse=True, stream=None, qk_norm=False):
    """Copy inputs to cuda:0, run the forward into guarded NaN-filled buffers,
    check the guards and the device status word, return CPU (out, lse)."""
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    B, N, H, D = q.shape
    n_out = B * N * H * D
    obuf = torch.full((n_out + 2 * GUARD,), float("nan"), dtype=q.dtype, device=dev)
    out = obuf[GUARD:GUARD + n_out].view(B, N, H, D)
    lbuf = torch.full((B * H * N + 2 * GUARD,), float("nan"), dtype=torch.float32, device=dev)
    lse = lbuf[GUARD:GUARD + B * H * N].view(B, H, N) if want_lse else None
    bd.longnet_dilated_attn_fwd(qd, kd, vd, out, lse, patterns, causal, impl, stream, qk_norm)
    st = bd.longnet_last_device_status(stream)
    assert st == 0, f"device status word: {bd.status_string(st)}"
    assert torch.isnan(obuf[:GUARD].float()).all() and torch.isnan(obuf[-GUARD:].float()).all(), \
        "write outside out"
    assert torch.isnan(lbuf[:GUARD]).all() and torch.isnan(lbuf[-GUARD:]).all(), "write outside lse"
    o = out.float().cpu().numpy()
    assert not np.isnan(o).any(), "some output rows were never written"
    l = lse.cpu().numpy() if want_lse else None
    if want_lse:
        assert not np.isnan(l).any(), "some lse entries were never written"
    return o, l


def compare_full(o, l, q, k, v, patterns, causal, dtype, label="", tol_out=None, qk_norm=False):
    ro, rl = oracle.dilated_attn_fp64(q, k, v, patterns, causal, qk_norm=qk_norm)
    err = float(np.abs(o - ro).max())
    tol = TOL_OUT[dtype] if tol_out is None else tol_out
    assert err <= tol, f"{label}: max|out - oracle| = {err} (tolerance {tol})"
    if l is not None:
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l), fin), f"{label}: -inf pattern of lse differs"
        lerr = float(np.abs(l[fin] - rl[fin]).max()) if fin.any() else 0.0
        assert lerr <= TOL_LSE, f"{label}: max|lse - oracle| = {lerr}"
    return err


def sample_rows(B, N, H, patterns, n_random, seed, boundary=0, boundary_heads=None):
    """(b, pos, h) rows to compare at full size, all kept (no subsampling of
    the structured ones):
      * the first and last kept row of every segment of every pattern, for
        every head and for the first and last batch (the tile edges);
      * with boundary > 0, the rows on both sides of every multiple of
        `boundary` positions and of its half (the kernel's range and split
        points), for the heads in boundary_heads (default: all);
      * n_random seeded random rows."""
    rows = set()
    g = np.random.default_rng(seed)
    for b in sorted({0, B - 1}):
        for h in range(H):
            for (w, r) in patterns:
                o = h % r
                for seg in range((N + w - 1) // w):
                    ln = min(w, N - seg * w)
                    if o < ln:
                        rows.add((b, seg * w + o, h))
                        rows.add((b, seg * w + o + r * ((ln - o - 1) // r), h))
        if boundary > 0:
            heads = range(H) if boundary_heads is None else boundary_heads
            half = max(1, boundary // 2)
            for x in range(0, N + 1, half):
                for pos in (x - 1, x):
                    if 0 <= pos < N:
                        for h in heads:
                            rows.add((b, pos, h))
    for _ in range(n_random):
        rows.add((int(g.integers(B)), int(g.integers(N)), int(g.integers(H))))
    return np.array(sorted(rows), dtype=np.int64)


def compare_rows(o, l, q, k, v, patterns, causal, dtype, rows, label=""):
    ro, rl = oracle.dilated_attn_rows_fp64(q, k, v, patterns, rows, causal)
    b, pos, h = rows[:, 0], rows[:, 1], rows[:, 2]
    got = o[b, pos, h]
    err = float(np.abs(got - ro).max())
    assert err <= TOL_OUT[dtype], f"{label}: max|out - oracle| = {err} over {len(rows)} rows"
    if l is not None:
        gl = l[b, h, pos]
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(gl), fin)
        lerr = float(np.abs(gl[fin] - rl[fin]).max()) if fin.any() else 0.0
        assert lerr <= TOL_LSE, f"{label}: max|lse - oracle| = {lerr}"
    return err


def lse_is_finite_everywhere(l):
    return bool(np.isfinite(l).all()) if l is not None else True


def log2(x):
    return math.log(x, 2)
