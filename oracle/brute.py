"""Second, independent fp64 formulation for tiny inputs (TEST INFRASTRUCTURE ONLY).

Instead of attending per pattern and then combining, every output row is one
softmax over the multiset of (pattern, key) pairs that reach it: a key kept by
two patterns appears twice.  Combining per-pattern results weighted by their
softmax denominators gives exactly this (the denominators add up), so the two
formulations must agree to rounding.  Pure Python loops over rows: tiny sizes
only.
"""
from __future__ import annotations

import math

import numpy as np


def keys_reaching(pos: int, h: int, patterns, causal: bool, N: int | None = None):
    """List of key positions (with repeats across patterns) that row `pos` of
    head `h` attends to: for each pattern (w, r) that keeps the row, the kept
    rows of its segment up to the row itself (all kept rows if not causal).
    The last segment of a pattern ends with the sequence (length N mod w)."""
    keys = []
    for (w, r) in patterns:
        seg_start = (pos // w) * w
        o = h % r
        off = pos - seg_start - o
        if off < 0 or off % r:
            continue
        j = 0
        while o + r * j < w and (N is None or seg_start + o + r * j < N):
            kp = seg_start + o + r * j
            if causal and kp > pos:
                break
            keys.append(kp)
            j += 1
    return keys


def dilated_attn_bruteforce(q, k, v, patterns, causal=True):
    """q, k, v: float arrays [B, N, H, D].  Returns (out, lse) in float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, D = q.shape
    out = np.zeros((B, N, H, D))
    lse = np.full((B, H, N), -math.inf)
    scale = 1.0 / math.sqrt(D)
    for b in range(B):
        for h in range(H):
            for pos in range(N):
                keys = keys_reaching(pos, h, patterns, causal, N)
                if not keys:
                    continue
                s = np.array([float(np.dot(q[b, pos, h], k[b, kp, h])) * scale for kp in keys])
                mx = s.max()
                e = np.exp(s - mx)
                out[b, pos, h] = (e[:, None] * v[b, keys, h]).sum(0) / e.sum()
                lse[b, h, pos] = mx + math.log(e.sum())
    return out, lse
