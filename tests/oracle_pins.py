"""Pins for the fp64 oracle, written as plain check functions.

Each check takes a loaded build of oracle.c (``lib``) and raises AssertionError
when the oracle disagrees with something fixed independently of it: a library
routine on a case that reduces to textbook attention, a second formulation,
a closed form, a hand-written fixture, or an invariant of the mathematics.
tests/test_oracle_pins.py runs them on the real oracle; tests/test_oracle_mutants.py
runs them on deliberately broken copies and expects each copy to fail one.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle.oracle as orc
from oracle.brute import dilated_attn_bruteforce

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


def _sdpa(q, k, v, mask=None, causal=False):
    """torch's scaled_dot_product_attention in fp64; inputs [N, D] per head."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, is_causal=causal)
    return o[0, 0].numpy()


def _logsumexp_masked(q, k, mask):
    s = torch.from_numpy(q) @ torch.from_numpy(k).T / math.sqrt(q.shape[-1])
    s = s.masked_fill(~torch.from_numpy(mask), -math.inf)
    return torch.logsumexp(s, dim=-1).numpy()


def check_dense_causal(lib):
    """One pattern with w = N, r = 1 is ordinary causal softmax attention."""
    B, N, H, D = 2, 48, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (1, 2, 3))
    out, lse = orc.dilated_attn_fp64(q, k, v, [(N, 1)], causal=True, lib=lib)
    tri = np.tril(np.ones((N, N), dtype=bool))
    for b in range(B):
        for h in range(H):
            ref = _sdpa(q[b, :, h], k[b, :, h], v[b, :, h], causal=True)
            np.testing.assert_allclose(out[b, :, h], ref, atol=1e-12, rtol=0)
            ref_l = _logsumexp_masked(q[b, :, h], k[b, :, h], tri)
            np.testing.assert_allclose(lse[b, h], ref_l, atol=1e-12, rtol=0)


def check_dense_noncausal(lib):
    """One pattern with w = N, r = 1, non-causal is full softmax attention."""
    B, N, H, D = 1, 40, 2, 16
    q, k, v = (_rand((B, N, H, D), s) for s in (4, 5, 6))
    out, lse = orc.dilated_attn_fp64(q, k, v, [(N, 1)], causal=False, lib=lib)
    full = np.ones((N, N), dtype=bool)
    for h in range(H):
        ref = _sdpa(q[0, :, h], k[0, :, h], v[0, :, h], causal=False)
        np.testing.assert_allclose(out[0, :, h], ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[0, h], _logsumexp_masked(q[0, :, h], k[0, :, h], full),
                                   atol=1e-12, rtol=0)


def check_block_diagonal(lib):
    """r = 1 with w < N is block-diagonal attention (causal inside each block);
    when w does not divide N the last block is the shorter rest (N = 60 with
    w = 16 or 25: last blocks of 12 and 10 positions), and w > N is one
    block over the whole sequence."""
    B, N, H, D = 1, 60, 2, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (7, 8, 9))
    for w in (12, 16, 25, 80):
        for causal in (True, False):
            out, _ = orc.dilated_attn_fp64(q, k, v, [(w, 1)], causal=causal, lib=lib)
            blk = np.arange(N) // w
            mask = blk[:, None] == blk[None, :]
            if causal:
                mask &= np.tril(np.ones((N, N), dtype=bool))
            for h in range(H):
                ref = _sdpa(q[0, :, h], k[0, :, h], v[0, :, h], mask=mask)
                np.testing.assert_allclose(out[0, :, h], ref, atol=1e-12, rtol=0)


def read_selection_fixture():
    sel = {}
    with open(os.path.join(GOLDEN, "selection_N24_w12_r5_H3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, rest = line.split(":")
            segs = [[int(t) for t in part.split()] for part in rest.split("|")]
            sel[int(head)] = segs
    return sel


def check_dilated_equals_gathered(lib):
    """One dilated pattern is dense attention on the rows listed by hand in
    the selection fixture; rows no head keeps come out as 0 / -inf."""
    sel = read_selection_fixture()
    B, N, H, D = 1, 24, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (10, 11, 12))
    for causal in (True, False):
        out, lse = orc.dilated_attn_fp64(q, k, v, [(12, 5)], causal=causal, lib=lib)
        for h in range(H):
            kept = set()
            for rows in sel[h]:
                kept.update(rows)
                idx = np.array(rows)
                ref = _sdpa(q[0, idx, h], k[0, idx, h], v[0, idx, h], causal=causal)
                np.testing.assert_allclose(out[0, idx, h], ref, atol=1e-12, rtol=0)
                m = np.tril(np.ones((len(rows),) * 2, dtype=bool)) if causal else \
                    np.ones((len(rows),) * 2, dtype=bool)
                np.testing.assert_allclose(lse[0, h, idx],
                                           _logsumexp_masked(q[0, idx, h], k[0, idx, h], m),
                                           atol=1e-12, rtol=0)
            for pos in range(N):
                if pos not in kept:
                    assert np.all(out[0, pos, h] == 0.0)
                    assert lse[0, h, pos] == -math.inf


def read_support_fixture():
    sup = {}
    with open(os.path.join(GOLDEN, "support_N12_mix.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split(":")
            h, pos = (int(t) for t in left.split())
            sup[(h, pos)] = [int(t) for t in right.split()]
    return sup


def check_support_and_uniform_weights(lib):
    """Q = 0 makes every score 0, so each row averages V over the multiset of
    keys that reach it, and lse = log(count).  With V one-hot over positions
    (D = N), out[pos] is the key histogram / count: compared with the
    hand-written multiset fixture."""
    sup = read_support_fixture()
    B, N, H = 1, 12, 2
    D = N
    q = np.zeros((B, N, H, D))
    k = _rand((B, N, H, D), 13)
    v = np.zeros((B, N, H, D))
    for pos in range(N):
        v[0, pos, :, pos] = 1.0
    out, lse = orc.dilated_attn_fp64(q, k, v, [(4, 1), (6, 2), (12, 3)], causal=True, lib=lib)
    for (h, pos), keys in sup.items():
        hist = np.bincount(keys, minlength=N) / len(keys)
        np.testing.assert_allclose(out[0, pos, h], hist, atol=1e-14, rtol=0)
        assert abs(lse[0, h, pos] - math.log(len(keys))) < 1e-14


def check_bruteforce_agreement(lib):
    """Per-pattern attention + combination agrees with one softmax over the
    multiset union of (pattern, key) pairs, on shapes where r does not divide
    w, heads have different offsets and rows are reached by 1..3 patterns."""
    cases = [
        (1, 36, 5, 4, [(12, 5), (18, 3), (36, 7)], True, 21),
        (2, 30, 3, 6, [(10, 1), (15, 4), (30, 6)], True, 22),
        (1, 24, 4, 5, [(8, 3), (24, 5)], False, 23),
        (1, 32, 2, 8, [(16, 1), (16, 1)], True, 24),  # duplicated pattern
        # w not dividing N (last segments of 10, 2 and 34 positions), w > N
        (1, 34, 3, 4, [(12, 1), (8, 3), (40, 5)], True, 25),
        (2, 26, 4, 4, [(8, 2), (11, 3), (26, 1)], False, 26),
    ]
    for (B, N, H, D, pats, causal, seed) in cases:
        q, k, v = (_rand((B, N, H, D), seed + 100 * i) for i in range(3))
        o1, l1 = orc.dilated_attn_fp64(q, k, v, pats, causal=causal, lib=lib)
        o2, l2 = dilated_attn_bruteforce(q, k, v, pats, causal=causal)
        np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
        np.testing.assert_allclose(l1, l2, atol=1e-12, rtol=0)


def check_disjoint_rows_single_pattern(lib):
    """Rows kept by exactly one pattern equal that pattern's attention alone
    (the disjoint case: the combination adds nothing)."""
    B, N, H, D = 1, 32, 2, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (31, 32, 33))
    pats = [(16, 2), (32, 4)]
    both, _ = orc.dilated_attn_fp64(q, k, v, pats, causal=True, lib=lib)
    only_a, _ = orc.dilated_attn_fp64(q, k, v, pats[:1], causal=True, lib=lib)
    # head 1 of (16, 2) keeps odd rows; (32, 4) keeps rows 1, 5, 9, ... for head 1
    for pos in range(1, N, 2):
        if (pos - 1) % 4 != 0:
            np.testing.assert_allclose(both[0, pos, 1], only_a[0, pos, 1], atol=1e-13, rtol=0)


def check_invariants(lib):
    """Order of patterns does not matter; a duplicated pattern keeps out and
    raises lse by log 2 on its rows; V + c shifts out by c; adding a constant
    vector c to every key shifts each row's scores (in every pattern) by the
    same <q, c>/sqrt(D), so out is unchanged and lse moves by that amount."""
    B, N, H, D = 1, 48, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (41, 42, 43))
    pats = [(12, 1), (24, 2), (48, 5)]
    o, l = orc.dilated_attn_fp64(q, k, v, pats, causal=True, lib=lib)
    o2, l2 = orc.dilated_attn_fp64(q, k, v, pats[::-1], causal=True, lib=lib)
    np.testing.assert_allclose(o2, o, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l2, l, atol=1e-13, rtol=0)
    # duplicate the (48, 5) pattern alone
    od, ld = orc.dilated_attn_fp64(q, k, v, [(48, 5), (48, 5)], causal=True, lib=lib)
    os_, ls_ = orc.dilated_attn_fp64(q, k, v, [(48, 5)], causal=True, lib=lib)
    np.testing.assert_allclose(od, os_, atol=1e-13, rtol=0)
    fin = np.isfinite(ls_)
    np.testing.assert_allclose(ld[fin], ls_[fin] + math.log(2.0), atol=1e-13, rtol=0)
    assert np.all(~np.isfinite(ld[~fin]))
    # V + c
    c = 0.75
    oc, _ = orc.dilated_attn_fp64(q, k, v + c, pats, causal=True, lib=lib)
    np.testing.assert_allclose(oc, o + c, atol=1e-12, rtol=0)
    # K + const vector
    cvec = _rand((D,), 44)
    ok, lk = orc.dilated_attn_fp64(q, k + cvec, v, pats, causal=True, lib=lib)
    np.testing.assert_allclose(ok, o, atol=1e-12, rtol=0)
    shift = np.einsum("bnhd,d->bhn", q, cvec) / math.sqrt(D)
    np.testing.assert_allclose(lk, l + shift, atol=1e-12, rtol=0)


def check_uncovered_rows(lib):
    """With no r = 1 pattern some rows are kept by no pattern: out 0, lse -inf."""
    B, N, H, D = 1, 24, 2, 4
    q, k, v = (_rand((B, N, H, D), s) for s in (51, 52, 53))
    out, lse = orc.dilated_attn_fp64(q, k, v, [(12, 3), (24, 4)], causal=True, lib=lib)
    for h in range(H):
        for pos in range(N):
            kept3 = (pos % 12 - h % 3) >= 0 and (pos % 12 - h % 3) % 3 == 0
            kept4 = (pos - h % 4) >= 0 and (pos - h % 4) % 4 == 0
            if not (kept3 or kept4):
                assert np.all(out[0, pos, h] == 0.0) and lse[0, h, pos] == -math.inf
            else:
                assert np.isfinite(lse[0, h, pos])


def check_rows_function(lib):
    """The per-row entry point returns the same rows as the full forward."""
    B, N, H, D = 2, 36, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (61, 62, 63))
    pats = [(12, 1), (18, 4), (36, 5)]
    for causal in (True, False):
        o, l = orc.dilated_attn_fp64(q, k, v, pats, causal=causal, lib=lib)
        rows = [(b, pos, h) for b in range(B) for pos in range(0, N, 5) for h in range(H)]
        orow, lrow = orc.dilated_attn_rows_fp64(q, k, v, pats, rows, causal=causal, lib=lib)
        for t, (b, pos, h) in enumerate(rows):
            np.testing.assert_allclose(orow[t], o[b, pos, h], atol=1e-13, rtol=0)
            assert abs(lrow[t] - l[b, h, pos]) < 1e-13


def check_rows_function_direct(lib):
    """The per-row entry point pinned on its own: against the multiset
    brute force, and against the Q = 0 closed form of the support fixture."""
    B, N, H, D = 1, 30, 3, 4
    q, k, v = (_rand((B, N, H, D), s) for s in (71, 72, 73))
    pats = [(10, 1), (15, 4), (30, 7)]
    rows = [(0, pos, h) for pos in range(N) for h in range(H)]
    orow, lrow = orc.dilated_attn_rows_fp64(q, k, v, pats, rows, causal=True, lib=lib)
    o2, l2 = dilated_attn_bruteforce(q, k, v, pats, causal=True)
    for t, (b, pos, h) in enumerate(rows):
        np.testing.assert_allclose(orow[t], o2[b, pos, h], atol=1e-12, rtol=0)
        assert abs(lrow[t] - l2[b, h, pos]) < 1e-12
    sup = read_support_fixture()
    D = 12
    qz = np.zeros((1, 12, 2, D))
    kz = _rand((1, 12, 2, D), 74)
    vz = np.zeros((1, 12, 2, D))
    for pos in range(12):
        vz[0, pos, :, pos] = 1.0
    rows = sorted(sup)
    orow, lrow = orc.dilated_attn_rows_fp64(qz, kz, vz, [(4, 1), (6, 2), (12, 3)],
                                            [(0, pos, h) for (h, pos) in rows], causal=True, lib=lib)
    for t, key in enumerate(rows):
        keys = sup[key]
        np.testing.assert_allclose(orow[t], np.bincount(keys, minlength=12) / len(keys), atol=1e-14, rtol=0)
        assert abs(lrow[t] - math.log(len(keys))) < 1e-14


def check_qk_norm(lib):
    """qk_norm: rows are scaled to unit L2 norm (torch's F.normalize in fp64 on
    the same rows, a zero row stays zero); attention with qk_norm equals plain
    attention on rows normalised by F.normalize; and it does not change when
    every q and k row is scaled by its own positive factor."""
    B, N, H, D = 1, 48, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (61, 62, 63))
    q[0, 5, 1] = 0.0  # a zero row
    nq = orc.qk_normalize_fp64(q)
    ref = F.normalize(torch.from_numpy(q), dim=-1, eps=1e-12).numpy()
    np.testing.assert_allclose(nq, ref, atol=1e-15, rtol=0)
    norms = np.linalg.norm(nq, axis=-1)
    assert np.allclose(np.delete(norms.reshape(-1), 5 * H + 1), 1.0, atol=1e-14, rtol=0)
    assert not nq[0, 5, 1].any()
    pats = [(12, 1), (24, 3), (48, 5)]
    for causal in (True, False):
        o1, l1 = orc.dilated_attn_fp64(q, k, v, pats, causal=causal, lib=lib, qk_norm=True)
        qn = F.normalize(torch.from_numpy(q), dim=-1, eps=1e-12).numpy()
        kn = F.normalize(torch.from_numpy(k), dim=-1, eps=1e-12).numpy()
        o2, l2 = orc.dilated_attn_fp64(qn, kn, v, pats, causal=causal, lib=lib)
        np.testing.assert_allclose(o1, o2, atol=1e-13, rtol=0)
        np.testing.assert_allclose(l1, l2, atol=1e-13, rtol=0)
        g = np.random.default_rng(64)
        cq = g.uniform(0.1, 10.0, size=(B, N, H, 1))
        ck = g.uniform(0.1, 10.0, size=(B, N, H, 1))
        o3, l3 = orc.dilated_attn_fp64(q * cq, k * ck, v, pats, causal=causal, lib=lib, qk_norm=True)
        np.testing.assert_allclose(o3, o1, atol=1e-12, rtol=0)
        np.testing.assert_allclose(l3, l1, atol=1e-12, rtol=0)
        # without the option the scaled rows give another result
        o4, _ = orc.dilated_attn_fp64(q * cq, k * ck, v, pats, causal=causal, lib=lib)
        assert np.abs(o4 - o1).max() > 1e-3


def _xpos_score(xpos, qv, m, kv, n, N):
    """xpos(q) at position m dotted with xpos_down(k) at position n, one head."""
    D = len(qv)
    Q = np.zeros((1, N, 1, D))
    K = np.zeros((1, N, 1, D))
    Q[0, m, 0] = qv
    K[0, n, 0] = kv
    return float(np.dot(xpos(Q)[0, m, 0], xpos(K, downscale=True)[0, n, 0]))


def check_xpos(lib, xpos=None):
    """XPOS (the published definition; the pages name the option only):
      * two hand-derived scores.  D = 2 (one pair, theta_0 = 1, zeta_0 =
        0.8 / 2.8 = 2/7), q = (1, 0) at m = 600, k = (0, 1) at n = 88: the
        rotated q is s_m (cos 600, sin 600), the rotated k is
        (-sin 88, cos 88) / s_n, so the score is (s_m / s_n) sin(600 - 88) =
        (2/7)^(512/512) sin(512).  D = 4, q = k = (0, 0, 1, 0) at m = 1100,
        n = 76: only pair 1 (theta_1 = 10000^(-1/2) = 0.01, zeta_1 = 3.6 / 5.6
        = 9/14) is non-zero, score (9/14)^(1024/512) cos(1024 * 0.01);
      * every pair's length scales by zeta_i^((n - c) / 512) (c = N // 2) for
        queries and by its inverse for keys;
      * a score depends on the positions' difference only (shift both by t).
    """
    xpos = xpos or orc.xpos_fp64
    got = _xpos_score(xpos, [1.0, 0.0], 600, [0.0, 1.0], 88, 1024)
    assert abs(got - (2.0 / 7.0) * math.sin(512.0)) < 1e-12, got
    got = _xpos_score(xpos, [0.0, 0.0, 1.0, 0.0], 1100, [0.0, 0.0, 1.0, 0.0], 76, 2048)
    assert abs(got - (9.0 / 14.0) ** 2 * math.cos(10.24)) < 1e-12, got
    B, N, H, D = 2, 300, 3, 8
    x = _rand((B, N, H, D), 71)
    zeta = np.array([(2 * i + 0.4 * D) / (1.4 * D) for i in range(D // 2)])
    rel = (np.arange(N) - N // 2)[:, None] / 512.0
    pair_len = lambda a: np.sqrt(a[..., 0::2] ** 2 + a[..., 1::2] ** 2)  # noqa: E731
    for down, sgn in ((False, 1.0), (True, -1.0)):
        want = pair_len(x) * (zeta[None, :] ** (sgn * rel))[None, :, None, :]
        np.testing.assert_allclose(pair_len(xpos(x, downscale=down)), want, rtol=1e-12, atol=0)
    g = np.random.default_rng(72)
    qv, kv = g.standard_normal(16), g.standard_normal(16)
    for (m, n, t) in ((700, 100, 1500), (64, 2000, 333), (3000, 3000, -2900)):
        a = _xpos_score(xpos, qv, m, kv, n, 4096)
        b = _xpos_score(xpos, qv, m + t, kv, n + t, 4096)
        assert abs(a - b) < 1e-9 * max(1.0, abs(a)), (m, n, t, a, b)
    # the option reaches the attention: it changes the result, and the
    # attention on pre-encoded rows is the same
    q, k, v = (_rand((1, 64, 2, 8), s) for s in (73, 74, 75))
    pats = [(16, 1), (64, 2)]
    o1, l1 = orc.dilated_attn_fp64(q, k, v, pats, lib=lib, xpos=True)
    o2, l2 = orc.dilated_attn_fp64(orc.xpos_fp64(q), orc.xpos_fp64(k, downscale=True), v, pats, lib=lib)
    np.testing.assert_allclose(o1, o2, atol=1e-13, rtol=0)
    o3, _ = orc.dilated_attn_fp64(q, k, v, pats, lib=lib)
    assert np.abs(o3 - o1).max() > 1e-3


# ---------------------------------------------------------------- backward


def _brute_autograd(q, k, v, dout, patterns, causal):
    """Gradients of sum(dout * out) by torch autograd through the multiset
    formulation of brute.py: one softmax per row over the (pattern, key) pairs
    that reach it, written as a dense masked softmax in which a key reached
    c times gets the logit s + log c.  A different formulation from the
    oracle's, differentiated by the library."""
    from oracle.brute import keys_reaching

    B, N, H, D = q.shape
    tq, tk, tv = (torch.from_numpy(np.array(x)).requires_grad_(True) for x in (q, k, v))
    bias = np.full((H, N, N), -math.inf)
    for h in range(H):
        for pos in range(N):
            keys = keys_reaching(pos, h, patterns, causal, N)
            cnt = np.bincount(keys, minlength=N) if keys else np.zeros(N)
            nz = cnt > 0
            bias[h, pos, nz] = np.log(cnt[nz])
    tb = torch.from_numpy(bias)
    rows_out = []
    for b in range(B):
        per_h = []
        for h in range(H):
            s = tq[b, :, h] @ tk[b, :, h].T / math.sqrt(D) + tb[h]
            kept = torch.isfinite(tb[h]).any(dim=-1)
            p = torch.softmax(torch.where(kept[:, None], s, torch.zeros_like(s)), dim=-1)
            o = (p @ tv[b, :, h]) * kept[:, None]
            per_h.append(o)
        rows_out.append(torch.stack(per_h, dim=1))
    outs = torch.stack(rows_out, dim=0)
    (outs * torch.from_numpy(np.array(dout))).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def check_bwd_dense_autograd(lib):
    """One pattern with w = N, r = 1 is ordinary softmax attention: its
    gradients equal torch autograd through scaled_dot_product_attention in
    fp64, causal and not."""
    B, N, H, D = 1, 40, 2, 8
    q, k, v, do = (_rand((B, N, H, D), s) for s in (81, 82, 83, 84))
    for causal in (True, False):
        dq, dk, dv = orc.dilated_attn_bwd_fp64(q, k, v, do, [(N, 1)], causal=causal, lib=lib)
        for h in range(H):
            tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x[0, :, h]))[None, None]
                          .requires_grad_(True) for x in (q, k, v))
            o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
            (o[0, 0] * torch.from_numpy(np.ascontiguousarray(do[0, :, h]))).sum().backward()
            np.testing.assert_allclose(dq[0, :, h], tq.grad[0, 0].numpy(), atol=1e-12, rtol=0)
            np.testing.assert_allclose(dk[0, :, h], tk.grad[0, 0].numpy(), atol=1e-12, rtol=0)
            np.testing.assert_allclose(dv[0, :, h], tv.grad[0, 0].numpy(), atol=1e-12, rtol=0)


def check_bwd_bruteforce_autograd(lib):
    """Several overlapping patterns (rows reached by 1..3 patterns, r not
    dividing w, partial last segments, w > N, a duplicated pattern): the
    oracle's gradients equal torch autograd through the multiset-softmax
    formulation."""
    cases = [
        (1, 36, 5, 4, [(12, 5), (18, 3), (36, 7)], True, 91),
        (2, 26, 4, 4, [(8, 2), (11, 3), (26, 1)], False, 92),
        (1, 34, 3, 4, [(12, 1), (8, 3), (40, 5)], True, 93),
        (1, 32, 2, 8, [(16, 1), (16, 1)], True, 94),
        (1, 24, 4, 5, [(12, 3), (24, 4)], True, 95),  # rows kept by no pattern
    ]
    for (B, N, H, D, pats, causal, seed) in cases:
        q, k, v, do = (_rand((B, N, H, D), seed + 100 * i) for i in range(4))
        got = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib)
        ref = _brute_autograd(q, k, v, do, pats, causal)
        for g, r_ in zip(got, ref):
            np.testing.assert_allclose(g, r_, atol=1e-12, rtol=0)


def check_bwd_finite_differences(lib):
    """Central differences of the oracle's own forward, sum(dout * out), on a
    handful of coordinates of q, k and v: the backward is the forward's
    derivative."""
    B, N, H, D = 1, 30, 3, 4
    pats = [(10, 1), (15, 2), (30, 4)]
    q, k, v, do = (_rand((B, N, H, D), s) for s in (101, 102, 103, 104))
    eps = 1e-5
    for causal in (True, False):
        grads = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib)
        g = np.random.default_rng(105)
        for which in range(3):
            for _ in range(6):
                idx = (0, int(g.integers(N)), int(g.integers(H)), int(g.integers(D)))
                vals = []
                for sgn in (1.0, -1.0):
                    args = [q.copy(), k.copy(), v.copy()]
                    args[which][idx] += sgn * eps
                    o, _ = orc.dilated_attn_fp64(*args, pats, causal=causal, lib=lib)
                    vals.append(float((o * do).sum()))
                fd = (vals[0] - vals[1]) / (2 * eps)
                assert abs(fd - grads[which][idx]) < 1e-7 * max(1.0, abs(fd)), (which, idx)


def check_bwd_invariants(lib):
    """Each row's probabilities sum to one over its pairs, so per (b, h) the
    dv rows add up to the sum of dout over the rows some pattern keeps; the
    score cotangents of a row sum to zero, so the dk rows add up to zero; a
    row kept by no pattern gets dq = dk = dv = 0; scaling dout scales every
    gradient."""
    B, N, H, D = 2, 24, 4, 5
    pats = [(12, 3), (24, 4)]
    q, k, v, do = (_rand((B, N, H, D), s) for s in (111, 112, 113, 114))
    for causal in (True, False):
        dq, dk, dv = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib)
        _, lse = orc.dilated_attn_fp64(q, k, v, pats, causal=causal, lib=lib)
        kept = np.isfinite(lse).transpose(0, 2, 1)  # [B, N, H]
        assert (~kept).any()
        np.testing.assert_allclose(dv.sum(axis=1), (do * kept[..., None]).sum(axis=1),
                                   atol=1e-12, rtol=0)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12, rtol=0)
        for g_ in (dq, dk, dv):
            assert not g_[~kept].any()
        d2 = orc.dilated_attn_bwd_fp64(q, k, v, 2.5 * do, pats, causal=causal, lib=lib)
        for a_, b_ in zip(d2, (dq, dk, dv)):
            np.testing.assert_allclose(a_, 2.5 * b_, atol=1e-12, rtol=0)


def check_bwd_rows_function(lib):
    """The per-row backward returns the full backward's rows, and on its own
    agrees with autograd through the multiset formulation."""
    B, N, H, D = 2, 36, 3, 4
    q, k, v, do = (_rand((B, N, H, D), s) for s in (121, 122, 123, 124))
    pats = [(12, 1), (18, 4), (40, 5)]
    rows = [(b, pos, h) for b in range(B) for pos in range(0, N, 5) for h in range(H)]
    for causal in (True, False):
        full = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib)
        got = orc.dilated_attn_bwd_rows_fp64(q, k, v, do, pats, rows, causal=causal, lib=lib)
        ref = _brute_autograd(q, k, v, do, pats, causal)
        for t, (b, pos, h) in enumerate(rows):
            for which in range(3):
                np.testing.assert_allclose(got[which][t], full[which][b, pos, h], atol=1e-13, rtol=0)
                np.testing.assert_allclose(got[which][t], ref[which][b, pos, h], atol=1e-12, rtol=0)


def check_bwd_closed_form(lib):
    """N = 2, D = 1, one pattern (2, 1), causal: row 0 sees key 0 only
    (out0 = v0), row 1 sees keys 0 and 1 with p0 = 1 / (1 + e^{q1 (k1 - k0)}).
    With L = g0 out0 + g1 out1, by hand: dv0 = g0 + g1 p0, dv1 = g1 p1,
    ds10 = g1 p0 p1 (v0 - v1) = -ds11, dq0 = 0, dq1 = ds10 (k0 - k1),
    dk0 = ds10 q1, dk1 = -ds10 q1.  And duplicating every pattern leaves out,
    hence every gradient, unchanged."""
    q0, q1, k0, k1, v0, v1, g0, g1 = 0.5, 1.0, 2.0, -1.0, 3.0, 1.0, 0.25, 2.0
    q = np.array([q0, q1]).reshape(1, 2, 1, 1)
    k = np.array([k0, k1]).reshape(1, 2, 1, 1)
    v = np.array([v0, v1]).reshape(1, 2, 1, 1)
    do = np.array([g0, g1]).reshape(1, 2, 1, 1)
    dq, dk, dv = orc.dilated_attn_bwd_fp64(q, k, v, do, [(2, 1)], causal=True, lib=lib)
    p0 = 1.0 / (1.0 + math.exp(q1 * (k1 - k0)))
    p1 = 1.0 - p0
    ds10 = g1 * p0 * p1 * (v0 - v1)
    np.testing.assert_allclose(dq.ravel(), [0.0, ds10 * (k0 - k1)], atol=1e-15, rtol=0)
    np.testing.assert_allclose(dk.ravel(), [ds10 * q1, -ds10 * q1], atol=1e-15, rtol=0)
    np.testing.assert_allclose(dv.ravel(), [g0 + g1 * p0, g1 * p1], atol=1e-15, rtol=0)
    B, N, H, D = 1, 36, 3, 4
    pats = [(12, 1), (18, 3), (36, 5)]
    qr, kr, vr, dor = (_rand((B, N, H, D), s) for s in (141, 142, 143, 144))
    for causal in (True, False):
        once = orc.dilated_attn_bwd_fp64(qr, kr, vr, dor, pats, causal=causal, lib=lib)
        twice = orc.dilated_attn_bwd_fp64(qr, kr, vr, dor, pats + pats, causal=causal, lib=lib)
        for a_, b_ in zip(once, twice):
            np.testing.assert_allclose(b_, a_, atol=1e-13, rtol=0)


def check_bwd_qk_norm(lib):
    """The backward with qk_norm: central differences of the qk_norm forward,
    torch autograd through F.normalize and the multiset formulation, a zero
    row (the 1/eps branch of the normalisation), and the per-row entry point
    against the full backward."""
    B, N, H, D = 1, 36, 3, 4
    pats = [(12, 1), (18, 3), (36, 4)]
    q, k, v, do = (_rand((B, N, H, D), s) for s in (131, 132, 133, 134))
    q[0, 7, 1] = 0.0  # a zero query row
    for causal in (True, False):
        grads = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib, qk_norm=True)
        # autograd through F.normalize, then the multiset formulation
        tq, tk = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k))
        qn = F.normalize(tq, dim=-1, eps=1e-12)
        kn = F.normalize(tk, dim=-1, eps=1e-12)
        gq, gk, gv = _brute_autograd(qn.detach().numpy(), kn.detach().numpy(), v, do, pats, causal)
        torch.autograd.backward([qn, kn], [torch.from_numpy(gq), torch.from_numpy(gk)])
        # the zero row's gradient is dqhat / 1e-12 (~1e12): compare it relatively
        np.testing.assert_allclose(grads[0], tq.grad.numpy(), atol=1e-11, rtol=1e-12)
        assert np.abs(grads[0][0, 7, 1]).max() > 1e9
        np.testing.assert_allclose(grads[1], tk.grad.numpy(), atol=1e-11, rtol=0)
        np.testing.assert_allclose(grads[2], gv, atol=1e-12, rtol=0)
        # central differences of the qk_norm forward (away from the zero row)
        eps = 1e-6
        g = np.random.default_rng(135)
        for which in range(3):
            for _ in range(5):
                idx = (0, int(g.integers(8, N)), int(g.integers(H)), int(g.integers(D)))
                vals = []
                for sgn in (1.0, -1.0):
                    args = [q.copy(), k.copy(), v.copy()]
                    args[which][idx] += sgn * eps
                    o, _ = orc.dilated_attn_fp64(*args, pats, causal=causal, lib=lib, qk_norm=True)
                    vals.append(float((o * do).sum()))
                fd = (vals[0] - vals[1]) / (2 * eps)
                assert abs(fd - grads[which][idx]) < 1e-6 * max(1.0, abs(fd)), (which, idx)
        rows = [(0, pos, h) for pos in range(0, N, 5) for h in range(H)] + [(0, 7, 1)]
        got = orc.dilated_attn_bwd_rows_fp64(q, k, v, do, pats, rows, causal=causal, lib=lib,
                                             qk_norm=True)
        for t, (b, pos, h) in enumerate(rows):
            for which in range(3):
                np.testing.assert_allclose(got[which][t], grads[which][b, pos, h], atol=1e-12,
                                           rtol=1e-12)


def check_bwd_xpos(lib, xpos_bwd=None):
    """The backward through XPOS (and qk_norm then XPOS): the adjoint identity
    <xpos(x), g> = <x, xpos_bwd(g)> for queries and keys (XPOS is linear in x),
    and central differences of the forward with the options."""
    xpos_bwd = xpos_bwd or orc.xpos_bwd_fp64
    B, N, H, D = 1, 40, 2, 4
    x, g = _rand((B, N, H, D), 141), _rand((B, N, H, D), 142)
    for down in (False, True):
        lhs = float((orc.xpos_fp64(x, downscale=down) * g).sum())
        rhs = float((x * xpos_bwd(g, downscale=down)).sum())
        assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs)), (down, lhs, rhs)
    pats = [(10, 1), (20, 2), (40, 4)]
    q, k, v, do = (_rand((B, N, H, D), s) for s in (143, 144, 145, 146))
    saved = orc.xpos_bwd_fp64
    orc.xpos_bwd_fp64 = xpos_bwd
    try:
        for qk_norm in (False, True):
            for causal in (True, False):
                grads = orc.dilated_attn_bwd_fp64(q, k, v, do, pats, causal=causal, lib=lib, qk_norm=qk_norm,
                                                  xpos=True)
                eps = 1e-6
                gen = np.random.default_rng(147)
                for which in range(3):
                    for _ in range(4):
                        idx = (0, int(gen.integers(N)), int(gen.integers(H)), int(gen.integers(D)))
                        vals = []
                        for sgn in (1.0, -1.0):
                            args = [q.copy(), k.copy(), v.copy()]
                            args[which][idx] += sgn * eps
                            o, _ = orc.dilated_attn_fp64(*args, pats, causal=causal, lib=lib, qk_norm=qk_norm,
                                                         xpos=True)
                            vals.append(float((o * do).sum()))
                        fd = (vals[0] - vals[1]) / (2 * eps)
                        assert abs(fd - grads[which][idx]) < 1e-6 * max(1.0, abs(fd)), (qk_norm, causal, which, idx)
    finally:
        orc.xpos_bwd_fp64 = saved


ALL_CHECKS = [
    check_rows_function_direct,
    check_qk_norm,
    check_xpos,
    check_dense_causal,
    check_dense_noncausal,
    check_block_diagonal,
    check_dilated_equals_gathered,
    check_support_and_uniform_weights,
    check_bruteforce_agreement,
    check_disjoint_rows_single_pattern,
    check_invariants,
    check_uncovered_rows,
    check_rows_function,
    check_bwd_dense_autograd,
    check_bwd_bruteforce_autograd,
    check_bwd_finite_differences,
    check_bwd_invariants,
    check_bwd_rows_function,
    check_bwd_closed_form,
    check_bwd_qk_norm,
    check_bwd_xpos,
]
