"""The backward tile kernels' walk, restated on the CPU (CPU only): the unit
decode, the key-tile and query-tile loops and the masks of bwd_dkv_tile_kernel
and bwd_dq_tile_kernel visit every (query, key) pair of every sparsified
segment exactly once, and every row they touch lies inside the sequence.
The restatement follows csrc/backward.cu line for line in its index
arithmetic (tile_geometry, decode_unit, the loop bounds, the `ok` masks)."""
import pytest

TILE = 64


def geometry(B, N, H, pats):
    unit_base, n_segs, units, t_max = [], [], 0, 0
    for (w, r) in pats:
        n_seg = (N + w - 1) // w
        m_max = (min(w, N) + r - 1) // r
        t_max = max(t_max, (m_max + TILE - 1) // TILE)
        unit_base.append(units)
        n_segs.append(n_seg)
        units += B * H * n_seg
    unit_base.append(units)
    return unit_base, n_segs, units, t_max


def decode(N, H, pats, unit_base, n_segs, x):
    p = 0
    while p + 1 < len(pats) and x >= unit_base[p + 1]:
        p += 1
    rem = x - unit_base[p]
    seg = rem % n_segs[p]
    rem //= n_segs[p]
    h, b = rem % H, rem // H
    w, r = pats[p]
    o = h % r
    ln = min(w, N - seg * w)
    m = (ln - o + r - 1) // r if ln > o else 0
    return p, b, h, seg, seg * w + o, r, m


def walk(B, N, H, pats, causal):
    unit_base, n_segs, units, t_max = geometry(B, N, H, pats)
    dkv, dq = set(), set()
    for x in range(units):
        p, b, h, seg, first, r, m = decode(N, H, pats, unit_base, n_segs, x)
        T = (m + TILE - 1) // TILE
        for t in range(m):
            assert 0 <= first + r * t < N
        for y in range(t_max):
            if y < T:  # dk/dv: key tile jt = y over query tiles it0 .. T-1
                jt = y
                for it in range(jt if causal else 0, T):
                    for kr in range(jt * TILE, jt * TILE + TILE):
                        for qi in range(it * TILE, it * TILE + TILE):
                            if qi < m and kr < m and (not causal or qi >= kr):
                                key = (p, b, h, seg, qi, kr)
                                assert key not in dkv
                                dkv.add(key)
                it = T - 1 - y  # dq: query tile it over key tiles 0 .. jt_end-1
                for jt in range(it + 1 if causal else T):
                    for qi in range(it * TILE, min(it * TILE + TILE, m)):  # rows past m not stored
                        for kj in range(jt * TILE, jt * TILE + TILE):
                            if kj < m and (not causal or kj <= qi):
                                key = (p, b, h, seg, qi, kj)
                                assert key not in dq
                                dq.add(key)
    return dkv, dq


def expected(B, N, H, pats, causal):
    out = set()
    for p, (w, r) in enumerate(pats):
        for b in range(B):
            for h in range(H):
                for seg in range((N + w - 1) // w):
                    o = h % r
                    ln = min(w, N - seg * w)
                    m = (ln - o + r - 1) // r if ln > o else 0
                    for qi in range(m):
                        for kj in range(m if not causal else qi + 1):
                            out.add((p, b, h, seg, qi, kj))
    return out


@pytest.mark.parametrize("B,N,H,pats,causal", [
    (1, 256, 2, ((64, 1), (128, 2), (256, 4)), True),
    (2, 300, 3, ((64, 1), (128, 3), (512, 5)), True),   # partial segments, w > N
    (1, 300, 2, ((128, 1), (160, 2)), False),
    (1, 200, 5, ((200, 1), (40, 3), (8, 2)), True),     # several tiles, tiny segments
    (1, 129, 3, ((129, 1), (7, 12)), True),             # a one-row ragged tile, r > w
])
def test_every_pair_once(B, N, H, pats, causal):
    dkv, dq = walk(B, N, H, pats, causal)
    exp = expected(B, N, H, pats, causal)
    assert dkv == exp
    assert dq == exp
