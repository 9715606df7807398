"""Seeded input generators (CPU only): determinism, shapes, qk_norm, FLOPs."""
import torch

from sparse_long_sequence_attn_b200 import workloads as wl


def test_seeded_and_deterministic():
    w = wl.WORKLOADS["tiny"]
    a = wl.make_inputs(w)
    b = wl.make_inputs(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert a[0].shape == (1, 256, 2, 16) and a[0].dtype == torch.float32
    c = wl.make_inputs(w, seed=w.seed + 1)
    assert not torch.equal(a[0], c[0])


def test_qk_norm_rows_unit_length():
    w = wl.WORKLOADS["smallseg"]
    q, k, v = wl.make_inputs(w, B=1, N=128)
    assert q.dtype == torch.bfloat16
    nq = q.float().norm(dim=-1)
    assert torch.allclose(nq, torch.ones_like(nq), atol=1e-2)
    nv = v.float().norm(dim=-1)
    assert nv.mean() > 4.0  # v is not normalised


def test_sweep_patterns_truncate():
    assert wl.sweep_patterns(65536) == ((2048, 1), (4096, 2), (8192, 4), (16384, 8), (32768, 16), (65536, 32))
    assert len(wl.sweep_patterns(4096)) == 2
    assert wl.sweep_workload(1048576).patterns == wl.sweep_patterns(65536)


def test_flops_formula_values():
    # sum_p 2*2*B*H*(N/r)*(w/r)*D / 2 for the causal workloads
    assert abs(wl.algorithmic_flops(wl.WORKLOADS["long32k"]) - 214.7e9) / 214.7e9 < 1e-3
    assert abs(wl.algorithmic_flops(wl.WORKLOADS["lm"]) - 180.4e9) / 180.4e9 < 1e-3
    assert abs(wl.algorithmic_flops(wl.WORKLOADS["smallseg"]) - 42.9e9) / 42.9e9 < 1e-2


def test_exact_pair_count_matches_key_lists():
    """The bench's exact pair count equals the number of (row, key) pairs the
    brute-force formulation lists, on shapes with r not dividing w, w < r,
    partial last segments and w > N."""
    from oracle.brute import keys_reaching
    from sparse_long_sequence_attn_b200 import workloads as wlm

    cases = [(2, 36, 5, ((12, 5), (18, 3), (36, 7)), True),
             (1, 34, 3, ((12, 1), (8, 3), (40, 5)), True),
             (1, 26, 4, ((8, 2), (11, 3), (2, 3)), False)]
    for B, N, H, pats, causal in cases:
        w = wlm.Workload("pairs", 0, B=B, N=N, H=H, D=8, dtype="fp32", causal=causal, patterns=pats)
        listed = B * sum(len(keys_reaching(pos, h, pats, causal, N)) for h in range(H) for pos in range(N))
        assert wlm.exact_pair_count(w) == listed
