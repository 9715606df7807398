"""GPU parity: every kernel family through the C ABI against the fp64 oracle
on the same seeded inputs (needs a B200)."""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

from sparse_long_sequence_attn_b200 import binding as bd
from sparse_long_sequence_attn_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

IMPLS = {"simt": bd.LONGNET_IMPL_SIMT, "tcgen05": bd.LONGNET_IMPL_TCGEN05,
         "smallseg": bd.LONGNET_IMPL_SMALLSEG, "patterns": bd.LONGNET_IMPL_PATTERNS}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    bd.load_library()
    yield


# Small cases spanning several tiles and ragged tails: r not dividing w,
# rows reached by 1..n patterns, rows reached by none, duplicates, B > 1.
SMALL_CASES = [
    # name, B, N, H, D, dtype, causal, patterns
    ("tiny_cfg", 1, 256, 2, 16, torch.float32, True, ((64, 1), (128, 2), (256, 4))),
    ("fp32_d32_rdivw", 2, 384, 3, 32, torch.float32, True, ((96, 1), (192, 5), (384, 7))),
    ("fp32_d64_noncausal", 1, 512, 2, 64, torch.float32, False, ((128, 1), (256, 3))),
    ("fp32_d128_uncovered", 1, 240, 3, 128, torch.float32, True, ((48, 3), (240, 4))),
    ("bf16_d64_lm_like", 2, 2048, 4, 64, torch.bfloat16, True, ((512, 1), (1024, 2), (2048, 4))),
    ("bf16_d64_paper_like", 1, 3072, 6, 64, torch.bfloat16, True,
     ((256, 1), (512, 2), (1024, 4), (1536, 6), (3072, 12))),
    ("bf16_d64_dup_unordered", 1, 1024, 3, 64, torch.bfloat16, True, ((1024, 4), (256, 1), (256, 1))),
    ("bf16_d64_noncausal_small", 2, 1024, 4, 64, torch.bfloat16, False, ((64, 1), (64, 2))),
    ("bf16_d64_no_r1", 1, 1536, 5, 64, torch.bfloat16, True, ((384, 3), (768, 4), (1536, 8))),
    ("bf16_d64_w_eq_N", 1, 640, 2, 64, torch.bfloat16, True, ((640, 1),)),
    ("bf16_d64_r_gt_w", 1, 512, 4, 64, torch.bfloat16, True, ((512, 1), (2, 3))),
    ("bf16_d32", 1, 512, 2, 32, torch.bfloat16, True, ((128, 1), (512, 2))),
    ("bf16_d64_seg32_causal", 2, 512, 3, 64, torch.bfloat16, True, ((32, 4), (32, 2), (32, 1))),
    ("bf16_d64_seg64_r3_noncausal", 1, 1024, 4, 64, torch.bfloat16, False, ((64, 3), (64, 1))),
    ("bf16_d64_seg64_r2_causal", 1, 1024, 4, 64, torch.bfloat16, True, ((64, 1), (64, 2))),
    # segment lengths that are not a multiple of 16, four patterns, r > W
    ("bf16_d64_seg40_4pat", 1, 800, 5, 64, torch.bfloat16, True, ((40, 1), (40, 3), (40, 7), (40, 48))),
    ("bf16_d64_seg8_noncausal", 2, 256, 3, 64, torch.bfloat16, False, ((8, 1), (8, 2))),
    ("bf16_d64_seg56_r5", 1, 560, 6, 64, torch.bfloat16, False, ((56, 5), (56, 1), (56, 2))),
    # one segment length: eight patterns (repeats count twice), no r = 1 (rows
    # no pattern keeps), W not a multiple of 16 with every r dividing 8
    ("bf16_d64_seg64_eight_patterns", 2, 1024, 8, 64, torch.bfloat16, False,
     ((64, 1), (64, 2), (64, 4), (64, 8), (64, 2), (64, 4), (64, 8), (64, 1))),
    ("bf16_d64_seg32_no_r1_causal", 1, 512, 8, 64, torch.bfloat16, True, ((32, 2), (32, 4), (32, 8))),
    ("f16_d64_seg48_r8_causal", 2, 480, 9, 64, torch.float16, True, ((48, 1), (48, 8), (48, 4))),
    # one segment length, the last segment the shorter rest (or w > N)
    ("bf16_d64_seg64_partial_noncausal", 2, 1000, 4, 64, torch.bfloat16, False, ((64, 1), (64, 2))),
    ("f16_d64_seg32_partial_causal", 1, 500, 3, 64, torch.float16, True, ((32, 1), (32, 4))),
    ("bf16_d64_seg48_w_gt_n", 2, 40, 2, 64, torch.bfloat16, False, ((48, 1), (48, 2), (48, 3))),
    ("f16_d64_seg32_odd_n", 1, 1001, 2, 64, torch.float16, False, ((32, 1), (32, 2), (32, 4))),
    # fp16 inputs (every family)
    ("f16_d64_lm_like", 2, 2048, 4, 64, torch.float16, True, ((512, 1), (1024, 2), (2048, 4))),
    ("f16_d64_r_not_dividing", 1, 1536, 5, 64, torch.float16, True, ((384, 3), (768, 4), (1536, 8))),
    ("f16_d64_seg64_r2_noncausal", 2, 1024, 4, 64, torch.float16, False, ((64, 1), (64, 2))),
    ("f16_d32", 1, 512, 2, 32, torch.float16, True, ((128, 1), (512, 2))),
    # w not dividing N: the last segment is the shorter rest; w > N is one segment
    ("fp32_d32_partial_segments", 1, 300, 3, 32, torch.float32, True, ((64, 1), (128, 3), (512, 5))),
    ("bf16_d64_partial_noncausal", 2, 1000, 4, 64, torch.bfloat16, False, ((256, 1), (384, 2))),
    ("f16_d64_partial_causal", 1, 777, 2, 64, torch.float16, True, ((128, 1), (256, 4))),
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
@pytest.mark.parametrize("impl_name", ["auto", "simt"])
def test_small_cases_vs_oracle(case, impl_name):
    name, B, N, H, D, dtype, causal, pats = case
    impl = bd.LONGNET_IMPL_AUTO if impl_name == "auto" else IMPLS[impl_name]
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=zlib.crc32(name.encode()) % 100000)
    o, l = gh.run_cuda(q, k, v, pats, causal, impl)
    gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"{name}/{impl_name}")


@pytest.mark.parametrize("case", [c for c in SMALL_CASES if c[5] in (torch.bfloat16, torch.float16) and c[4] == 64],
                         ids=[c[0] for c in SMALL_CASES if c[5] in (torch.bfloat16, torch.float16) and c[4] == 64])
@pytest.mark.parametrize("impl_name", ["tcgen05", "smallseg", "patterns"])
def test_specialised_families_vs_oracle(case, impl_name):
    name, B, N, H, D, dtype, causal, pats = case
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=zlib.crc32(name.encode()) % 100000)
    try:
        o, l = gh.run_cuda(q, k, v, pats, causal, IMPLS[impl_name])
    except bd.LongNetError as e:
        if e.code == bd.LONGNET_ERR_UNSUPPORTED:
            pytest.skip(f"{impl_name} does not take {name}")
        raise
    gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"{name}/{impl_name}")


# Shapes the fused tcgen05 family does not take: D = 128, more than six
# patterns, more than eight distinct r; the per-pattern family does.
PATTERNS_CASES = [
    # name, B, N, H, D, dtype, causal, patterns
    ("bf16_d128_lm_like", 2, 2048, 4, 128, torch.bfloat16, True, ((512, 1), (1024, 2), (2048, 4))),
    ("bf16_d128_noncausal_partial", 1, 1500, 3, 128, torch.bfloat16, False, ((384, 1), (700, 3), (2000, 5))),
    ("f16_d128_causal", 1, 1024, 2, 128, torch.float16, True, ((256, 1), (1024, 4))),
    ("bf16_d64_seven_patterns", 1, 2048, 5, 64, torch.bfloat16, True,
     ((128, 1), (256, 2), (384, 3), (512, 4), (768, 5), (1024, 6), (2048, 8))),
    ("bf16_d128_one_pattern", 1, 1024, 2, 128, torch.bfloat16, True, ((256, 1),)),
    ("bf16_d128_uncovered", 1, 960, 3, 128, torch.bfloat16, True, ((192, 3), (960, 4))),
    # narrow heads: one 64- or 32-byte swizzle panel per row
    ("bf16_d32_lm_like", 2, 2048, 4, 32, torch.bfloat16, True, ((512, 1), (1024, 2), (2048, 4))),
    ("f16_d32_noncausal_partial", 1, 1500, 3, 32, torch.float16, False, ((384, 1), (700, 3), (2000, 5))),
    ("bf16_d16_causal", 1, 2048, 4, 16, torch.bfloat16, True, ((256, 1), (1024, 4))),
    ("f16_d16_noncausal", 2, 1024, 2, 16, torch.float16, False, ((128, 1), (512, 2), (1024, 8))),
]


@pytest.mark.parametrize("case", PATTERNS_CASES, ids=[c[0] for c in PATTERNS_CASES])
@pytest.mark.parametrize("impl_name", ["auto", "patterns"])
def test_per_pattern_family_vs_oracle(case, impl_name):
    name, B, N, H, D, dtype, causal, pats = case
    impl = bd.LONGNET_IMPL_AUTO if impl_name == "auto" else IMPLS[impl_name]
    if impl_name == "auto":
        assert bd.longnet_select_impl(B, N, H, D, pats, causal, dtype) == bd.LONGNET_IMPL_PATTERNS
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=zlib.crc32(name.encode()) % 100000)
    o, l = gh.run_cuda(q, k, v, pats, causal, impl)
    err = gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"{name}/{impl_name}")
    print(f"{name}/{impl_name}: max|out - oracle| = {err:.3e}")


def test_per_pattern_family_without_lse():
    """One pattern needs no lse; several need it (else AUTO picks SIMT and the
    forced family is refused)."""
    q, k, v = wl.random_inputs(1, 1024, 2, 128, torch.bfloat16, seed=41)
    o1, _ = gh.run_cuda(q, k, v, ((256, 1),), True, bd.LONGNET_IMPL_PATTERNS, want_lse=False)
    gh.compare_full(o1, None, q, k, v, ((256, 1),), True, torch.bfloat16, label="one pattern, no lse")
    with pytest.raises(bd.LongNetError) as e:
        gh.run_cuda(q, k, v, ((256, 1), (1024, 2)), True, bd.LONGNET_IMPL_PATTERNS, want_lse=False)
    assert e.value.code == bd.LONGNET_ERR_UNSUPPORTED


@pytest.mark.parametrize("impl_name", ["auto", "tcgen05", "simt"])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("ramp", ["rising", "falling"])
def test_scores_far_beyond_exp2_range(impl_name, causal, ramp):
    """Keys scaled by a factor ramping between 1 and 40 along the sequence, so
    that a row's scores differ by far more than exp2's range (over 100 in
    log2 units).  Rising: later key blocks exceed the first block's maximum
    and the softmax must move its exponent offset and rescale O; falling: the
    first block dominates and later blocks underflow.  Compared with the fp64
    oracle, which subtracts the exact maximum.

    Attention this peaked makes |out| approach max|v| (about 4.5 here), so the
    bf16 bound scales with it: the rounding of P to bf16 (2^-9 relative per
    weight), of a parked pattern's partial row and of the output each add at
    most 2^-9 max|v|; the test allows 3 * 2^-9 * max|v| (10 % margin), and
    never less than the default 2e-2."""
    B, N, H, D = 1, 2048, 4, 64
    pats = ((512, 1), (1024, 2), (2048, 4))
    q, k, v = wl.random_inputs(B, N, H, D, torch.float32, seed=4242 + causal)
    f = torch.linspace(1.0, 40.0, N) if ramp == "rising" else torch.linspace(40.0, 1.0, N)
    k = k * f.view(1, N, 1, 1)
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    o, l = gh.run_cuda(q, k, v, pats, causal, IMPLS[impl_name] if impl_name != "auto" else bd.LONGNET_IMPL_AUTO)
    tol = max(gh.TOL_OUT[torch.bfloat16], 1.1 * 3 * 2.0 ** -9 * float(v.float().abs().max()))
    err = gh.compare_full(o, l, q, k, v, pats, causal, torch.bfloat16,
                          label=f"ramp_{ramp}_{causal}/{impl_name}", tol_out=tol)
    print(f"ramp_{ramp} causal={causal} {impl_name}: max|out - oracle| = {err:.3e} (bound {tol:.3e})")


def test_repeated_shape_with_new_tensors():
    """The launcher keeps the host set-up of the last shape and tensors: the
    same shape with other tensors (and back) must still read the new ones."""
    B, N, H, D = 1, 1024, 3, 64
    pats = ((256, 1), (512, 2), (1024, 4))
    sets = [wl.random_inputs(B, N, H, D, torch.bfloat16, seed=s) for s in (11, 12)]
    for q, k, v in (sets[0], sets[1], sets[0], sets[1]):
        for impl in (bd.LONGNET_IMPL_TCGEN05, bd.LONGNET_IMPL_AUTO):
            o, l = gh.run_cuda(q, k, v, pats, True, impl)
            gh.compare_full(o, l, q, k, v, pats, True, torch.bfloat16, label=f"repeat/{impl}")


QK_NORM_CASES = [
    # name, B, N, H, D, dtype, causal, patterns
    ("smallseg_shape_bf16", 4, 1024, 4, 64, torch.bfloat16, False, ((64, 1), (64, 2))),
    ("smallseg_shape_f16_causal", 2, 512, 3, 64, torch.float16, True, ((32, 1), (32, 4))),
    ("lm_like_bf16", 1, 1024, 3, 64, torch.bfloat16, True, ((256, 1), (512, 2), (1024, 4))),
    ("paper_like_f16_partial", 1, 3000, 4, 64, torch.float16, True, ((256, 1), (512, 2), (1024, 4), (3000, 6))),
    ("long_noncausal_bf16", 2, 2048, 2, 64, torch.bfloat16, False, ((512, 1), (2048, 4))),
    # six patterns: the fused kernel's streams get 3 + 2 ring stages
    ("six_patterns_bf16", 1, 3072, 2, 64, torch.bfloat16, True,
     ((256, 1), (512, 2), (768, 3), (1024, 4), (1536, 6), (3072, 12))),
    ("fp32_d32", 1, 384, 2, 32, torch.float32, True, ((96, 1), (192, 5), (384, 7))),
    # head sizes other than 64: the per-pattern family (several tiles, a partial one)
    ("d128_bf16", 1, 1280, 2, 128, torch.bfloat16, True, ((256, 1), (1280, 4))),
    ("d32_f16_noncausal", 2, 640, 3, 32, torch.float16, False, ((128, 1), (640, 2))),
    ("d16_bf16", 1, 896, 2, 16, torch.bfloat16, True, ((256, 1), (896, 3))),
]


@pytest.mark.parametrize("case", QK_NORM_CASES, ids=[c[0] for c in QK_NORM_CASES])
def test_qk_norm_option(case):
    """LONGNET_FLAG_QK_NORM on raw q and k (rows of norm about 3*sqrt(D); v
    of unit scale, so the 16-bit bounds keep their meaning), against the
    oracle with its q, k rows normalised in fp64; AUTO, SIMT, the small-
    segment kernel, the tcgen05 and the per-pattern kernels (which scale the
    scores by the rows' inverse norms) take it where they take the shape."""
    name, B, N, H, D, dtype, causal, pats = case
    seed = zlib.crc32(name.encode()) % 100000
    q, k, _ = wl.random_inputs(B, N, H, D, dtype, seed=seed, scale=3.0)
    _, _, v = wl.random_inputs(B, N, H, D, dtype, seed=seed + 1)
    for impl in (bd.LONGNET_IMPL_AUTO, bd.LONGNET_IMPL_SIMT, bd.LONGNET_IMPL_SMALLSEG, bd.LONGNET_IMPL_TCGEN05,
                 bd.LONGNET_IMPL_PATTERNS):
        try:
            o, l = gh.run_cuda(q, k, v, pats, causal, impl, qk_norm=True)
        except bd.LongNetError as e:
            assert impl in (bd.LONGNET_IMPL_SMALLSEG, bd.LONGNET_IMPL_TCGEN05, bd.LONGNET_IMPL_PATTERNS)
            assert e.code == bd.LONGNET_ERR_UNSUPPORTED
            continue
        gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"qk_norm {name}/{impl}", qk_norm=True)


def test_named_tiny_workload_fp32():
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.make_inputs(w)
    o, l = gh.run_cuda(q, k, v, w.patterns, w.causal, bd.LONGNET_IMPL_AUTO)
    err = gh.compare_full(o, l, q, k, v, w.patterns, w.causal, torch.float32, "tiny")
    assert err <= 1e-4


@pytest.mark.parametrize("name,impl_name", [("lm", "auto"), ("long32k", "auto"), ("smallseg", "auto"),
                                             ("lm", "patterns"), ("long32k", "patterns")])
def test_named_workloads_every_element(name, impl_name):
    """Full-size workloads in the launch configuration the benchmark times
    (AUTO), and on the per-pattern family, every element of out and lse
    against the full fp64 oracle."""
    w = wl.WORKLOADS[name]
    q, k, v = wl.make_inputs(w)
    impl = bd.LONGNET_IMPL_AUTO if impl_name == "auto" else IMPLS[impl_name]
    o, l = gh.run_cuda(q, k, v, w.patterns, w.causal, impl)
    assert gh.lse_is_finite_everywhere(l)  # every row is kept by an r = 1 pattern
    err = gh.compare_full(o, l, q, k, v, w.patterns, w.causal, torch.bfloat16, label=f"{name}/{impl_name}")
    print(f"{name}/{impl_name}: max|out - oracle| = {err:.3e} over {o.size} elements")


@pytest.mark.parametrize("N", wl.SWEEP_NS)
def test_sweep_sampled_rows(N):
    """The linear-scaling sweep (to 1M tokens, six patterns) in the launch
    configuration the benchmark times, on sampled rows: every segment's first
    and last kept row per pattern and head, the rows on both sides of every
    multiple of 2048 positions (range and split points of the work units for
    every r_max <= 32), and random rows."""
    w = wl.sweep_workload(N)
    q, k, v = wl.make_inputs(w)
    o, l = gh.run_cuda(q, k, v, w.patterns, w.causal, bd.LONGNET_IMPL_AUTO)
    assert gh.lse_is_finite_everywhere(l)
    rows = gh.sample_rows(w.B, w.N, w.H, w.patterns, n_random=1000, seed=w.seed + N, boundary=4096)
    err = gh.compare_rows(o, l, q, k, v, w.patterns, w.causal, torch.bfloat16, rows, label=f"sweep{N}")
    print(f"sweep{N}: max|out - oracle| = {err:.3e} over {len(rows)} rows")


@pytest.mark.parametrize("impl_name", ["auto", "patterns"])
@pytest.mark.parametrize("causal", [True, False])
def test_partial_last_segments_full_size(causal, impl_name):
    """The 32K-token shape 64 positions short, so every pattern's last segment
    is cut by the sequence's end (and the longest segment exceeds it), in the
    benchmark's launch configuration (AUTO): sampled rows, including every
    segment's first and last kept row and all rows of the last 2048
    positions, against the oracle."""
    w = wl.WORKLOADS["long32k"]
    N = w.N - 64
    q, k, v = wl.make_inputs(w, N=N)
    impl = bd.LONGNET_IMPL_AUTO if impl_name == "auto" else IMPLS[impl_name]
    o, l = gh.run_cuda(q, k, v, w.patterns, causal, impl)
    rows = gh.sample_rows(w.B, N, w.H, w.patterns, n_random=1000, seed=17, boundary=4096)
    tail = np.array([(0, x, h) for x in range(N - 2048, N) for h in range(w.H)], dtype=np.int64)
    rows = np.unique(np.concatenate([rows, tail]), axis=0)
    err = gh.compare_rows(o, l, q, k, v, w.patterns, causal, torch.bfloat16, rows, label=f"long32k-64/{causal}")
    print(f"long32k-64 causal={causal} {impl_name}: max|out - oracle| = {err:.3e} over {len(rows)} rows")


def test_lse_optional_and_deterministic():
    pats = ((256, 1), (512, 2), (1024, 4))
    q, k, v = wl.random_inputs(1, 1024, 4, 64, torch.bfloat16, seed=5)
    o1, _ = gh.run_cuda(q, k, v, pats, True, bd.LONGNET_IMPL_AUTO, want_lse=False)
    o2, l2 = gh.run_cuda(q, k, v, pats, True, bd.LONGNET_IMPL_AUTO, want_lse=True)
    assert np.array_equal(o1, o2), "two runs differ"
    gh.compare_full(o2, l2, q, k, v, pats, True, torch.bfloat16, "lse_optional")


def test_runs_on_a_side_stream():
    pats = ((128, 1), (256, 2))
    q, k, v = wl.random_inputs(1, 512, 2, 64, torch.bfloat16, seed=6)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, l = gh.run_cuda(q, k, v, pats, True, bd.LONGNET_IMPL_AUTO, stream=s)
    gh.compare_full(o, l, q, k, v, pats, True, torch.bfloat16, "side_stream")


def test_misaligned_device_pointer_rejected():
    dev = torch.device("cuda:0")
    buf = torch.zeros(1 * 64 * 2 * 16 + 8, dtype=torch.float32, device=dev)
    x = buf[1:1 + 64 * 2 * 16].view(1, 64, 2, 16)  # 4-byte offset
    with pytest.raises(bd.LongNetError) as ei:
        bd.longnet_dilated_attn_fwd(x, x, x, x, None, ((64, 1),), True)
    assert ei.value.code == bd.LONGNET_ERR_MISALIGNED


def test_watchdog_timeout_is_reported_and_context_survives():
    assert bd.longnet_last_device_status() == 0
    assert bd.longnet_watchdog_selftest(200_000) == 0
    assert bd.longnet_last_device_status() == bd.LONGNET_ERR_DEVICE_TIMEOUT
    assert bd.longnet_last_device_status() == 0  # cleared
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.make_inputs(w)
    o, l = gh.run_cuda(q, k, v, w.patterns, w.causal, bd.LONGNET_IMPL_AUTO)
    gh.compare_full(o, l, q, k, v, w.patterns, w.causal, torch.float32, "after_watchdog")


def _random_config(seed):
    """A seeded random problem: dtype, D, B, H, N, 1..5 patterns (w may or may
    not divide N, r may exceed w), causal or full; sized for the oracle."""
    g = np.random.default_rng(1000 + seed)
    dtype = [torch.float32, torch.bfloat16, torch.float16][seed % 3]
    D = 64 if (dtype != torch.float32 and g.random() < 0.8) else int(g.choice([16, 32, 64, 128]))
    B, H = int(g.integers(1, 3)), int(g.integers(1, 7))
    n_pat = int(g.integers(1, 6))
    if g.random() < 0.3:  # one shared short segment (the small-segment shape)
        W = int(g.choice([8, 16, 24, 32, 40, 48, 56, 64]))
        N = W * int(g.integers(2, 24))
        rs = [1] + [int(g.integers(2, 9)) for _ in range(n_pat - 1)]
        pats = tuple((W, r) for r in rs)
    else:
        N = int(g.choice([256, 384, 512, 640, 768, 1024, 1536, 2048]))
        if g.random() < 0.2:
            N += int(g.integers(1, 64))  # partial last segments
        pats = []
        for _ in range(n_pat):
            r = int(g.choice([1, 1, 2, 3, 4, 5, 8, 12]))
            w = int(g.choice([64, 128, 192, 256, 512, 1024, 2048]))
            pats.append((min(w, max(N // 2, 64)) if g.random() < 0.5 else w, r))
        pats = tuple(pats)
    causal = bool(g.random() < 0.7)
    return dtype, D, B, H, N, pats, causal


@pytest.mark.parametrize("seed", range(24))
def test_random_configurations_every_family(seed):
    """Seeded random shapes through AUTO and through every family that takes
    them; a family that declines returns UNSUPPORTED."""
    dtype, D, B, H, N, pats, causal = _random_config(seed)
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=7000 + seed)
    label = f"seed{seed} {dtype} D{D} B{B} H{H} N{N} {pats} causal={causal}"
    ro, rl = None, None
    for impl in (bd.LONGNET_IMPL_AUTO, bd.LONGNET_IMPL_SIMT, bd.LONGNET_IMPL_TCGEN05, bd.LONGNET_IMPL_SMALLSEG):
        try:
            o, l = gh.run_cuda(q, k, v, pats, causal, impl)
        except bd.LongNetError as e:
            assert impl not in (bd.LONGNET_IMPL_AUTO, bd.LONGNET_IMPL_SIMT) and e.code == bd.LONGNET_ERR_UNSUPPORTED, \
                f"{label}: impl {impl} -> {e}"
            continue
        gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"{label} impl={impl}")
