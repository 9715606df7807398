"""GPU parity of the backward (dq, dk, dv) through the C ABI against the fp64
oracle's backward on the same seeded inputs (needs a B200).

The CUDA backward takes the CUDA forward's out and lse, as a training step
would; the oracle recomputes its own forward in fp64, so nothing from the
CUDA path enters the reference.  The gradients come back in fp32.
Tolerance, per gradient, on max|g - ref| / max(1, max|ref|):
  - SIMT: delta_i = <dout_i, out_i> uses the forward's out rounded to the
    input format (2^-9 relative for bf16, 2^-11 for fp16); fp32 accumulation
    adds ~1e-6.  Measured 0.3 % (bf16) on an fp32 emulation.
  - Tiles and tcgen05: P and dS are rounded to the input format before their
    products (again 2^-9 / 2^-11 relative, once per pair, averaging out over
    the sum).
1e-2 (bf16), 2e-3 (fp16) and 1e-4 (fp32) hold these with a margin of about 3.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_attn_b200 import binding as bd
from sparse_long_sequence_attn_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

TOL_GRAD = {torch.float32: 1e-4, torch.bfloat16: 1e-2, torch.float16: 2e-3}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    bd.load_library()
    yield


def run_cuda_bwd(q, k, v, dout, patterns, causal, impl=bd.LONGNET_IMPL_AUTO, qk_norm=False):
    """CUDA forward (AUTO family) then the backward into NaN-guarded fp32
    buffers; checks the guards and the status word; returns CPU float64
    (dq, dk, dv)."""
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (x.to(dev).contiguous() for x in (q, k, v, dout))
    out, lse = bd.dilated_attn(qd, kd, vd, patterns, causal, qk_norm=qk_norm)
    n = q.numel()
    G = gh.GUARD
    bufs = [torch.full((n + 2 * G,), float("nan"), dtype=torch.float32, device=dev) for _ in range(3)]
    views = [b[G:G + n].view(q.shape) for b in bufs]
    bd.longnet_dilated_attn_bwd(qd, kd, vd, out, lse, dod, *views, patterns, causal, impl,
                                qk_norm=qk_norm)
    st = bd.longnet_last_device_status(None)
    assert st == 0, f"device status word: {bd.status_string(st)}"
    for b in bufs:
        assert torch.isnan(b[:G]).all() and torch.isnan(b[-G:]).all(), "write outside a gradient"
    res = [x.double().cpu().numpy() for x in views]
    for x in res:
        assert not np.isnan(x).any(), "some gradient rows were never written"
    return res


def check(got, ref, dtype, label):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        err = float(np.abs(g - r).max())
        bound = TOL_GRAD[dtype] * max(1.0, float(np.abs(r).max()))
        assert err <= bound, f"{label} {name}: max err {err} > {bound}"


# name, B, N, H, D, dtype, causal, patterns
CASES = [
    ("tiny_cfg", 1, 256, 2, 16, torch.float32, True, ((64, 1), (128, 2), (256, 4))),
    ("fp32_d32_rdivw", 2, 384, 3, 32, torch.float32, True, ((96, 1), (192, 5), (384, 7))),
    ("fp32_d64_noncausal", 1, 512, 2, 64, torch.float32, False, ((128, 1), (256, 3))),
    ("fp32_d128_uncovered", 1, 240, 3, 128, torch.float32, True, ((48, 3), (240, 4))),
    ("fp32_partial_segments", 1, 300, 3, 32, torch.float32, True, ((64, 1), (128, 3), (512, 5))),
    ("bf16_d64_lm_like", 2, 1024, 4, 64, torch.bfloat16, True, ((256, 1), (512, 2), (1024, 4))),
    ("bf16_d64_paper_like", 1, 1536, 6, 64, torch.bfloat16, True,
     ((128, 1), (256, 2), (512, 4), (768, 6), (1536, 12))),
    ("bf16_d64_dup_unordered", 1, 512, 3, 64, torch.bfloat16, True, ((512, 4), (128, 1), (128, 1))),
    ("bf16_d64_smallseg_noncausal", 2, 1024, 4, 64, torch.bfloat16, False, ((64, 1), (64, 2))),
    ("bf16_d32_partial", 1, 700, 2, 32, torch.bfloat16, False, ((128, 1), (300, 2))),
    ("f16_d64_r_not_dividing", 1, 768, 5, 64, torch.float16, True, ((192, 3), (384, 4), (768, 8))),
    ("f16_d128", 1, 256, 2, 128, torch.float16, True, ((64, 1), (256, 2))),
    ("bf16_d128_lm_like", 1, 1024, 3, 128, torch.bfloat16, True, ((256, 1), (512, 2), (1024, 4))),
    ("bf16_d128_noncausal_partial", 2, 700, 2, 128, torch.bfloat16, False, ((256, 1), (300, 3))),
    # narrow heads on the tensor cores: one 64- or 32-byte swizzle panel per row
    ("bf16_d32_lm_like", 1, 1024, 3, 32, torch.bfloat16, True, ((256, 1), (512, 2), (1024, 4))),
    ("f16_d32_noncausal", 2, 512, 2, 32, torch.float16, False, ((128, 1), (512, 4))),
    ("bf16_d16_causal", 1, 1024, 4, 16, torch.bfloat16, True, ((256, 1), (1024, 4))),
]


def _impls(dtype, D):
    out = [("simt", bd.LONGNET_IMPL_SIMT)]
    if dtype != torch.float32 and D == 64:
        out.append(("tiles", bd.LONGNET_IMPL_TILES))
    if dtype != torch.float32 and D in (16, 32, 64, 128):
        out.append(("tcgen05", bd.LONGNET_IMPL_TCGEN05))
    return out


def run_or_skip(q, k, v, dout, pats, causal, impl, qk_norm=False):
    try:
        return run_cuda_bwd(q, k, v, dout, pats, causal, impl, qk_norm)
    except bd.LongNetError as e:
        if e.code == bd.LONGNET_ERR_UNSUPPORTED:
            pytest.skip("the family does not take this case")
        raise


PARAMS = [(c, nm, code) for c in CASES for (nm, code) in _impls(c[5], c[4])]


@pytest.mark.parametrize("case,impl_name,impl", PARAMS,
                         ids=[f"{c[0]}-{nm}" for (c, nm, _) in PARAMS])
def test_backward_matches_oracle(case, impl_name, impl):
    name, B, N, H, D, dtype, causal, pats = case
    seed = zlib.crc32(name.encode()) % 100000
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=seed)
    dout = wl.random_cotangent(B, N, H, D, dtype, seed=seed)
    got = run_or_skip(q, k, v, dout, pats, causal, impl)
    ref = oracle.dilated_attn_bwd_fp64(q, k, v, dout, pats, causal)
    check(got, ref, dtype, f"{name} ({impl_name})")


def test_auto_picks_tcgen05_for_16bit_d64():
    """AUTO gives the gradients of the forced tcgen05 family on a bf16 D = 64
    case; the tile family agrees within the rounding of P and dS."""
    B, N, H, D = 1, 512, 3, 64
    pats = ((128, 1), (256, 2), (512, 4))
    q, k, v = wl.random_inputs(B, N, H, D, torch.bfloat16, seed=31)
    dout = wl.random_cotangent(B, N, H, D, torch.bfloat16, seed=31)
    a = run_cuda_bwd(q, k, v, dout, pats, True, bd.LONGNET_IMPL_AUTO)
    t = run_cuda_bwd(q, k, v, dout, pats, True, bd.LONGNET_IMPL_TCGEN05)
    for x, y in zip(a, t):
        # fp32 atomics across patterns: equal up to the order of at most 3 adds
        assert np.abs(x - y).max() <= 1e-5 * max(1.0, np.abs(y).max())
    m = run_cuda_bwd(q, k, v, dout, pats, True, bd.LONGNET_IMPL_TILES)
    for x, y in zip(m, t):
        assert np.abs(x - y).max() <= TOL_GRAD[torch.bfloat16] * max(1.0, np.abs(y).max())


def test_tensor_core_families_ragged_and_many_tiles():
    """Segments of 2731 and 2730 kept rows (43 tiles, ragged last tile), partial
    segments, N mod r != 0, non-causal, fp16 and bf16, on both tensor-core
    families."""
    cases = [
        (1, 4096, 2, torch.bfloat16, True, ((4096, 1), (2048, 2), (4000, 3))),
        (1, 1500, 3, torch.float16, False, ((700, 1), (1500, 5))),
        (2, 800, 2, torch.bfloat16, True, ((800, 12), (96, 1))),
    ]
    for i, (B, N, H, dtype, causal, pats) in enumerate(cases):
        q, k, v = wl.random_inputs(B, N, H, 64, dtype, seed=50 + i)
        dout = wl.random_cotangent(B, N, H, 64, dtype, seed=50 + i)
        ref = oracle.dilated_attn_bwd_fp64(q, k, v, dout, pats, causal)
        for impl_name, impl in (("tiles", bd.LONGNET_IMPL_TILES), ("tcgen05", bd.LONGNET_IMPL_TCGEN05)):
            try:
                got = run_cuda_bwd(q, k, v, dout, pats, causal, impl)
            except bd.LongNetError as e:
                # tcgen05 declines N < 128 r + 2 (N mod r): (800, 12) here
                assert impl_name == "tcgen05" and e.code == bd.LONGNET_ERR_UNSUPPORTED and i == 2
                continue
            check(got, ref, dtype, f"ragged case {i} ({impl_name})")


def test_uncovered_rows_get_zero_gradients():
    B, N, H, D = 1, 240, 3, 64
    pats = ((48, 3), (240, 4))
    q, k, v = wl.random_inputs(B, N, H, D, torch.bfloat16, seed=5)
    dout = wl.random_cotangent(B, N, H, D, torch.bfloat16, seed=5)
    _, lse = oracle.dilated_attn_fp64(q, k, v, pats, True)
    kept = np.isfinite(lse).transpose(0, 2, 1)
    assert (~kept).any()
    for impl in (bd.LONGNET_IMPL_SIMT, bd.LONGNET_IMPL_TILES, bd.LONGNET_IMPL_TCGEN05):
        got = run_cuda_bwd(q, k, v, dout, pats, True, impl)
        for g in got:
            assert not g[~kept].any()


def test_autograd_function_matches_direct_calls():
    B, N, H, D = 1, 512, 4, 64
    pats = ((128, 1), (256, 2), (512, 4))
    q, k, v = (x.cuda().requires_grad_(True)
               for x in wl.random_inputs(B, N, H, D, torch.bfloat16, seed=17))
    dout = wl.random_cotangent(B, N, H, D, torch.bfloat16, seed=17).cuda()
    out = bd.dilated_attention(q, k, v, pats, True)
    (out.float() * dout.float()).sum().backward()
    with torch.no_grad():
        o2, l2 = bd.dilated_attn(q.detach(), k.detach(), v.detach(), pats, True)
        dq, dk, dv = bd.dilated_attn_bwd(q.detach(), k.detach(), v.detach(), o2, l2, dout, pats, True)
    assert torch.equal(out.detach(), o2)
    for a, b in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        assert a.dtype == torch.bfloat16
        # fp32 atomics across patterns: equal up to the order of the adds
        assert (a.float() - b.to(torch.bfloat16).float()).abs().max() <= 1e-2 * max(1.0, b.abs().max().item())


@pytest.mark.parametrize("name", ["lm", "long32k"])
def test_backward_full_size_sampled_rows(name):
    """The bench workloads at full size: the gradients of sampled rows against
    the oracle's per-row backward.  Rows at the ends of every pattern's first
    segment (many keys as queries, few queries as keys), rows at the starts of
    segments (every query of the segment reaches them) and random rows near the
    end of the sequence."""
    w = wl.WORKLOADS[name]
    q, k, v = wl.make_inputs(w)
    dout = wl.random_cotangent(w.B, w.N, w.H, w.D, w.torch_dtype, seed=w.seed)
    got = run_cuda_bwd(q, k, v, dout, w.patterns, w.causal)
    g = np.random.default_rng(w.seed)
    rows = []
    for h in (0, w.H - 1):
        for (wp, rp) in w.patterns:
            o = h % rp
            last = wp - 1 - ((wp - 1 - o) % rp)  # last kept row of segment 0
            rows.append((w.B - 1, last, h))
    for _ in range(4):
        rows.append((int(g.integers(w.B)), int(w.N - 1 - g.integers(256)), int(g.integers(w.H))))
    # first kept row of a segment of the densest pattern: every query of the
    # segment reaches it as a key
    w0, r0 = w.patterns[0]
    rows.append((0, w0, 0))
    rows.append((w.B - 1, w.N - w0 + (w.H - 1) % r0, w.H - 1))
    rows = np.array(sorted(set(rows)), dtype=np.int64)
    ref = oracle.dilated_attn_bwd_rows_fp64(q, k, v, dout, w.patterns, rows, w.causal)
    b, pos, h = rows[:, 0], rows[:, 1], rows[:, 2]
    for nm, full, r in zip(("dq", "dk", "dv"), got, ref):
        err = float(np.abs(full[b, pos, h] - r).max())
        bound = TOL_GRAD[w.torch_dtype] * max(1.0, float(np.abs(r).max()))
        assert err <= bound, f"{name} {nm}: max err {err} > {bound} over {len(rows)} rows"


# qk_norm: q and k rows scaled to unit L2 norm before the scores, gradients
# taken back through the normalisation.  Inputs are drawn at scale 3 so the
# norms are far from 1; one zero key row takes the 1/eps branch (its dk is
# compared relatively: it is dkhat / 1e-12).
QK_NORM_CASES = [
    ("qkn_bf16_lm_like", 1, 512, 3, 64, torch.bfloat16, True, ((128, 1), (256, 2), (512, 4))),
    ("qkn_f16_noncausal_small", 2, 256, 4, 64, torch.float16, False, ((64, 1), (64, 2))),
    ("qkn_fp32_d32_partial", 1, 300, 3, 32, torch.float32, True, ((64, 1), (128, 3), (512, 5))),
]
QKN_PARAMS = [(c, nm, code) for c in QK_NORM_CASES for (nm, code) in _impls(c[5], c[4])]


@pytest.mark.parametrize("case,impl_name,impl", QKN_PARAMS,
                         ids=[f"{c[0]}-{nm}" for (c, nm, _) in QKN_PARAMS])
def test_backward_qk_norm(case, impl_name, impl):
    name, B, N, H, D, dtype, causal, pats = case
    seed = zlib.crc32(name.encode()) % 100000
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=seed, scale=3.0)
    dout = wl.random_cotangent(B, N, H, D, dtype, seed=seed)
    k[0, 5, 1] = 0.0  # a zero key row
    got = run_or_skip(q, k, v, dout, pats, causal, impl, qk_norm=True)
    ref = oracle.dilated_attn_bwd_fp64(q, k, v, dout, pats, causal, qk_norm=True)
    zero = got[1][0, 5, 1].copy(), ref[1][0, 5, 1].copy()
    got[1][0, 5, 1] = ref[1][0, 5, 1] = 0.0
    check(got, ref, dtype, f"{name} ({impl_name})")
    bound = 10 * TOL_GRAD[dtype] * max(1.0, float(np.abs(zero[1]).max()))
    assert np.abs(zero[0] - zero[1]).max() <= bound, "zero key row (1/eps branch)"


# The backward of the workspace forward (longnet_dilated_attn_fwd_ws): the
# options qk_norm and XPOS on the encoded rows, gradients taken back through
# them, against the oracle's backward with the same options.
WS_CASES = [
    ("ws_bf16_d64_lm_like", 1, 1024, 3, 64, torch.bfloat16, True, ((256, 1), (512, 2), (1024, 4))),
    ("ws_f16_d64_noncausal", 2, 512, 2, 64, torch.float16, False, ((128, 1), (512, 4))),
    ("ws_bf16_d128", 1, 1024, 2, 128, torch.bfloat16, True, ((256, 1), (1024, 2))),
    ("ws_fp32_d32_partial", 1, 300, 2, 32, torch.float32, True, ((64, 1), (128, 3))),
    ("ws_bf16_d32", 1, 1024, 2, 32, torch.bfloat16, True, ((256, 1), (1024, 4))),
]
WS_OPTIONS = {"qk_norm": (True, False), "xpos": (False, True), "both": (True, True)}


@pytest.mark.parametrize("case", WS_CASES, ids=[c[0] for c in WS_CASES])
@pytest.mark.parametrize("opt", sorted(WS_OPTIONS))
@pytest.mark.parametrize("impl_name", ["auto", "tcgen05", "tiles", "simt"])
def test_backward_through_the_prologue(case, opt, impl_name):
    name, B, N, H, D, dtype, causal, pats = case
    qk_norm, xpos = WS_OPTIONS[opt]
    impl = {"auto": bd.LONGNET_IMPL_AUTO, "tcgen05": bd.LONGNET_IMPL_TCGEN05, "tiles": bd.LONGNET_IMPL_TILES,
            "simt": bd.LONGNET_IMPL_SIMT}[impl_name]
    seed = zlib.crc32((name + opt).encode()) % 100000
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=seed, scale=3.0 if qk_norm else 1.0)
    dout = wl.random_cotangent(B, N, H, D, dtype, seed=seed)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (x.to(dev).contiguous() for x in (q, k, v, dout))
    out, lse = bd.dilated_attn(qd, kd, vd, pats, causal, qk_norm=qk_norm, xpos=xpos)
    n = q.numel()
    G = gh.GUARD
    bufs = [torch.full((n + 2 * G,), float("nan"), dtype=torch.float32, device=dev) for _ in range(3)]
    views = [b[G:G + n].view(q.shape) for b in bufs]
    ws = torch.empty(bd.longnet_fwd_workspace_bytes(B, N, H, D, dtype, qk_norm, xpos), dtype=torch.uint8,
                     device=dev)
    try:
        bd.longnet_dilated_attn_bwd_ws(qd, kd, vd, out, lse, dod, *views, pats, causal, ws, impl,
                                       qk_norm=qk_norm, xpos=xpos)
    except bd.LongNetError as e:
        if e.code == bd.LONGNET_ERR_UNSUPPORTED:
            pytest.skip("the family does not take this case")
        raise
    assert bd.longnet_last_device_status() == 0
    for b in bufs:
        assert torch.isnan(b[:G]).all() and torch.isnan(b[-G:]).all(), "write outside a gradient"
    got = [x.double().cpu().numpy() for x in views]
    ref = oracle.dilated_attn_bwd_fp64(q, k, v, dout, pats, causal, qk_norm=qk_norm, xpos=xpos)
    check(got, ref, dtype, f"{name}/{opt} ({impl_name})")


def test_autograd_with_xpos_matches_direct_calls():
    B, N, H, D = 1, 1024, 2, 64
    pats = ((256, 1), (1024, 4))
    q, k, v = (x.cuda().requires_grad_(True) for x in wl.random_inputs(B, N, H, D, torch.bfloat16, seed=23))
    dout = wl.random_cotangent(B, N, H, D, torch.bfloat16, seed=23).cuda()
    out = bd.dilated_attention(q, k, v, pats, True, qk_norm=True, xpos=True)
    (out.float() * dout.float()).sum().backward()
    with torch.no_grad():
        o2, l2 = bd.dilated_attn(q.detach(), k.detach(), v.detach(), pats, True, qk_norm=True, xpos=True)
        dq, dk, dv = bd.dilated_attn_bwd(q.detach(), k.detach(), v.detach(), o2, l2, dout, pats, True,
                                         qk_norm=True, xpos=True)
    assert torch.equal(out.detach(), o2)
    for a, b in ((q.grad, dq), (k.grad, dk), (v.grad, dv)):
        assert (a.float() - b.to(torch.bfloat16).float()).abs().max() <= 1e-2 * max(1.0, b.abs().max().item())
