"""The input-side options through the prologue pass (longnet_dilated_attn_fwd_ws):
qk_norm and XPOS on q and k written to a workspace, then any attention
family on it, against the fp64 oracle with the same options."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_attn_b200 import binding as bd
from sparse_long_sequence_attn_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

IMPLS = {"auto": bd.LONGNET_IMPL_AUTO, "simt": bd.LONGNET_IMPL_SIMT, "tcgen05": bd.LONGNET_IMPL_TCGEN05,
         "smallseg": bd.LONGNET_IMPL_SMALLSEG}
OPTIONS = {"qk_norm": (True, False), "xpos": (False, True), "both": (True, True)}
GUARD = 4096  # bytes of NaN guard on each side of the workspace


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    bd.load_library()
    yield


CASES = [
    # name, B, N, H, D, dtype, causal, patterns
    ("bf16_lm_like", 2, 2048, 4, 64, torch.bfloat16, True, ((512, 1), (1024, 2), (2048, 4))),
    ("bf16_noncausal", 1, 1024, 3, 64, torch.bfloat16, False, ((256, 1), (512, 4))),
    ("f16_small", 1, 1024, 4, 64, torch.float16, True, ((256, 1), (512, 2))),
    ("bf16_seg64", 2, 1024, 4, 64, torch.bfloat16, True, ((64, 1), (64, 2))),
    ("fp32_d32", 1, 512, 2, 32, torch.float32, True, ((128, 1), (512, 2))),
    ("fp32_d128_partial", 1, 300, 2, 128, torch.float32, False, ((64, 1), (128, 3))),
    ("bf16_d16", 1, 512, 2, 16, torch.bfloat16, True, ((128, 1), (512, 4))),
]


def run_ws(q, k, v, pats, causal, impl, qk_norm, xpos):
    """Forward through the workspace entry with NaN guards around out and the
    workspace; returns (out, lse, transformed q, transformed k) on the CPU."""
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    B, N, H, D = q.shape
    nbytes = bd.longnet_fwd_workspace_bytes(B, N, H, D, q.dtype, qk_norm, xpos)
    assert nbytes >= 2 * q.numel() * q.element_size()
    wbuf = torch.full((nbytes + 2 * GUARD,), 0xFF, dtype=torch.uint8, device=dev)
    ws = wbuf[GUARD:GUARD + nbytes]
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    bd.longnet_dilated_attn_fwd_ws(qd, kd, vd, out, lse, pats, causal, ws, impl, qk_norm=qk_norm, xpos=xpos)
    st = bd.longnet_last_device_status()
    assert st == 0, bd.status_string(st)
    assert (wbuf[:GUARD] == 0xFF).all() and (wbuf[-GUARD:] == 0xFF).all(), "write outside the workspace"
    half = nbytes // 2
    qt = ws[:q.numel() * q.element_size()].view(q.dtype).view(q.shape).float().cpu().numpy()
    kt = ws[half:half + k.numel() * k.element_size()].view(k.dtype).view(k.shape).float().cpu().numpy()
    return out.float().cpu().numpy(), lse.cpu().numpy(), qt, kt


def _expected_qk(q, k, qk_norm, xpos):
    qq, kk = oracle.oracle._f64(q), oracle.oracle._f64(k)
    if qk_norm:
        qq, kk = oracle.qk_normalize_fp64(qq), oracle.qk_normalize_fp64(kk)
    if xpos:
        qq, kk = oracle.xpos_fp64(qq), oracle.xpos_fp64(kk, downscale=True)
    return qq, kk


# a transformed element is the fp32 result rounded once to the input format
ROUND = {torch.float32: 2.0 ** -20, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -10}


def xpos_growth(pats, N, causal):
    """Largest factor by which XPOS scales a score above its unscaled size:
    zeta_0^((m - n) / 512) for a key n after the row m (non-causal only),
    n - m up to the longest segment.  The rounding error of the encoded
    rows, relative to each product, grows with the scores by this factor."""
    if causal:
        return 1.0
    far = min(max(w for w, _ in pats), N) - 1
    return (0.4 / 1.4) ** (-far / 512.0)


def lse_tolerance(q, k, rows, dtype, qk_norm, xpos, causal):
    """Per-row lse tolerance: the parity bar TOL_LSE or, where the scores come
    from XPOS rows the prologue rounded to a 16-bit format, the bound that
    rounding sets.  A transformed element carries a relative error of at
    most u = ROUND[dtype] / 2, so the product q~_i k~_i is off by at most
    2u |q~_i| |k~_i| (first order), a score by at most
    2u / sqrt(D) sum_i |q~_i| |k~_i|, and lse (a soft maximum of the row's
    scores) by at most the largest such move over the keys, bounded here by
    the largest over all keys (all keys at or before the row when causal)."""
    tol = np.full(len(rows), gh.TOL_LSE)
    if not xpos or dtype == torch.float32:
        return tol
    qq, kk = oracle.oracle._f64(q), oracle.oracle._f64(k)
    if qk_norm:
        qq, kk = oracle.qk_normalize_fp64(qq), oracle.qk_normalize_fp64(kk)
    qa, ka = np.abs(oracle.xpos_fp64(qq)), np.abs(oracle.xpos_fp64(kk, downscale=True))
    D, N = q.shape[-1], q.shape[1]
    rows = np.asarray(rows)
    for b in np.unique(rows[:, 0]):
        for h in np.unique(rows[:, 2]):
            sel = np.nonzero((rows[:, 0] == b) & (rows[:, 2] == h))[0]
            for c0 in range(0, len(sel), 1024):
                part = sel[c0:c0 + 1024]
                m = rows[part, 1]
                move = qa[b, m, h] @ ka[b, :, h].T  # [rows, N]
                if causal:
                    move = np.where(np.arange(N)[None, :] <= m[:, None], move, 0.0)
                bound = ROUND[dtype] / np.sqrt(D) * move.max(axis=1)
                tol[part] = np.maximum(tol[part], 1.01 * bound)
    return tol


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("opt", sorted(OPTIONS))
@pytest.mark.parametrize("impl_name", ["auto", "simt", "tcgen05", "smallseg"])
def test_prologue_then_attention_vs_oracle(case, opt, impl_name):
    name, B, N, H, D, dtype, causal, pats = case
    qk_norm, xpos = OPTIONS[opt]
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=zlib.crc32((name + opt).encode()) % 100000)
    try:
        o, l, qt, kt = run_ws(q, k, v, pats, causal, IMPLS[impl_name], qk_norm, xpos)
    except bd.LongNetError as e:
        if e.code == bd.LONGNET_ERR_UNSUPPORTED:
            pytest.skip(f"{impl_name} does not take {name}")
        raise
    eq, ek = _expected_qk(q, k, qk_norm, xpos)
    for got, want in ((qt, eq), (kt, ek)):
        # relative to each pair's size (XPOS scales pairs by very different factors)
        mag = np.repeat(np.sqrt(want[..., 0::2] ** 2 + want[..., 1::2] ** 2), 2, axis=-1)
        assert (np.abs(got - want) <= 2 * ROUND[dtype] * mag + 1e-30).all(), "prologue rows"
    ro, rl = oracle.dilated_attn_fp64(q, k, v, pats, causal, qk_norm=qk_norm, xpos=xpos)
    err = float(np.abs(o - ro).max())
    tol = gh.TOL_OUT[dtype] * xpos_growth(pats, N, causal) if xpos else gh.TOL_OUT[dtype]
    assert err <= tol, f"{name}/{opt}/{impl_name}: max|out - oracle| = {err} (tolerance {tol})"
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l), fin)
    rows = np.argwhere(np.ones((B, N, H), dtype=bool))
    tol = lse_tolerance(q, k, rows, dtype, qk_norm, xpos, causal).reshape(B, N, H).transpose(0, 2, 1)
    lerr = np.where(fin, np.abs(l - np.where(fin, rl, 0.0)), 0.0)
    assert (lerr <= tol).all(), f"lse off by {lerr.max():.3e} (bound {tol[lerr == lerr.max()].min():.3e})"
    print(f"{name}/{opt}/{impl_name}: max|out - oracle| = {err:.3e}, max|lse - oracle| = {lerr.max():.3e}")


@pytest.mark.parametrize("opt", ["qk_norm", "xpos"])
def test_long32k_options_on_tcgen05_sampled(opt):
    """The 32K-token workload with an option, on the tcgen05 family (forced),
    sampled rows against the oracle."""
    w = wl.WORKLOADS["long32k"]
    qk_norm, xpos = OPTIONS[opt]
    q, k, v = wl.make_inputs(w)
    o, l, _, _ = run_ws(q, k, v, w.patterns, w.causal, bd.LONGNET_IMPL_TCGEN05, qk_norm, xpos)
    rows = gh.sample_rows(w.B, w.N, w.H, w.patterns, n_random=1500, seed=5, boundary=4096)
    ro, rl = oracle.dilated_attn_rows_fp64(q, k, v, w.patterns, rows, w.causal, qk_norm=qk_norm, xpos=xpos)
    b, pos, h = rows[:, 0], rows[:, 1], rows[:, 2]
    err = float(np.abs(o[b, pos, h] - ro).max())
    lerr = np.abs(l[b, h, pos] - rl)
    tol = lse_tolerance(q, k, rows, torch.bfloat16, qk_norm, xpos, w.causal)
    print(f"long32k/{opt}/tcgen05: max|out - oracle| = {err:.3e}, lse {lerr.max():.3e} over {len(rows)} rows")
    assert err <= gh.TOL_OUT[torch.bfloat16] and (lerr <= tol).all()


def test_workspace_checks():
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in wl.random_inputs(1, 1024, 2, 64, torch.bfloat16, seed=9))
    out = torch.empty_like(q)
    pats = ((256, 1),)
    n = bd.longnet_fwd_workspace_bytes(1, 1024, 2, 64, torch.bfloat16, True, False)
    ws = torch.empty(n + 512, dtype=torch.uint8, device=dev)
    with pytest.raises(bd.LongNetError) as e:
        bd.longnet_dilated_attn_fwd_ws(q, k, v, out, None, pats, True, ws[:n - 16], qk_norm=True)
    assert e.value.code == bd.LONGNET_ERR_INVALID_ARG
    with pytest.raises(bd.LongNetError) as e:
        bd.longnet_dilated_attn_fwd_ws(q, k, v, out, None, pats, True, ws[16:16 + n], qk_norm=True)
    assert e.value.code == bd.LONGNET_ERR_MISALIGNED
    # fp16 XPOS beyond the format's range
    qh, kh, vh = (x.to(dev) for x in wl.random_inputs(1, 8192, 1, 64, torch.float16, seed=9))
    n16 = bd.longnet_fwd_workspace_bytes(1, 8192, 1, 64, torch.float16, False, True)
    ws16 = torch.empty(n16, dtype=torch.uint8, device=dev)
    with pytest.raises(bd.LongNetError) as e:
        bd.longnet_dilated_attn_fwd_ws(qh, kh, vh, torch.empty_like(qh), None, pats, True, ws16, xpos=True)
    assert e.value.code == bd.LONGNET_ERR_UNSUPPORTED
    # no options: the workspace is not needed
    bd.longnet_dilated_attn_fwd_ws(q, k, v, out, None, pats, True, None)
    assert bd.longnet_last_device_status() == 0
