"""longnet_dilated_attn_fwd_host: the forward on host tensors, cut into
pieces (batches, positions or heads) whose copies overlap the attention.
Against the oracle on every element, and against the device entry; two calls
in a row on the same staging buffers; pinned and pageable host memory; piece
counts that do not divide the extent."""
import zlib

import numpy as np
import pytest
import torch

from sparse_long_sequence_attn_b200 import binding as bd
from sparse_long_sequence_attn_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    bd.load_library()
    yield


CASES = [
    # name, B, N, H, D, dtype, causal, patterns, pieces, pinned, with lse
    # B = 1, H < 4, causal: ranges of positions (default 8; 3 uneven; one per block of 256)
    ("positions_default", 1, 4096, 3, 64, torch.bfloat16, True, ((512, 1), (1024, 2), (4096, 4)), 0, True, True),
    ("positions_uneven", 1, 2000, 2, 64, torch.bfloat16, True, ((256, 1), (2048, 8)), 3, True, True),
    ("positions_many", 1, 2048, 2, 64, torch.float16, True, ((256, 1), (1024, 4)), 64, True, True),
    # B = 1, H >= 4 or full: ranges of heads
    ("heads_causal_default", 1, 4096, 6, 64, torch.bfloat16, True, ((512, 1), (1024, 2), (4096, 4)), 0, True, True),
    ("heads_uneven", 1, 1024, 6, 64, torch.bfloat16, False, ((256, 1), (512, 2)), 4, True, True),
    ("heads_one_each_no_lse", 1, 512, 5, 32, torch.float32, False, ((128, 1), (512, 4)), 5, True, False),
    # B >= 2: ranges of batches
    ("batches_f16", 3, 1024, 3, 64, torch.float16, False, ((256, 1), (512, 2)), 2, True, True),
    ("batches_smallseg_pageable", 4, 1024, 4, 64, torch.bfloat16, False, ((64, 1), (64, 2)), 0, False, True),
    ("batches_causal_fp32", 2, 512, 3, 32, torch.float32, True, ((128, 1), (512, 4)), 0, True, True),
]


def _host(t, pinned):
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=pinned)
    h.copy_(t)
    return h


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_entry_matches_oracle_and_device_entry(case):
    name, B, N, H, D, dtype, causal, pats, chunk, pinned, with_lse = case
    dev = torch.device("cuda:0")
    seed = zlib.crc32(name.encode()) % 100000
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=seed)
    qh, kh, vh = (_host(x, pinned) for x in (q, k, v))
    out_h = torch.full((B, N, H, D), float("nan"), dtype=dtype, pin_memory=pinned)
    lse_h = torch.full((B, H, N), float("nan"), dtype=torch.float32, pin_memory=pinned) if with_lse else None
    # device staging full of NaN: a row read before its copy arrived, or an
    # output row never written, shows
    qd, kd, vd = (torch.full((B, N, H, D), float("nan"), dtype=dtype, device=dev) for _ in range(3))
    out_d = torch.full((B, N, H, D), float("nan"), dtype=dtype, device=dev)
    lse_d = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev) if with_lse else None
    stream = torch.cuda.Stream(device=dev)
    bd.longnet_dilated_attn_fwd_host(qh, kh, vh, out_h, lse_h, qd, kd, vd, out_d, lse_d, pats, causal,
                                     stream=stream, pieces=chunk)
    stream.synchronize()
    assert bd.longnet_last_device_status(stream) == 0
    o = out_h.float().numpy()
    l = lse_h.numpy() if with_lse else None
    assert not np.isnan(o).any(), "rows never copied back"
    if with_lse:
        assert not np.isnan(l).any(), "lse entries never copied back"
    err = gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"host entry {name}")
    # the device entry on the same inputs: the same kernels over head ranges
    o2, l2 = gh.run_cuda(q, k, v, pats, causal, bd.LONGNET_IMPL_AUTO, want_lse=with_lse)
    d = float(np.abs(o - o2).max())
    assert d <= gh.TOL_OUT[dtype], (name, d)
    if with_lse:
        assert float(np.abs(l - l2).max()) <= gh.TOL_LSE
    print(f"{name}: max|out - oracle| = {err:.3e}, max|out - device entry| = {d:.3e}")


@pytest.mark.parametrize("H", [8, 2], ids=["heads", "positions"])
def test_two_calls_in_a_row_reuse_the_staging_buffers(H):
    """The second call's copies in (and, by positions, the zeroing of the
    key and value rows still to come) wait for the first call's attention
    (the staging buffers are shared), and each call's results are its own."""
    dev = torch.device("cuda:0")
    B, N, D, dtype, pats = 1, 4096, 64, torch.bfloat16, ((512, 1), (2048, 4))
    sets = [wl.random_inputs(B, N, H, D, dtype, seed=s) for s in (31, 32)]
    hosts = [tuple(_host(x, True) for x in s) for s in sets]
    outs = [torch.empty(B, N, H, D, dtype=dtype, pin_memory=True) for _ in range(2)]
    lses = [torch.empty(B, H, N, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    qd, kd, vd, od = (torch.full((B, N, H, D), float("nan"), dtype=dtype, device=dev) for _ in range(4))
    ld = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    for (qh, kh, vh), oh, lh in zip(hosts, outs, lses):
        bd.longnet_dilated_attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, pats, True, stream=stream,
                                         pieces=2)
    stream.synchronize()
    assert bd.longnet_last_device_status(stream) == 0
    for (q, k, v), oh, lh in zip(sets, outs, lses):
        o2, l2 = gh.run_cuda(q, k, v, pats, True, bd.LONGNET_IMPL_AUTO)
        assert float(np.abs(oh.float().numpy() - o2).max()) <= gh.TOL_OUT[dtype]
        assert float(np.abs(lh.numpy() - l2).max()) <= gh.TOL_LSE


def test_host_entry_with_qk_norm():
    """The flag passes through to the pieces' forwards (the fused kernel's
    qk_norm variant here)."""
    dev = torch.device("cuda:0")
    B, N, H, D, dtype, pats = 2, 2048, 4, 64, torch.bfloat16, ((256, 1), (512, 2), (2048, 4))
    q, k, _ = wl.random_inputs(B, N, H, D, dtype, seed=41, scale=3.0)
    _, _, v = wl.random_inputs(B, N, H, D, dtype, seed=42)
    qh, kh, vh = (_host(x, True) for x in (q, k, v))
    out_h = torch.full((B, N, H, D), float("nan"), dtype=dtype, pin_memory=True)
    lse_h = torch.full((B, H, N), float("nan"), dtype=torch.float32, pin_memory=True)
    qd, kd, vd, od = (torch.full((B, N, H, D), float("nan"), dtype=dtype, device=dev) for _ in range(4))
    ld = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    bd.longnet_dilated_attn_fwd_host(qh, kh, vh, out_h, lse_h, qd, kd, vd, od, ld, pats, True, stream=stream,
                                     qk_norm=True)
    stream.synchronize()
    assert bd.longnet_last_device_status(stream) == 0
    gh.compare_full(out_h.float().numpy(), lse_h.numpy(), q, k, v, pats, True, dtype, label="host entry qk_norm",
                    qk_norm=True)
