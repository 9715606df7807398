"""The sequence-parallel forward on one GPU: the G ranks of a split sequence
emulated in turn (each holding only its shard, poison elsewhere), the exchange's
all-gather replaced by handing every rank the list of packed buffers, the
packing and unpacking done by the library's row kernels and each rank's rows
computed by longnet_dilated_attn_fwd_part.  The assembled output is compared
with the fp64 oracle and with the single-device forward; writes outside a
rank's part are caught by sentinel values."""
import zlib

import numpy as np
import pytest
import torch

from sparse_long_sequence_attn_b200 import binding as bd
from sparse_long_sequence_attn_b200 import seqpar
from sparse_long_sequence_attn_b200 import workloads as wl
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

IMPLS = {"auto": bd.LONGNET_IMPL_AUTO, "simt": bd.LONGNET_IMPL_SIMT, "tcgen05": bd.LONGNET_IMPL_TCGEN05,
         "smallseg": bd.LONGNET_IMPL_SMALLSEG, "patterns": bd.LONGNET_IMPL_PATTERNS}
OUT_SENTINEL, LSE_SENTINEL = 3.0, -7.0
POISON = 1.0e4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    bd.load_library()
    yield


CASES = [
    # name, B, N, H, D, dtype, causal, patterns, G
    ("lm_like_g2", 2, 4096, 4, 64, torch.bfloat16, True, ((512, 1), (1024, 2), (4096, 4)), 2),
    ("three_long_g4", 1, 8192, 8, 64, torch.bfloat16, True, ((2048, 1), (4096, 2), (8192, 4)), 4),
    ("noncausal_g2", 1, 4096, 4, 64, torch.bfloat16, False, ((1024, 1), (4096, 4)), 2),
    ("segments_straddle_g2", 1, 3072, 4, 64, torch.bfloat16, True, ((1024, 1), (2048, 2)), 2),
    ("partial_last_g4", 1, 2048, 3, 64, torch.bfloat16, True, ((384, 1), (768, 3)), 4),
    ("fp32_g2", 1, 512, 2, 32, torch.float32, True, ((128, 1), (512, 2)), 2),
    ("small_segments_g2", 2, 2048, 4, 64, torch.bfloat16, True, ((64, 1), (64, 2)), 2),
    ("f16_g4", 1, 4096, 4, 64, torch.float16, True, ((1024, 1), (4096, 8)), 4),
    ("bf16_d128_g2", 1, 4096, 2, 128, torch.bfloat16, True, ((1024, 1), (4096, 4)), 2),
]


def emulate_ranks(q, k, v, patterns, causal, G, impl):
    """Run the sequence-parallel forward of G emulated ranks on cuda:0;
    returns the assembled (out, lse) on the CPU."""
    dev = torch.device("cuda:0")
    B, N, H, D = q.shape
    lists = seqpar.exchange_lists(B, N, H, patterns, G)
    held = []
    for g in range(G):
        s0, s1 = seqpar.shard_bounds(N, G, g)
        t = list(seqpar.hold_shard(*(x[:, s0:s1].to(dev) for x in (q, k, v)), N, G, g))
        # poison what the rank does not hold: NaN queries (rows are
        # independent), huge finite keys and values (a masked read weighs them
        # by 0; a needed row that never arrived swamps the output)
        for i, val in ((0, float("nan")), (1, POISON), (2, POISON)):
            t[i][:, :s0] = val
            t[i][:, s1:] = val
        held.append(t)
    packed_k = [seqpar.pack_rows(held[g][1], lists, g) for g in range(G)]
    packed_v = [seqpar.pack_rows(held[g][2], lists, g) for g in range(G)]
    assert bd.longnet_last_device_status() == 0
    out = np.empty((B, N, H, D), dtype=np.float32)
    lse = np.empty((B, H, N), dtype=np.float32)
    for g in range(G):
        s0, s1 = seqpar.shard_bounds(N, G, g)
        qf, kf, vf = held[g]
        seqpar.unpack_rows(kf, packed_k, lists, g)
        seqpar.unpack_rows(vf, packed_v, lists, g)
        o = torch.full((B, N, H, D), OUT_SENTINEL, dtype=q.dtype, device=dev)
        l = torch.full((B, H, N), LSE_SENTINEL, dtype=torch.float32, device=dev)
        bd.longnet_dilated_attn_fwd_part(qf, kf, vf, o, l, patterns, causal, (s0, s1), None, impl)
        st = bd.longnet_last_device_status()
        assert st == 0, f"device status word: {bd.status_string(st)}"
        oc, lc = o.float().cpu().numpy(), l.cpu().numpy()
        outside = np.ones(N, dtype=bool)
        outside[s0:s1] = False
        assert (oc[:, outside] == OUT_SENTINEL).all(), f"rank {g} wrote output rows outside its part"
        assert (lc[:, :, outside] == LSE_SENTINEL).all(), f"rank {g} wrote lse outside its part"
        out[:, s0:s1] = oc[:, s0:s1]
        lse[:, :, s0:s1] = lc[:, :, s0:s1]
    return out, lse


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("impl_name", ["auto", "simt", "tcgen05", "patterns"])
def test_emulated_ranks_vs_oracle_and_single_device(case, impl_name):
    name, B, N, H, D, dtype, causal, pats, G = case
    impl = IMPLS[impl_name]
    q, k, v = wl.random_inputs(B, N, H, D, dtype, seed=zlib.crc32(name.encode()) % 100000)
    try:
        o1, l1 = gh.run_cuda(q, k, v, pats, causal, impl)
    except bd.LongNetError as e:
        if e.code == bd.LONGNET_ERR_UNSUPPORTED:
            pytest.skip(f"{impl_name} does not take {name}")
        raise
    o, l = emulate_ranks(q, k, v, pats, causal, G, impl)
    assert not np.isnan(o).any() and not np.isnan(l).any(), "a shard row mixed with another row"
    err = gh.compare_full(o, l, q, k, v, pats, causal, dtype, label=f"{name}/{impl_name}")
    d = float(np.abs(o - o1).max())
    print(f"{name}/{impl_name}: max|out - oracle| = {err:.3e}, max|out - single device| = {d:.3e}")
    assert d <= gh.TOL_OUT[dtype]


@pytest.mark.parametrize("impl_name", ["auto", "simt", "tcgen05", "patterns"])
def test_head_ranges_assemble_the_full_forward(impl_name):
    """Heads split into three ranges, each computed by its own call: the
    assembled output equals the single-call forward, and nothing outside a
    call's heads is written."""
    B, N, H, D = 1, 4096, 6, 64
    pats = ((1024, 1), (2048, 2), (4096, 4))
    q, k, v = wl.random_inputs(B, N, H, D, torch.bfloat16, seed=77)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    o1, l1 = gh.run_cuda(q, k, v, pats, True, IMPLS[impl_name])
    out = np.empty_like(o1)
    lse = np.empty_like(l1)
    for h0, h1 in ((0, 1), (1, 4), (4, 6)):
        o = torch.full((B, N, H, D), OUT_SENTINEL, dtype=q.dtype, device=dev)
        l = torch.full((B, H, N), LSE_SENTINEL, dtype=torch.float32, device=dev)
        bd.longnet_dilated_attn_fwd_part(qd, kd, vd, o, l, pats, True, (0, N), (h0, h1), IMPLS[impl_name])
        assert bd.longnet_last_device_status() == 0
        oc, lc = o.float().cpu().numpy(), l.cpu().numpy()
        others = [h for h in range(H) if not h0 <= h < h1]
        assert (oc[:, :, others] == OUT_SENTINEL).all() and (lc[:, others] == LSE_SENTINEL).all()
        out[:, :, h0:h1] = oc[:, :, h0:h1]
        lse[:, h0:h1] = lc[:, h0:h1]
    assert float(np.abs(out - o1).max()) <= gh.TOL_OUT[torch.bfloat16]
    gh.compare_full(out, lse, q, k, v, pats, True, torch.bfloat16, label=f"heads/{impl_name}")


def test_part_of_long32k_workload_sampled():
    """A quarter of the 32K-token workload (positions [16384, 24576), heads
    [3, 9)) in the configuration the benchmark times, sampled rows against
    the oracle."""
    w = wl.WORKLOADS["long32k"]
    q, k, v = wl.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    s0, s1, h0, h1 = 16384, 24576, 3, 9
    o = torch.full(qd.shape, OUT_SENTINEL, dtype=q.dtype, device=dev)
    l = torch.full((w.B, w.H, w.N), LSE_SENTINEL, dtype=torch.float32, device=dev)
    bd.longnet_dilated_attn_fwd_part(qd, kd, vd, o, l, w.patterns, w.causal, (s0, s1), (h0, h1))
    assert bd.longnet_last_device_status() == 0
    oc, lc = o.float().cpu().numpy(), l.cpu().numpy()
    mask = np.zeros((w.N, w.H), dtype=bool)
    mask[s0:s1, h0:h1] = True
    assert (oc[:, ~mask] == OUT_SENTINEL).all() and (lc.transpose(0, 2, 1)[:, ~mask] == LSE_SENTINEL).all()
    rows = gh.sample_rows(w.B, w.N, w.H, w.patterns, n_random=3000, seed=11, boundary=4096)
    rows = rows[(rows[:, 1] >= s0) & (rows[:, 1] < s1) & (rows[:, 2] >= h0) & (rows[:, 2] < h1)]
    assert len(rows) > 300
    err = gh.compare_rows(oc, lc, q, k, v, w.patterns, w.causal, torch.bfloat16, rows, label="long32k_part")
    print(f"long32k part: max|out - oracle| = {err:.3e} over {len(rows)} rows")


def test_row_moves_round_trip_and_bounds():
    """gather then scatter restores the rows; an index out of range is skipped
    and reported in the status word."""
    dev = torch.device("cuda:0")
    src = torch.randn(1000, 64, device=dev).to(torch.bfloat16)
    idx = torch.randperm(1000, device=dev)[:300].contiguous()
    packed = torch.empty(300, 64, dtype=src.dtype, device=dev)
    bd.longnet_gather_rows(src, idx, packed, 64)
    assert torch.equal(packed, src[idx])
    dst = torch.zeros_like(src)
    bd.longnet_scatter_rows(packed, idx, dst, 64)
    assert bd.longnet_last_device_status() == 0
    assert torch.equal(dst[idx], src[idx])
    rest = torch.ones(1000, dtype=torch.bool, device=dev)
    rest[idx] = False
    assert (dst[rest] == 0).all()
    bad = idx.clone()
    bad[7] = 1000  # one past the last row: checked in the kernel, never read
    packed.zero_()
    bd.longnet_gather_rows(src, bad, packed, 64)
    assert bd.longnet_last_device_status() == bd.LONGNET_ERR_DEVICE_BOUNDS
    assert (packed[7] == 0).all() and torch.equal(packed[8:], src[idx[8:]])
    assert bd.longnet_last_device_status() == 0  # the word was cleared by the read


def test_sequence_parallel_forward_single_rank_group():
    """The public entry on a one-rank group (no exchange) gives the
    single-device forward."""
    import datetime
    import socket

    import torch.distributed as dist

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        pats = ((1024, 1), (2048, 2), (4096, 4))
        q, k, v = wl.random_inputs(1, 4096, 4, 64, torch.bfloat16, seed=3)
        dev = torch.device("cuda:0")
        o, l = seqpar.sequence_parallel_forward(q.to(dev), k.to(dev), v.to(dev), 4096, pats, True)
        o1, l1 = gh.run_cuda(q, k, v, pats, True, bd.LONGNET_IMPL_AUTO)
        assert np.array_equal(o.float().cpu().numpy(), o1) and np.array_equal(l.cpu().numpy(), l1)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("impl_name,D", [("auto", 128), ("patterns", 64), ("tcgen05", 64), ("auto", 32)])
def test_qk_norm_parts_assemble_the_full_forward(impl_name, D):
    """qk_norm through the part entry: ranges of positions, then ranges of
    heads, each computed by its own call (as the sequence-parallel and head
    splits make them).  Each assembled output equals the single call and the
    oracle on normalised rows; nothing outside a call's part is written."""
    B, N, H = 1, 3000, max(1, 256 // D)
    pats = ((512, 1), (1024, 2), (3000, 4))
    q, k, _ = wl.random_inputs(B, N, H, D, torch.bfloat16, seed=91 + D, scale=3.0)
    _, _, v = wl.random_inputs(B, N, H, D, torch.bfloat16, seed=92 + D)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    impl = IMPLS[impl_name]
    o1, l1 = gh.run_cuda(q, k, v, pats, True, impl, qk_norm=True)
    splits = {"positions": [((a, e), None) for a, e in ((0, 1000), (1000, 2200), (2200, N))],
              "heads": [((0, N), (h0, h1)) for h0, h1 in ((0, 1), (1, H))] if H > 1 else [((0, N), (0, 1))]}
    for kind, parts in splits.items():
        out = np.full_like(o1, np.nan)
        lse = np.full_like(l1, np.nan)
        for (a, e), hr in parts:
            h0, h1 = hr if hr is not None else (0, H)
            o = torch.full((B, N, H, D), OUT_SENTINEL, dtype=q.dtype, device=dev)
            l = torch.full((B, H, N), LSE_SENTINEL, dtype=torch.float32, device=dev)
            bd.longnet_dilated_attn_fwd_part(qd, kd, vd, o, l, pats, True, (a, e), hr, impl, qk_norm=True)
            assert bd.longnet_last_device_status() == 0
            oc, lc = o.float().cpu().numpy(), l.cpu().numpy()
            inside = np.zeros((N, H), dtype=bool)
            inside[a:e, h0:h1] = True
            assert (oc[:, ~inside] == OUT_SENTINEL).all(), f"{kind}: a write outside the part"
            assert (lc.transpose(0, 2, 1)[:, ~inside] == LSE_SENTINEL).all(), f"{kind}: an lse write outside"
            out[:, a:e, h0:h1] = oc[:, a:e, h0:h1]
            lse[:, h0:h1, a:e] = lc[:, h0:h1, a:e]
        assert not np.isnan(out).any() and not np.isnan(lse).any()
        assert float(np.abs(out - o1).max()) <= gh.TOL_OUT[torch.bfloat16], kind
        gh.compare_full(out, lse, q, k, v, pats, True, torch.bfloat16, label=f"qk_norm {kind}/{impl_name}/D{D}",
                        qk_norm=True)
