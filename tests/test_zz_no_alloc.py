"""longnet_dilated_attn_fwd_noalloc: the forward with the input-side options,
its workspace the library's fixed device scratch.  Compared with the
caller-workspace entry (longnet_dilated_attn_fwd_ws) on two calls in a row;
no device memory is allocated by the calls; a problem larger than the scratch
is refused.  Collected last, and independent of what ran before it."""
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


CALLS = [
    # B, N, H, D, dtype, causal, patterns, qk_norm, xpos
    (1, 8192, 8, 64, torch.bfloat16, True, ((2048, 1), (4096, 2), (8192, 4)), True, False),
    (2, 2048, 4, 64, torch.float16, False, ((512, 1), (2048, 4)), False, True),
]


def test_two_calls_match_the_workspace_entry_and_allocate_nothing():
    dev = torch.device("cuda:0")
    inputs, outs = [], []
    for i, (B, N, H, D, dtype, causal, pats, qk_norm, xpos) in enumerate(CALLS):
        q, k, v = (x.to(dev) for x in wl.random_inputs(B, N, H, D, dtype, seed=100 + i))
        inputs.append((q, k, v))
        outs.append((torch.full_like(q, float("nan")),
                     torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)))
        need = bd.longnet_fwd_workspace_bytes(B, N, H, D, dtype, qk_norm, xpos)
        assert 0 < need <= bd.LONGNET_NOALLOC_SCRATCH_BYTES
    # a first call on this device does the one-time scratch lookup
    B, N, H, D, dtype, causal, pats, qk_norm, xpos = CALLS[0]
    q, k, v = inputs[0]
    bd.longnet_dilated_attn_fwd_noalloc(q, k, v, *outs[0], pats, causal, qk_norm=qk_norm, xpos=xpos)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    used0 = torch.cuda.memory_allocated()
    # two calls in a row on one stream, then nothing allocated since
    for (B, N, H, D, dtype, causal, pats, qk_norm, xpos), (q, k, v), (o, l) in zip(CALLS, inputs, outs):
        bd.longnet_dilated_attn_fwd_noalloc(q, k, v, o, l, pats, causal, qk_norm=qk_norm, xpos=xpos)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_allocated() == used0
    assert bd.longnet_last_device_status() == 0
    for (B, N, H, D, dtype, causal, pats, qk_norm, xpos), (q, k, v), (o, l) in zip(CALLS, inputs, outs):
        ws = torch.empty(bd.longnet_fwd_workspace_bytes(B, N, H, D, dtype, qk_norm, xpos), dtype=torch.uint8,
                         device=dev)
        o2, l2 = torch.empty_like(o), torch.empty_like(l)
        bd.longnet_dilated_attn_fwd_ws(q, k, v, o2, l2, pats, causal, ws, qk_norm=qk_norm, xpos=xpos)
        assert bd.longnet_last_device_status() == 0
        assert not torch.isnan(o).any() and not torch.isnan(l).any()
        d_out = float((o.float() - o2.float()).abs().max())
        d_lse = float((l - l2).abs().max())
        assert d_out <= gh.TOL_OUT[dtype] and d_lse <= gh.TOL_LSE, (d_out, d_lse)
        print(f"noalloc vs workspace entry, N={N} {dtype}: max|out diff| = {d_out:.3e}, lse {d_lse:.3e}")


def test_problem_beyond_the_scratch_is_refused():
    dev = torch.device("cuda:0")
    B, N, H, D = 1, 32768, 8, 64  # 2 x 32 MiB of bf16 q and k: twice the scratch
    assert bd.longnet_fwd_workspace_bytes(B, N, H, D, torch.bfloat16, True) > bd.LONGNET_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, N, H, D, dtype=torch.bfloat16, device=dev)
    out = torch.full_like(q, 7.0)
    with pytest.raises(bd.LongNetError) as e:
        bd.longnet_dilated_attn_fwd_noalloc(q, q, q, out, None, ((1024, 1),), True, qk_norm=True)
    assert e.value.code == bd.LONGNET_ERR_SCRATCH_LIMIT
    assert "fixed scratch" in str(e.value)
    assert bool((out == 7.0).all())  # nothing was launched
    # without options no scratch is needed, whatever the size
    bd.longnet_dilated_attn_fwd_noalloc(q, q, q, out, None, ((1024, 1),), True)
    assert bd.longnet_last_device_status() == 0
    assert not bool((out == 7.0).any())
