"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/longnet.h declares, rejects bad arguments before touching a
device, and reports the missing device instead of crashing (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_long_sequence_attn_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "longnet.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(longnet_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = bd.load_library()
    names = declared_functions()
    assert len(names) >= 7
    for name in names:
        assert hasattr(lib, name), f"{name} declared in longnet.h but not exported"
        assert name in bd.SIGNATURES, f"{name} missing from the Python binding"


def test_status_strings_and_version():
    assert bd.status_string(0) == "ok"
    assert "invalid" in bd.status_string(bd.LONGNET_ERR_INVALID_ARG)
    assert bd.status_string(12345) == "unknown status"
    assert bd.version().startswith("longnet-b200")


def _call(lib, B=1, N=64, H=2, D=16, pats=((16, 1),), causal=1, dtype=0, ptr=None, lse=None, impl=0):
    buf = ptr if ptr is not None else ctypes.c_void_p(0x1000)  # never dereferenced on the host
    n = len(pats)
    w = (ctypes.c_int64 * max(n, 1))(*[p[0] for p in pats])
    r = (ctypes.c_int64 * max(n, 1))(*[p[1] for p in pats])
    return lib.longnet_dilated_attn_fwd_impl(buf, buf, buf, buf, lse, B, N, H, D, n, w, r, causal,
                                             dtype, impl, None)


@pytest.mark.parametrize("kw", [
    dict(B=0), dict(N=-1), dict(H=0), dict(D=0), dict(pats=()), dict(pats=((16, 0),)),
    dict(pats=((0, 1),)), dict(causal=2),
    dict(dtype=7), dict(pats=tuple((16, 1) for _ in range(17))), dict(impl=9),
])
def test_invalid_arguments_rejected_on_host(kw):
    lib = bd.load_library()
    rc = _call(lib, **kw)
    assert rc == bd.LONGNET_ERR_INVALID_ARG, rc


def test_unknown_flag_bits_rejected_on_host():
    lib = bd.load_library()
    buf = ctypes.c_void_p(0x1000)
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)
    for flags in (2, 4, -1):
        rc = lib.longnet_dilated_attn_fwd_ex(buf, buf, buf, buf, None, 1, 64, 2, 16, 1, w, r, 1, 0,
                                             flags, 0, None)
        assert rc == bd.LONGNET_ERR_INVALID_ARG, (flags, rc)


def test_null_and_misaligned_pointers():
    lib = bd.load_library()
    assert _call(lib, ptr=ctypes.c_void_p(0)) == bd.LONGNET_ERR_INVALID_ARG
    assert _call(lib, ptr=ctypes.c_void_p(0x1008)) == bd.LONGNET_ERR_MISALIGNED
    assert _call(lib, lse=ctypes.c_void_p(0x1002)) == bd.LONGNET_ERR_MISALIGNED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_no_device():
    lib = bd.load_library()
    assert _call(lib) == bd.LONGNET_ERR_NO_DEVICE
    # w not dividing N (a shorter last segment) and w > N are valid shapes
    assert _call(lib, pats=((24, 1),)) == bd.LONGNET_ERR_NO_DEVICE
    assert _call(lib, pats=((128, 1), (16, 2))) == bd.LONGNET_ERR_NO_DEVICE
    assert lib.longnet_last_device_status(None) == bd.LONGNET_ERR_NO_DEVICE
    assert lib.longnet_watchdog_selftest(1000, None) == bd.LONGNET_ERR_NO_DEVICE


def test_select_impl_host_logic():
    f32, bf16 = torch.float32, torch.bfloat16
    assert bd.longnet_select_impl(1, 256, 2, 16, ((64, 1), (128, 2)), True, f32) == bd.LONGNET_IMPL_SIMT
    assert bd.longnet_select_impl(1, 256, 2, 48, ((64, 1),), True, f32) == bd.LONGNET_ERR_UNSUPPORTED
    # a shorter last segment (255 = 3 * 64 + 63) goes to the general kernel
    assert bd.longnet_select_impl(1, 255, 2, 16, ((64, 1),), True, f32) == bd.LONGNET_IMPL_SIMT
    # bf16 D = 64 with shorter last segments (4000 = 3 * 1024 + 928) goes to tcgen05
    assert bd.longnet_select_impl(1, 4000, 4, 64, ((1024, 1), (2048, 2)), True, bf16) == bd.LONGNET_IMPL_TCGEN05
    # D = 128 (16-bit) goes to the per-pattern tcgen05 family, fp32 to the general kernel
    assert bd.longnet_select_impl(1, 4096, 4, 128, ((1024, 1), (2048, 2)), True, bf16) == bd.LONGNET_IMPL_PATTERNS
    assert bd.longnet_select_impl(1, 4096, 4, 128, ((1024, 1), (2048, 2)), True, f32) == bd.LONGNET_IMPL_SIMT
    # one short segment length with a shorter last segment: the small-segment family
    assert bd.longnet_select_impl(2, 1000, 4, 64, ((64, 1), (64, 2)), False, bf16) == bd.LONGNET_IMPL_SMALLSEG
    # so do D = 32 and 16 (16-bit)
    for D in (16, 32):
        assert bd.longnet_select_impl(1, 4096, 4, D, ((1024, 1), (2048, 2)), True, bf16) == bd.LONGNET_IMPL_PATTERNS
    # more than 6 patterns at D = 64: per-pattern family
    seven = tuple((256 * (i + 1), i + 1) for i in range(7))
    assert bd.longnet_select_impl(1, 4096, 4, 64, seven, True, bf16) == bd.LONGNET_IMPL_PATTERNS
    assert bd.longnet_select_impl(1, 256, 2, 16, ((64, 0),), True, f32) == bd.LONGNET_ERR_INVALID_ARG
    # the fused family takes 16-bit D = 64 shapes with up to six patterns
    impl = bd.longnet_select_impl(1, 32768, 12, 64, ((2048, 1), (4096, 2)), True, bf16)
    assert impl == bd.LONGNET_IMPL_TCGEN05


def _call_bwd(lib, B=1, N=64, H=2, D=16, pats=((16, 1),), causal=1, dtype=0, flags=0,
              ptrs=None, impl=0):
    buf = ctypes.c_void_p(0x1000)  # never dereferenced on the host
    p = dict(q=buf, k=buf, v=buf, out=buf, lse=buf, dout=buf, dq=buf, dk=buf, dv=buf)
    p.update(ptrs or {})
    n = len(pats)
    w = (ctypes.c_int64 * max(n, 1))(*[x[0] for x in pats])
    r = (ctypes.c_int64 * max(n, 1))(*[x[1] for x in pats])
    return lib.longnet_dilated_attn_bwd(p["q"], p["k"], p["v"], p["out"], p["lse"], p["dout"],
                                        p["dq"], p["dk"], p["dv"], B, N, H, D, n, w, r, causal,
                                        dtype, flags, impl, None)


def test_backward_argument_checks_on_host():
    lib = bd.load_library()
    null = ctypes.c_void_p(0)
    for name in ("q", "out", "lse", "dout", "dq", "dk", "dv"):
        assert _call_bwd(lib, ptrs={name: null}) == bd.LONGNET_ERR_INVALID_ARG, name
    for name in ("out", "dout", "dk", "dv", "q"):
        assert _call_bwd(lib, ptrs={name: ctypes.c_void_p(0x1008)}) == bd.LONGNET_ERR_MISALIGNED, name
    assert _call_bwd(lib, ptrs={"lse": ctypes.c_void_p(0x1002)}) == bd.LONGNET_ERR_MISALIGNED
    assert _call_bwd(lib, flags=2) == bd.LONGNET_ERR_INVALID_ARG
    assert _call_bwd(lib, D=48) == bd.LONGNET_ERR_UNSUPPORTED
    assert _call_bwd(lib, pats=((16, 0),)) == bd.LONGNET_ERR_INVALID_ARG
    assert _call_bwd(lib, causal=3) == bd.LONGNET_ERR_INVALID_ARG
    for impl in (3, 5, -1):
        assert _call_bwd(lib, impl=impl) == bd.LONGNET_ERR_INVALID_ARG, impl
    # the tensor-core families: bf16/fp16 only; the tile family at D = 64, the
    # tcgen05 one at D = 16, 32, 64 or 128, without qk_norm, with at most 6
    # patterns
    for impl in (bd.LONGNET_IMPL_TILES, bd.LONGNET_IMPL_TCGEN05):
        assert _call_bwd(lib, impl=impl) == bd.LONGNET_ERR_UNSUPPORTED
        assert _call_bwd(lib, impl=impl, dtype=1, D=48) == bd.LONGNET_ERR_UNSUPPORTED
    assert _call_bwd(lib, impl=bd.LONGNET_IMPL_TILES, dtype=1, D=32) == bd.LONGNET_ERR_UNSUPPORTED
    assert _call_bwd(lib, impl=bd.LONGNET_IMPL_TCGEN05, dtype=1, D=64,
                     flags=bd.LONGNET_FLAG_QK_NORM) == bd.LONGNET_ERR_UNSUPPORTED
    assert _call_bwd(lib, impl=bd.LONGNET_IMPL_TCGEN05, dtype=1, D=64,
                     pats=tuple((16, 1) for _ in range(7))) == bd.LONGNET_ERR_UNSUPPORTED
    # the forward has no tile family
    buf = ctypes.c_void_p(0x1000)
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)
    assert lib.longnet_dilated_attn_fwd_ex(buf, buf, buf, buf, None, 1, 64, 2, 16, 1, w, r, 1, 0, 0,
                                           bd.LONGNET_IMPL_TILES, None) == bd.LONGNET_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_backward_valid_call_without_device_reports_no_device():
    lib = bd.load_library()
    for dtype in (0, 1, 2):
        assert _call_bwd(lib, dtype=dtype, pats=((24, 1), (64, 4))) == bd.LONGNET_ERR_NO_DEVICE
    assert _call_bwd(lib, dtype=1, D=64, impl=bd.LONGNET_IMPL_TILES) == bd.LONGNET_ERR_NO_DEVICE
    assert _call_bwd(lib, dtype=1, D=64, impl=bd.LONGNET_IMPL_TCGEN05) == bd.LONGNET_ERR_NO_DEVICE
    assert _call_bwd(lib, dtype=1, D=32, impl=bd.LONGNET_IMPL_TCGEN05) == bd.LONGNET_ERR_NO_DEVICE
    # qk_norm is taken by both families
    assert _call_bwd(lib, flags=bd.LONGNET_FLAG_QK_NORM) == bd.LONGNET_ERR_NO_DEVICE
    assert _call_bwd(lib, dtype=2, D=64, flags=bd.LONGNET_FLAG_QK_NORM,
                     impl=bd.LONGNET_IMPL_TILES) == bd.LONGNET_ERR_NO_DEVICE


def test_backward_tile_grid_limit_on_host():
    """A segment of more than 65535 tiles (2^22 + rows at r = 1) is beyond the
    tile kernels' grid: a forced tile call is UNSUPPORTED before any device
    access, while SIMT (and AUTO, which falls back to it) get as far as the
    device check."""
    lib = bd.load_library()
    N = 65536 * 64 + 64
    assert _call_bwd(lib, N=N, D=64, dtype=1, pats=((N, 1),),
                     impl=bd.LONGNET_IMPL_TILES) == bd.LONGNET_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        for impl in (bd.LONGNET_IMPL_AUTO, bd.LONGNET_IMPL_SIMT):
            assert _call_bwd(lib, N=N, D=64, dtype=1, pats=((N, 1),),
                             impl=impl) == bd.LONGNET_ERR_NO_DEVICE
    # one tile fewer is inside the limit
    N2 = 65535 * 64
    if not torch.cuda.is_available():
        assert _call_bwd(lib, N=N2, D=64, dtype=1, pats=((N2, 1),),
                         impl=bd.LONGNET_IMPL_TILES) == bd.LONGNET_ERR_NO_DEVICE


def _call_part(lib, q_range=(0, 64), h_range=(0, 2), N=64, H=2):
    buf = ctypes.c_void_p(0x1000)  # never dereferenced on the host
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)
    return lib.longnet_dilated_attn_fwd_part(buf, buf, buf, buf, None, 1, N, H, 16, 1, w, r, 1, 0, 0, 0,
                                             q_range[0], q_range[1], h_range[0], h_range[1], None)


@pytest.mark.parametrize("q_range,h_range", [
    ((-1, 64), (0, 2)), ((0, 65), (0, 2)), ((32, 32), (0, 2)), ((40, 8), (0, 2)),
    ((0, 64), (-1, 2)), ((0, 64), (0, 3)), ((0, 64), (1, 1)),
])
def test_part_ranges_checked_on_host(q_range, h_range):
    assert _call_part(bd.load_library(), q_range, h_range) == bd.LONGNET_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_part_valid_ranges_reach_the_device_check():
    lib = bd.load_library()
    for qr, hr in (((0, 64), (0, 2)), ((17, 33), (1, 2)), ((63, 64), (0, 1))):
        assert _call_part(lib, qr, hr) == bd.LONGNET_ERR_NO_DEVICE


def test_row_moves_checked_on_host():
    lib = bd.load_library()
    buf, idx = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000)
    g, s = lib.longnet_gather_rows, lib.longnet_scatter_rows
    assert g(buf, 10, idx, 0, buf, 128, None) == bd.LONGNET_OK  # nothing to move
    assert g(buf, 10, idx, -1, buf, 128, None) == bd.LONGNET_ERR_INVALID_ARG
    assert g(buf, 10, idx, 4, buf, 24, None) == bd.LONGNET_ERR_INVALID_ARG  # not whole 16-byte words
    assert g(buf, 10, idx, 4, buf, 0, None) == bd.LONGNET_ERR_INVALID_ARG
    assert g(buf, 10, None, 4, buf, 128, None) == bd.LONGNET_ERR_INVALID_ARG
    assert g(ctypes.c_void_p(0x1008), 10, idx, 4, buf, 128, None) == bd.LONGNET_ERR_MISALIGNED
    assert g(buf, 10, ctypes.c_void_p(0x2004), 4, buf, 128, None) == bd.LONGNET_ERR_MISALIGNED
    assert s(buf, 4, idx, ctypes.c_void_p(0x1004), 10, 128, None) == bd.LONGNET_ERR_MISALIGNED
    assert s(buf, 4, idx, buf, -1, 128, None) == bd.LONGNET_ERR_INVALID_ARG
    if not torch.cuda.is_available():
        assert g(buf, 10, idx, 4, buf, 128, None) == bd.LONGNET_ERR_NO_DEVICE
        assert s(buf, 4, idx, buf, 10, 128, None) == bd.LONGNET_ERR_NO_DEVICE


def test_workspace_bytes_on_host():
    lib = bd.load_library()
    f = lib.longnet_fwd_workspace_bytes
    assert f(1, 1000, 3, 64, 1, 0) == 0  # no options, no workspace
    one = 1000 * 3 * 64 * 2
    assert f(1, 1000, 3, 64, 1, 1) == 2 * ((one + 255) // 256 * 256)
    assert f(1, 1000, 3, 64, 0, 3) == 2 * ((2 * one + 255) // 256 * 256)
    assert f(0, 1000, 3, 64, 1, 1) == bd.LONGNET_ERR_INVALID_ARG
    assert f(1, 1000, 3, 64, 7, 1) == bd.LONGNET_ERR_INVALID_ARG
    assert f(1, 1000, 3, 64, 1, 4) == bd.LONGNET_ERR_INVALID_ARG


def _call_ws(lib, flags, ws=0x10000, ws_bytes=1 << 30, D=64, N=64, dtype=1):
    buf = ctypes.c_void_p(0x1000)  # never dereferenced on the host
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)
    return lib.longnet_dilated_attn_fwd_ws(buf, buf, buf, buf, None, 1, N, 2, D, 1, w, r, 1, dtype, flags, 0,
                                           None if ws is None else ctypes.c_void_p(ws), ws_bytes, None)


def test_workspace_entry_checked_on_host():
    lib = bd.load_library()
    assert _call_ws(lib, 4) == bd.LONGNET_ERR_INVALID_ARG           # unknown option
    assert _call_ws(lib, 1, ws=None) == bd.LONGNET_ERR_INVALID_ARG   # options need a workspace
    assert _call_ws(lib, 2, ws_bytes=100) == bd.LONGNET_ERR_INVALID_ARG
    assert _call_ws(lib, 3, ws=0x10010) == bd.LONGNET_ERR_MISALIGNED
    assert _call_ws(lib, 1, D=24) == bd.LONGNET_ERR_UNSUPPORTED       # the prologue's D
    # fp16 XPOS: |log2 s| reaches 1.807 * 4096 / 512 > 8 at N = 8192
    assert _call_ws(lib, 2, N=8192, dtype=2) == bd.LONGNET_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert _call_ws(lib, 3) == bd.LONGNET_ERR_NO_DEVICE
        assert _call_ws(lib, 0, ws=None, ws_bytes=0) == bd.LONGNET_ERR_NO_DEVICE
        assert _call_ws(lib, 2, N=4096, dtype=2) == bd.LONGNET_ERR_NO_DEVICE  # within fp16's range


def test_noalloc_entry_checked_on_host():
    lib = bd.load_library()
    buf = ctypes.c_void_p(0x1000)  # never dereferenced on the host
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)

    def call(N, H, flags):
        return lib.longnet_dilated_attn_fwd_noalloc(buf, buf, buf, buf, None, 1, N, H, 64, 1, w, r, 1, 1,
                                                    flags, 0, None)

    assert call(1024, 2, 4) == bd.LONGNET_ERR_INVALID_ARG
    # 2 x 32768 x 8 x 64 bf16 = 64 MiB of workspace > the 32 MiB scratch
    assert call(32768, 8, 1) == bd.LONGNET_ERR_SCRATCH_LIMIT
    assert "fixed scratch" in bd.status_string(bd.LONGNET_ERR_SCRATCH_LIMIT)
    if not torch.cuda.is_available():
        assert call(1024, 2, 1) == bd.LONGNET_ERR_NO_DEVICE
        assert call(32768, 8, 0) == bd.LONGNET_ERR_NO_DEVICE  # no options: no scratch needed


def test_host_buffer_entry_checked_on_host():
    """longnet_dilated_attn_fwd_host rejects bad arguments before touching a
    device, and a valid call without a device reports no device."""
    lib = bd.load_library()
    buf = ctypes.c_void_p(0x1000)  # never dereferenced on the host
    w = (ctypes.c_int64 * 1)(16)
    r = (ctypes.c_int64 * 1)(1)

    def call(q_host=buf, lse_host=None, lse_dev=None, flags=0, impl=0, pieces=0, D=64, dev=buf):
        return lib.longnet_dilated_attn_fwd_host(q_host, buf, buf, buf, lse_host, dev, buf, buf, buf, lse_dev,
                                                 1, 256, 4, D, 1, w, r, 1, 1, flags, impl, pieces, None)

    assert call(q_host=None) == bd.LONGNET_ERR_INVALID_ARG
    assert call(lse_host=buf) == bd.LONGNET_ERR_INVALID_ARG  # lse_host without lse_dev
    assert call(pieces=-1) == bd.LONGNET_ERR_INVALID_ARG
    assert call(flags=bd.LONGNET_FLAG_XPOS) == bd.LONGNET_ERR_INVALID_ARG  # XPOS needs a workspace
    assert call(impl=bd.LONGNET_IMPL_TILES) == bd.LONGNET_ERR_INVALID_ARG  # backward-only family
    assert call(D=0) == bd.LONGNET_ERR_INVALID_ARG
    assert call(dev=ctypes.c_void_p(0x1004)) == bd.LONGNET_ERR_MISALIGNED
    if not torch.cuda.is_available():
        assert call() == bd.LONGNET_ERR_NO_DEVICE
        assert call(lse_host=buf, lse_dev=buf, pieces=3) == bd.LONGNET_ERR_NO_DEVICE
