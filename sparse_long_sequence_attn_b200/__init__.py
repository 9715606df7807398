"""B200 (sm_100a) multi-pattern dilated-attention forward of LongNet, and its
backward.

The product is the C-ABI library liblongnet.so (include/longnet.h); this
package holds its CUDA sources (csrc/), the build script, a thin ctypes
binding, the named synthetic workloads and the sequence-parallel
forward (seqpar).
"""
from .binding import (  # noqa: F401
    LONGNET_IMPL_AUTO,
    LONGNET_IMPL_PATTERNS,
    LONGNET_IMPL_SIMT,
    LONGNET_IMPL_SMALLSEG,
    LONGNET_IMPL_TCGEN05,
    LONGNET_IMPL_TILES,
    DilatedAttnFunction,
    LongNetError,
    dilated_attention,
    dilated_attn,
    dilated_attn_bwd,
    load_library,
    longnet_dilated_attn_bwd,
    longnet_dilated_attn_bwd_ws,
    longnet_dilated_attn_fwd,
    longnet_dilated_attn_fwd_noalloc,
    longnet_dilated_attn_fwd_host,
    longnet_dilated_attn_fwd_part,
    longnet_dilated_attn_fwd_ws,
    longnet_fwd_workspace_bytes,
    longnet_gather_rows,
    longnet_last_device_status,
    longnet_scatter_rows,
    longnet_select_impl,
    longnet_watchdog_selftest,
    status_string,
    version,
)
