"""Sequence-parallel forward: the sequence split over the devices of a group.

The pages scale LongNet to long sequences by splitting the sequence across
devices ("LONGNET: Scaling Transformer to 1 billion tokens", section "Token
expansion reaches 1 billion+"; the two-device figure of
"1000000000！微软改进Transformer一次能记住这么多token了", section "如何做到？"):
each device holds a contiguous shard of the tokens and attends for its own
rows; a pattern whose segments fit inside a shard needs nothing from the
other devices, and for a pattern whose segments span several shards the
keys and values of the rows that pattern keeps are exchanged, which the
dilation makes a small fraction of the shard (w / r rows per segment and
head).  The exchange is one all-gather per tensor; the combination of the
patterns is row-local, so the outputs need no reduction.

This module is host logic only (which rows move, in what order) plus the
calls that move them: the rows are packed and unpacked by the library's own
gather/scatter kernels (longnet_gather_rows / longnet_scatter_rows), moved by
torch.distributed's all_gather (NCCL over NVLink on GPUs), and the attention
of the shard runs in longnet_dilated_attn_fwd_part.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import binding as bd

Pattern = Tuple[int, int]


def shard_bounds(N: int, G: int, g: int) -> Tuple[int, int]:
    """Positions [s0, s1) of shard g of G equal shards (G must divide N)."""
    if N % G != 0:
        raise ValueError(f"the sequence length {N} is not a multiple of {G} shards")
    S = N // G
    return g * S, (g + 1) * S


def is_local(w: int, N: int, G: int) -> bool:
    """True when no segment of length w straddles two shards (each shard then
    holds whole segments and attends for them alone)."""
    S = N // G
    return w <= S and S % w == 0


def long_patterns(patterns: Sequence[Pattern], N: int, G: int) -> List[Pattern]:
    """The patterns whose segments span several shards."""
    return [tuple(p) for p in patterns if not is_local(int(p[0]), N, G)]


def _kept_mask(x: np.ndarray, H: int, patterns: Sequence[Pattern]) -> np.ndarray:
    """[len(x), H] booleans: position x is kept for head h by some pattern
    (segments of w, head offset o = h mod r, kept rows o + r k)."""
    h = np.arange(H, dtype=np.int64)[None, :]
    keep = np.zeros((x.shape[0], H), dtype=bool)
    for (w, r) in patterns:
        rel = (x[:, None] % w) - (h % r)
        keep |= (rel >= 0) & (rel % r == 0)
    return keep


def exchanged_rows(B: int, N: int, H: int, patterns: Sequence[Pattern], G: int, g: int) -> np.ndarray:
    """Rows of shard g that the other shards may need: every (b, x, h) with x
    in the shard kept by a pattern whose segments span several shards, as
    flat row indices (b N + x) H + h of a [B, N, H, D] tensor, ascending.
    Every device computes the same lists for every shard."""
    longp = long_patterns(patterns, N, G)
    if not longp:
        return np.zeros(0, dtype=np.int64)
    s0, s1 = shard_bounds(N, G, g)
    x = np.arange(s0, s1, dtype=np.int64)
    keep = _kept_mask(x, H, longp)
    xi, hi = np.nonzero(keep)
    local = (x[xi] * H + hi).astype(np.int64)
    return np.concatenate([b * N * H + local for b in range(B)]).astype(np.int64)


def needed_rows(B: int, N: int, H: int, patterns: Sequence[Pattern], G: int, g: int,
                causal: bool) -> np.ndarray:
    """Rows outside shard g that its attention reads: for each pattern whose
    segments span several shards and each segment holding a kept row of the
    shard, the segment's kept rows outside the shard, only those before the
    shard's last kept row when causal (a kept row attends to kept rows at or
    before itself).  Flat row
    indices as in exchanged_rows, ascending (used to check an exchange)."""
    s0, s1 = shard_bounds(N, G, g)
    rows = []
    for (w, r) in long_patterns(patterns, N, G):
        for h in range(H):
            o = h % r
            for seg in range(s0 // w, (s1 - 1) // w + 1):
                base = seg * w + o
                end = min(seg * w + w, N)
                if base >= end:
                    continue
                kept = np.arange(base, end, r, dtype=np.int64)
                in_shard = kept[(kept >= s0) & (kept < s1)]
                if in_shard.size == 0:
                    continue
                if causal:
                    kept = kept[kept <= in_shard.max()]
                kept = kept[(kept < s0) | (kept >= s1)]
                rows.append(kept * H + h)
    if not rows:
        return np.zeros(0, dtype=np.int64)
    one = np.unique(np.concatenate(rows))
    return np.concatenate([b * N * H + one for b in range(B)]).astype(np.int64)


def _library_gather(src: torch.Tensor, idx: torch.Tensor, dst: torch.Tensor) -> None:
    bd.longnet_gather_rows(src, idx, dst, src.shape[-1])


def _library_scatter(src: torch.Tensor, idx: torch.Tensor, dst: torch.Tensor) -> None:
    bd.longnet_scatter_rows(src, idx, dst, dst.shape[-1])


def exchange_lists(B: int, N: int, H: int, patterns: Sequence[Pattern], G: int) -> List[np.ndarray]:
    """exchanged_rows of every shard (the same on every device)."""
    return [exchanged_rows(B, N, H, patterns, G, gg) for gg in range(G)]


def pack_rows(t: torch.Tensor, lists: List[np.ndarray], g: int, gather=_library_gather) -> torch.Tensor:
    """This shard's exchanged rows of t [B, N, H, D], packed into a buffer of
    max(len(list)) rows (the tail past its own list is zero), the operand of
    the all-gather."""
    n_max = max(len(x) for x in lists)
    packed = torch.zeros((n_max, t.shape[-1]), dtype=t.dtype, device=t.device)
    if len(lists[g]):
        gather(t, torch.from_numpy(lists[g]).to(t.device), packed[:len(lists[g])])
    return packed


def unpack_rows(t: torch.Tensor, parts: List[torch.Tensor], lists: List[np.ndarray], g: int,
                scatter=_library_scatter) -> None:
    """Write every other shard's packed rows (parts[gg], the all-gather's
    result) into place in t."""
    for gg, part in enumerate(parts):
        if gg != g and len(lists[gg]):
            scatter(part[:len(lists[gg])], torch.from_numpy(lists[gg]).to(t.device), t)


def exchange_kv(k_full: torch.Tensor, v_full: torch.Tensor, patterns: Sequence[Pattern], group=None,
                gather=_library_gather, scatter=_library_scatter) -> int:
    """Fill the rows of k_full and v_full (full-length [B, N, H, D] on this
    device, the own shard already in place) that the other shards hold and a
    pattern spanning several shards keeps: pack the own shard's exchanged
    rows, all-gather the packed buffers, unpack every other shard's rows into
    place.  gather(src, idx, packed) and scatter(packed, idx, dst) move rows
    of the last dimension by flat row index; by default they are the
    library's kernels, and the CPU tests of the partition pass plain
    indexing.  Returns the bytes this device sends per tensor."""
    G, g = dist.get_world_size(group), dist.get_rank(group)
    B, N, H, D = k_full.shape
    if G == 1 or not long_patterns(patterns, N, G):
        return 0
    lists = exchange_lists(B, N, H, patterns, G)
    for t in (k_full, v_full):
        packed = pack_rows(t, lists, g, gather)
        parts = [torch.empty_like(packed) for _ in range(G)]
        dist.all_gather(parts, packed, group=group)
        unpack_rows(t, parts, lists, g, scatter)
    return packed.numel() * packed.element_size()


def hold_shard(q_shard: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, N: int, G: int,
               g: int):
    """Full-length [B, N, H, D] buffers holding shard g of G in place.  k and
    v are zero outside the shard until the exchange fills the rows it moves:
    the forward may read kept rows past a segment's end and mask them, and
    a masked row's weight, 0, multiplies its v row, so every row must be
    finite.  q outside the shard is never combined with the shard's rows
    and is left unset."""
    B, S, H, D = q_shard.shape
    if S * G != N:
        raise ValueError("each shard must hold N / G positions")
    s0, s1 = shard_bounds(N, G, g)
    q_full = torch.empty((B, N, H, D), dtype=q_shard.dtype, device=q_shard.device)
    k_full = torch.zeros_like(q_full)
    v_full = torch.zeros_like(q_full)
    q_full[:, s0:s1] = q_shard
    k_full[:, s0:s1] = k_shard
    v_full[:, s0:s1] = v_shard
    return q_full, k_full, v_full


def sequence_parallel_forward(q_shard: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor,
                              N: int, patterns: Sequence[Pattern], causal: bool = True, group=None,
                              impl: int = bd.LONGNET_IMPL_AUTO, qk_norm: bool = False):
    """The forward of this device's shard of a sequence split over the group.

    q_shard, k_shard, v_shard: this device's tokens [B, N / G, H, D] (shard g
    of G is positions [g N / G, (g + 1) N / G)).  Returns (out_shard
    [B, N / G, H, D], lse_shard [B, H, N / G]): the rows the single-device
    forward gives for those positions, by the same kernels."""
    G, g = dist.get_world_size(group), dist.get_rank(group)
    B, H = q_shard.shape[0], q_shard.shape[2]
    q_full, k_full, v_full = hold_shard(q_shard, k_shard, v_shard, N, G, g)
    exchange_kv(k_full, v_full, patterns, group)
    s0, s1 = shard_bounds(N, G, g)
    out_full = torch.empty_like(q_full)
    lse_full = torch.empty((B, H, N), dtype=torch.float32, device=q_full.device)
    bd.longnet_dilated_attn_fwd_part(q_full, k_full, v_full, out_full, lse_full, patterns, causal,
                                     (s0, s1), None, impl, qk_norm=qk_norm)
    return out_full[:, s0:s1].contiguous(), lse_full[:, :, s0:s1].contiguous()
