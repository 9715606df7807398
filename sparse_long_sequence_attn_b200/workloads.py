"""Named workloads and seeded synthetic inputs.

This module is shared by the tests, the benchmark and the smoke check.  It
holds shapes, pattern sets and random-number recipes only: none of the
attention arithmetic lives here, so the CUDA path and the fp64 oracle can both
be fed from it without sharing any of the method.

Shapes and pattern sets come from the pages:
  * the experiment setting of "1000000000！微软改进Transformer一次能记住这么多token了"
    (section "实验评估"): segment lengths w = {2048, 4096, 8192, 16384, 32768}
    with dilations r = {1, 2, 4, 6, 12}, sequences up to 32K;
  * the DilatedAttention usage example of "LongNet" (docsearch page, section
    on the DilatedAttention class): batch 32, 8192 tokens, dim 512 over 8 heads,
    dilation 2, segment 64, qk_norm on.

Inputs: q, k, v are drawn in fp32 from a CPU torch.Generator seeded with
20260000 + workload index, in the order q, k, v, each torch.randn(B, N, H, D);
with qk_norm the rows of q and k are scaled to unit L2 norm over D in fp32;
then everything is cast to the workload dtype (round to nearest even).  No
dataset is used: these N(0, 1) tensors stand in for the enwik8 / Stack text the
pages train on.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import List, Tuple

import torch

Pattern = Tuple[int, int]


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    N: int
    H: int
    D: int
    dtype: str  # "fp32", "bf16" or "fp16"
    causal: bool
    patterns: Tuple[Pattern, ...]
    qk_norm: bool = False
    note: str = ""
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def seed(self) -> int:
        return 20260000 + self.index

    @property
    def torch_dtype(self):
        return {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}[self.dtype]

    def with_n(self, N: int) -> "Workload":
        """Same workload at another length, patterns truncated to w <= N."""
        pats = tuple(p for p in self.patterns if p[0] <= N)
        return replace(self, N=N, patterns=pats)

    def tokens(self) -> int:
        return self.B * self.N


def sweep_patterns(N: int) -> Tuple[Pattern, ...]:
    """(2048 * 2^i, 2^i) for i = 0..5, kept while w <= N (sparse length 2048)."""
    return tuple((2048 << i, 1 << i) for i in range(6) if (2048 << i) <= N)


WORKLOADS = {
    "tiny": Workload("tiny", 0, B=1, N=256, H=2, D=16, dtype="fp32", causal=True,
                     patterns=((64, 1), (128, 2), (256, 4)),
                     note="small fp32 case the oracle finishes instantly"),
    "lm": Workload("lm", 1, B=4, N=8192, H=12, D=64, dtype="bf16", causal=True,
                   patterns=((2048, 1), (4096, 2), (8192, 4)),
                   note="language-model layer"),
    "long32k": Workload("long32k", 2, B=1, N=32768, H=12, D=64, dtype="bf16", causal=True,
                        patterns=((2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)),
                        note="the pages' experiment pattern set at 32K tokens"),
    "smallseg": Workload("smallseg", 3, B=32, N=8192, H=8, D=64, dtype="bf16", causal=False,
                         patterns=((64, 1), (64, 2)), qk_norm=True,
                         note="DilatedAttention usage example shape; memory-bound"),
    "sweep": Workload("sweep", 4, B=1, N=65536, H=8, D=64, dtype="bf16", causal=True,
                      patterns=sweep_patterns(65536),
                      note="linear-scaling sweep; N in {65536, 262144, 1048576}"),
}
SWEEP_NS = (65536, 262144, 1048576)


def sweep_workload(N: int) -> Workload:
    return replace(WORKLOADS["sweep"], N=N, patterns=sweep_patterns(N))


def make_inputs(wl: Workload, seed: int | None = None, B: int | None = None,
                N: int | None = None, H: int | None = None):
    """Seeded q, k, v on the CPU in the workload dtype, shape [B, N, H, D]."""
    B = wl.B if B is None else B
    N = wl.N if N is None else N
    H = wl.H if H is None else H
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    q = torch.randn(B, N, H, wl.D, generator=g, dtype=torch.float32)
    k = torch.randn(B, N, H, wl.D, generator=g, dtype=torch.float32)
    v = torch.randn(B, N, H, wl.D, generator=g, dtype=torch.float32)
    if wl.qk_norm:
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
    return q.to(wl.torch_dtype), k.to(wl.torch_dtype), v.to(wl.torch_dtype)


def random_inputs(B: int, N: int, H: int, D: int, dtype, seed: int, scale: float = 1.0):
    """Seeded N(0, scale^2) q, k, v of any shape (parity cases beyond the named ones)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.randn(B, N, H, D, generator=g, dtype=torch.float32) * scale
        out.append(x.to(dtype))
    return tuple(out)


def random_cotangent(B: int, N: int, H: int, D: int, dtype, seed: int):
    """Seeded N(0, 1) dout [B, N, H, D] for the backward (drawn after a
    distinct seed offset so it never repeats q, k or v)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 1000003)
    return torch.randn(B, N, H, D, generator=g, dtype=torch.float32).to(dtype)


def algorithmic_flops(wl: Workload) -> float:
    """sum_p 2*2*B*H*(N/r)*(w/r)*D, halved when causal (sparse work only)."""
    tot = 0.0
    for (w, r) in wl.patterns:
        f = 2.0 * 2.0 * wl.B * wl.H * (wl.N / r) * (w / r) * wl.D
        tot += f / 2.0 if wl.causal else f
    return tot


def exact_pair_count(wl: Workload) -> int:
    """Exact number of (query, key) score pairs the method evaluates: per
    pattern, head and segment, m(m+1)/2 when causal or m^2 when not, with m the
    rows the head keeps in that segment (the last segment may be shorter)."""
    tot = 0
    for (w, r) in wl.patterns:
        n_seg = (wl.N + w - 1) // w
        for h in range(wl.H):
            o = h % r
            for seg in range(n_seg):
                ln = min(w, wl.N - seg * w)
                m = 0 if o >= ln else (ln - o + r - 1) // r
                tot += m * (m + 1) // 2 if wl.causal else m * m
    return tot * wl.B


def algorithmic_bytes(wl: Workload) -> float:
    """q, k, v read once, out written once, lse (fp32) written once."""
    es = 4 if wl.dtype == "fp32" else 2
    return 4.0 * wl.B * wl.N * wl.H * wl.D * es + 4.0 * wl.B * wl.H * wl.N


def pattern_lists(patterns) -> Tuple[List[int], List[int]]:
    return [int(p[0]) for p in patterns], [int(p[1]) for p in patterns]
