"""fp64 CPU oracle for the multi-pattern dilated-attention forward.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check
and by the benchmark's CPU-baseline leg, never by the product path.  It shares
no code with the CUDA library (see oracle.c for the method it restates).
"""
from .oracle import (  # noqa: F401
    build_oracle,
    dilated_attn_bwd_fp64,
    dilated_attn_bwd_rows_fp64,
    dilated_attn_fp64,
    dilated_attn_rows_fp64,
    num_threads,
    qk_normalize_bwd_fp64,
    qk_normalize_fp64,
    xpos_bwd_fp64,
    xpos_fp64,
)
from .brute import dilated_attn_bruteforce  # noqa: F401
