"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one of them (CPU only).  The real oracle is never modified: each
mutant is a text edit of oracle.c compiled into a temporary library."""
import os
import subprocess

import pytest

from tests import oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, text in oracle.c, replacement): dropped terms, wrong indices, a
# transposed operand, wrong rounding of the kept-row count, a missing weight.
MUTANTS = [
    ("no_head_offset", "const int64_t o = h % r[p];\n        const int64_t m",
     "const int64_t o = 0;\n        const int64_t m"),
    ("causal_off_by_one", "const int64_t n_keys = causal ? i + 1 : m;",
     "const int64_t n_keys = causal ? (i > 0 ? i : 1) : m;"),
    ("scale_1_over_D", "const double scale = 1.0 / sqrt((double)D);\n  for (int64_t i = 0; i < m; ++i)",
     "const double scale = 1.0 / (double)D;\n  for (int64_t i = 0; i < m; ++i)"),
    ("unweighted_merge", "const double wt = exp(lse_p[p] - mx);", "const double wt = 1.0;"),
    ("lse_without_max", "ls[i] = mx + log(denom);", "ls[i] = log(denom);"),
    ("transposed_qk", "s += qs[i * D + d] * ks[j * D + d];", "s += qs[j * D + d] * ks[i * D + d];"),
    ("floor_row_count", "return (len - o + r - 1) / r;", "return (len - o) / r;"),
    ("partial_segment_short", "return rest < w ? rest : w;", "return rest < w ? rest - 1 : w;"),
    ("partial_segment_dropped", "n_tasks_total += B * H * ((N + w[p] - 1) / w[p]);",
     "n_tasks_total += B * H * (N / w[p]);"),
    ("stride_dropped", "const int64_t pos = seg * w[p] + o + r[p] * i;\n          const int64_t src",
     "const int64_t pos = seg * w[p] + o + i;\n          const int64_t src"),
    ("v_from_query_row", "acc += scores[j] * vs[j * D + d];", "acc += scores[j] * vs[i * D + d];"),
    ("merge_lse_no_log", "*lse = mx + log(wsum);", "*lse = mx + wsum;"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(path), "-lm"])
    from oracle.oracle import load_library

    return load_library(str(lib))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    lib = _build_mutant(tmp_path, name, old, new)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin caught mutant {name}"
