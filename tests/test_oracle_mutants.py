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
    # backward: a dropped term, a wrong operand, a missing weight, a sign, a bound
    ("bwd_no_delta", "const double ds = pij * (dp - delta + dls[i]);",
     "const double ds = pij * (dp + dls[i]);"),
    ("bwd_no_dlse", "const double ds = pij * (dp - delta + dls[i]);",
     "const double ds = pij * (dp - delta);"),
    ("bwd_dk_from_k", "dks[j * D + d] += scale * ds * qs[i * D + d];",
     "dks[j * D + d] += scale * ds * ks[i * D + d];"),
    ("bwd_dv_without_prob", "dvs[j * D + d] += pij * dos[i * D + d];",
     "dvs[j * D + d] += dos[i * D + d];"),
    ("bwd_unweighted_cotangent", "do_p[p][d] = a * dout[d];", "do_p[p][d] = dout[d];"),
    ("bwd_combine_sign", "dot += dout[d] * (o_p[p][d] - out[d]);",
     "dot += dout[d] * (out[d] - o_p[p][d]);"),
    ("bwd_rows_causal_start", "for (int64_t i = causal ? j : 0; i < m; ++i) {",
     "for (int64_t i = causal ? j + 1 : 0; i < m; ++i) {"),
    ("bwd_rows_dq_scale", "for (int64_t d = 0; d < D; ++d) dq_r[d] += scale * ds * kj[d];",
     "for (int64_t d = 0; d < D; ++d) dq_r[d] += ds * kj[d];"),
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


# The chain rule through the qk normalisation lives in oracle.py: planted
# mistakes there are swapped in for the duration of the check.
def _no_projection(x, dxhat):
    import numpy as np

    from oracle.oracle import _f64

    x, dxhat = _f64(x), _f64(dxhat)
    return dxhat / np.maximum(np.sqrt((x * x).sum(axis=-1, keepdims=True)), 1e-12)


def _squared_norm_scale(x, dxhat):
    import numpy as np

    from oracle.oracle import _f64

    x, dxhat = _f64(x), _f64(dxhat)
    n2 = np.maximum((x * x).sum(axis=-1, keepdims=True), 1e-24)
    xhat = x / np.sqrt(n2)
    return (dxhat - xhat * (xhat * dxhat).sum(axis=-1, keepdims=True)) / n2


@pytest.mark.parametrize("mutant", [_no_projection, _squared_norm_scale],
                         ids=lambda f: f.__name__.strip("_"))
def test_pins_catch_python_mutant(monkeypatch, oracle_lib, mutant):
    import oracle.oracle as orc

    monkeypatch.setattr(orc, "qk_normalize_bwd_fp64", mutant)
    with pytest.raises(AssertionError):
        pins.check_bwd_qk_norm(oracle_lib)


def _xpos_variant(sin_sign=1.0, halves=False, invert_keys=True, gamma=0.4, freq_step=2.0, base=512.0):
    """An XPOS with one planted mistake (the parameters name it)."""
    import numpy as np

    from oracle.oracle import _f64

    def xp(x, downscale=False):
        x = _f64(x)
        B, N, H, D = x.shape
        n = np.arange(N, dtype=np.float64)[:, None]
        i = np.arange(D // 2, dtype=np.float64)[None, :]
        theta = 10000.0 ** (-freq_step * i / D)
        zeta = (2.0 * i + gamma * D) / ((1.0 + gamma) * D)
        s = zeta ** ((n - N // 2) / base)
        if downscale and invert_keys:
            s = 1.0 / s
        cos = (np.cos(n * theta) * s)[None, :, None, :]
        sin = (sin_sign * np.sin(n * theta) * s)[None, :, None, :]
        if halves:
            a, b = x[..., : D // 2], x[..., D // 2:]
        else:
            a, b = x[..., 0::2], x[..., 1::2]
        y = np.empty_like(x)
        ya, yb = a * cos - b * sin, b * cos + a * sin
        if halves:
            y[..., : D // 2], y[..., D // 2:] = ya, yb
        else:
            y[..., 0::2], y[..., 1::2] = ya, yb
        return y

    return xp


XPOS_MUTANTS = {
    "sin_sign": dict(sin_sign=-1.0),
    "half_split_pairs": dict(halves=True),
    "keys_not_inverted": dict(invert_keys=False),
    "gamma_0p5": dict(gamma=0.5),
    "freq_step_1": dict(freq_step=1.0),
    "scale_base_256": dict(base=256.0),
}


@pytest.mark.parametrize("name", sorted(XPOS_MUTANTS))
def test_xpos_pins_catch_mutant(oracle_lib, name):
    with pytest.raises(AssertionError):
        pins.check_xpos(oracle_lib, xpos=_xpos_variant(**XPOS_MUTANTS[name]))


def test_xpos_unmutated_variant_passes(oracle_lib):
    pins.check_xpos(oracle_lib, xpos=_xpos_variant())


def _xpos_bwd_variant(sin_sign=1.0, invert_keys=True):
    """xpos_bwd with one planted mistake: the rotation's direction, or the key scale."""
    import numpy as np

    from oracle.oracle import _f64

    def xb(g, downscale=False):
        g = _f64(g)
        B, N, H, D = g.shape
        n = np.arange(N, dtype=np.float64)[:, None]
        i = np.arange(D // 2, dtype=np.float64)[None, :]
        theta = 10000.0 ** (-2.0 * i / D)
        zeta = (2.0 * i + 0.4 * D) / (1.4 * D)
        s = zeta ** ((n - N // 2) / 512.0)
        if downscale and invert_keys:
            s = 1.0 / s
        cos = (np.cos(n * theta) * s)[None, :, None, :]
        sin = (sin_sign * np.sin(n * theta) * s)[None, :, None, :]
        g0, g1 = g[..., 0::2], g[..., 1::2]
        x = np.empty_like(g)
        x[..., 0::2] = g0 * cos + g1 * sin
        x[..., 1::2] = g1 * cos - g0 * sin
        return x

    return xb


@pytest.mark.parametrize("kw", [dict(sin_sign=-1.0), dict(invert_keys=False)], ids=["rotation_sign", "key_scale"])
def test_xpos_backward_pins_catch_mutant(oracle_lib, kw):
    with pytest.raises(AssertionError):
        pins.check_bwd_xpos(oracle_lib, xpos_bwd=_xpos_bwd_variant(**kw))
