"""Host-side checks of the tcgen05 kernel's tile logic (tests/host/tile_walk_check.cu).

The kernel source is compiled with nvcc for sm_100a, but only its host code
runs: the tile walk and combination order, the parking-slot lifetimes, the TMA
coordinates, and the multiply-shift divider against integer division, on the
named shapes and 300 seeded random ones (with SM counts that change the unit
plan).  Every case prints OK and the program exits 0.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_tile_walk_host_checks():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "tile_walk_check")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "sparse_long_sequence_attn_b200", "csrc"),
           "--expt-relaxed-constexpr", "-o", exe,
           os.path.join(ROOT, "tests", "host", "tile_walk_check.cu")]
    subprocess.run(cmd, check=True, capture_output=True, timeout=600)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]
    assert "fails=0" in res.stdout
    assert "fastdiv OK" in res.stdout
    assert "FAIL" not in res.stdout
    # the seeded random shapes: most of them must be ones the kernel takes
    line = [l for l in res.stdout.splitlines() if l.startswith("random cases:")][0]
    assert int(line.split()[2]) >= 200, line
