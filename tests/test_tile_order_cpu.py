"""The tensor-core tile order covers every basis row once, and its feature
generator (device code compiled for the host) reproduces w * prod(x) for every
slot of every tile.  Builds tests/cpu/tile_order_check.cu with nvcc; no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_tile_order_and_generator(tmp_path):
    exe = str(tmp_path / "tile_order_check")
    csrc = os.path.join(ROOT, "linear_cost_attention_b200", "csrc")
    cmd = [_nvcc(), "-std=c++17", "--expt-relaxed-constexpr", "-O1", "-o", exe,
           os.path.join(ROOT, "tests", "cpu", "tile_order_check.cu"),
           os.path.join(csrc, "tile_order.cu"), os.path.join(csrc, "basis.cpp")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0 and "OK" in run.stdout, run.stdout + run.stderr
