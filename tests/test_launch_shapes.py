"""Launch-shape helpers of the library (host C++), compiled with nvcc as a
host-only program and run on the CPU: layout grids and chunks cover the
tokens and fit the workspace; copy-kernel column slices cover each row in
whole warp-widths."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_launch_shapes(tmp_path):
    exe = tmp_path / "launch_shapes"
    src = os.path.join(ROOT, "tests", "host_cpp", "launch_shapes.cu")
    inc = os.path.join(ROOT, "combine_router_softmax_02_b200", "csrc")
    subprocess.run(["nvcc", "-std=c++17", "--expt-relaxed-constexpr", "-I", inc,
                    "-gencode", "arch=compute_100a,code=sm_100a", "-o", str(exe), src],
                   check=True, capture_output=True, timeout=300)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
