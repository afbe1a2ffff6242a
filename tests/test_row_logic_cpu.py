"""The kernels' per-row histogram logic, compiled for the host and checked against brute force."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_row_logic_against_brute_force(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = tmp_path / "row_logic_test"
    src = os.path.join(ROOT, "tests", "cpp", "row_logic_test.cu")
    inc = os.path.join(ROOT, "adaptive_sparse_flash_b200", "csrc")
    subprocess.run([nvcc, "-std=c++17", "-O2", "-I", inc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), src],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "ring mask mismatches 0" in out.stdout and "hist_tau mismatches 0" in out.stdout
