"""The decode kernel's shared-memory layout helpers are consistent (CPU only).

Compiles tests/native/layout_check.cu against the kernel header as a host
program and runs it: the row permutation is a bijection, owner-order slots
invert it, and the rows one quarter-warp reads together fall in different
banks under the 128-byte swizzle.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_delta_rule_recurrent_b200", "csrc")


def test_layout_helpers(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "layout_check")
    build = subprocess.run([nvcc, "-std=c++17", "-arch=sm_100a", "--expt-relaxed-constexpr",
                            "-I", CSRC, "-o", exe,
                            os.path.join(ROOT, "tests", "native", "layout_check.cu")],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.count("ok") == 4
