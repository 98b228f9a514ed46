"""CPU check of the work-splitting arithmetic shared by the kernels (piece
bounds, piece owner, automatic piece count, units per segment): the helpers in
csrc/pa_device.cuh are host-callable, and tests/host_plan_check.cu exercises
their invariants over random streams."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_splitting_arithmetic_invariants():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "plan_check")
        subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", os.path.join(ROOT, "paged_split_kv_attention_b200", "csrc"),
                        "-o", exe, os.path.join(ROOT, "tests", "host_plan_check.cu")],
                       check=True, capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout
    assert "ok" in r.stdout
