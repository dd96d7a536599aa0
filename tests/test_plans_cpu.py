"""The launch planners against the invariants their kernels rely on (host
only: tests/host/plan_check.cu is compiled with nvcc, linked to libqs.so and
run without a GPU)."""
import os
import subprocess

import pytest

from top_activation_sparse_b200 import build as qs_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plans_keep_their_invariants(tmp_path):
    try:
        nvcc = qs_build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    lib = qs_build.build()
    exe = tmp_path / "plan_check"
    csrc = os.path.join(ROOT, "top_activation_sparse_b200", "csrc")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"), "-I", csrc,
                    os.path.join(ROOT, "tests", "host", "plan_check.cu"), "-o", str(exe),
                    "-L", os.path.dirname(lib), "-lqs", f"-Xlinker=-rpath={os.path.dirname(lib)}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert " 0 failed" in r.stdout
