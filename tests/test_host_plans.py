"""Host logic: the launch planners of the persistent and split kernels, built
from the library's own sources into a host-only harness (tests/plan_harness.cu)
and checked against the invariants their kernels rely on -- shared memory per
CTA, warp counts, shape preconditions, and that every cell a warp shares is
cut into exactly two parts.  No GPU is needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not found")
def test_planner_invariants(tmp_path):
    exe = tmp_path / "plan_harness"
    cmd = ["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=compute_100a",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "decode_packed_bit_b200", "csrc"),
           os.path.join(ROOT, "tests", "plan_harness.cu"), "-o", str(exe)]
    build = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert build.returncode == 0, build.stderr[-2000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout[-2000:]
    assert " 0 failed" in run.stdout
