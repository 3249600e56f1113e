"""The GEMM tiling planner's choices satisfy the launch path's requirements
(tests/native/planner_check.cu, a host-only program built from the runtime's
source and the library's other objects; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not on PATH")
def test_gemm_planner_choices(tmp_path):
    from token_locking_b200 import build as b
    b.build()
    objs = [os.path.join(b.BUILD, f) for f in ("layers.o", "lock.o", "attn.o", "attn_tc.o", "gemm_tc.o")]
    exe = str(tmp_path / "planner_check")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
           "-I" + os.path.join(ROOT, "include"), "-I" + b.CSRC,
           os.path.join(ROOT, "tests", "native", "planner_check.cu"), *objs, "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    print(r.stdout)
    assert r.returncode == 0, r.stdout[-4000:]
    assert " 0 failures" in r.stdout
