"""Host-side invariants of the split-K work partition (compiled with g++ from
the same header the kernels use; no GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_partition_invariants(tmp_path):
    exe = tmp_path / "partition_check"
    src = os.path.join(ROOT, "tests", "native", "partition_check.cpp")
    inc = [os.path.join(ROOT, "weighted_coreset_softmax_b200", "csrc"), os.path.join(ROOT, "include")]
    cmd = ["g++", "-std=c++17", "-O1", src, "-o", str(exe)] + [f"-I{d}" for d in inc]
    subprocess.run(cmd, check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("OK")
