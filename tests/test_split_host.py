"""The stream-K split-K bookkeeping of the decode-attention kernels, checked on
the CPU: tests/native/split_check.cu compiles the kernels' own index helpers
(CTA ranges, tile owner, contributor count, the partial slot a contributor
writes and the slot the merge reads, the unit lookup) for the host with nvcc
and compares them with brute force over thousands of splits."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_split_bookkeeping_matches_brute_force():
    src = os.path.join(ROOT, "tests", "native", "split_check.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "split_check")
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                        "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-o", exe, src],
                       check=True, capture_output=True, text=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
