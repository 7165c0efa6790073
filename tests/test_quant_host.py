"""The arithmetic the NVFP4 quantize kernels use in place of runtime
divisions, checked on the CPU: tests/native/quant_check.cu compiles the
kernels' own helpers from nvfp4kv_device.cuh for the host with nvcc --
FastDiv (division by an invariant integer) and div_rn_by_correction
(Markstein's division by correction) -- and compares them with the integer
quotient and the IEEE quotient over tens of millions of operands of the
kernels' domain, rounding ties of E2M1 and of the E4M3 scale included."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_quantizer_division_helpers_match_exact_quotients():
    src = os.path.join(ROOT, "tests", "native", "quant_check.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "quant_check")
        # no contraction on the host: the helper's multiply and fused
        # multiply-adds must run as written
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2",
                        "-Xcompiler", "-ffp-contract=off", "-I", os.path.join(ROOT, "include"), "-o", exe, src],
                       check=True, capture_output=True, text=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
