"""Build-time resource checks of the tensor-core attention kernels (CPU only:
ptxas runs here without a GPU).  Their warpgroups resize their register files
at run time (setmaxnreg), so the kernels must use no local memory: no stack
frame and no spills."""
import os
import re
import subprocess

import pytest

from bit_decode_attention_b200 import build as nvbuild

SRC = os.path.join(nvbuild.CSRC, "nvfp4kv_decode_attention_tc.cu")


def test_tensor_core_kernels_use_no_local_memory(tmp_path):
    out = str(tmp_path / "tc.o")
    cmd = [nvbuild.nvcc(), *[f for f in nvbuild.NVCC_FLAGS if f != "-shared"], "-c", "-Xptxas", "-v",
           "-I", nvbuild.INCLUDE, "-o", out, SRC]
    try:
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    except FileNotFoundError:
        pytest.skip("nvcc not available")
    assert r.returncode == 0, r.stderr[-2000:]
    info = r.stderr
    blocks = re.findall(r"Compiling entry function '([^']+)'.*?\n(.*?)ptxas info\s+: Used (\d+) registers",
                        info, flags=re.S)
    tc = [(name, body) for name, body, _ in blocks if "decode_attention_tc_kernel" in name]
    assert len(tc) == 2, "expected the two tensor-core kernel instantiations"
    for name, body in tc:
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", body)
        assert m is not None, body
        assert m.groups() == ("0", "0", "0"), "%s: %s" % (name, m.group(0))
