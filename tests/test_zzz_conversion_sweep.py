"""The hardware format conversions the kernels use, against the oracle's
encoders over every finite fp32 bit pattern (2^32 - 2^24 of them), on the GPU.

tests/native/conversion_sweep.cu is compiled into a shared library that runs
the kernels' own conversion helpers from nvfp4kv_device.cuh: the E2M1 encode
of the quantizer's fast path (cvt.rn.satfinite.e2m1x2.f32), the E4M3 encode of
the attention kernels' query and probability splits
(cvt.rn.satfinite.e4m3x2.f32), and the exact E4M3 -> f16 decode
(cvt.rn.f16x2.e4m3x2).  Every byte must equal the oracle's -- round to
nearest even, saturation at the largest finite value, the sign of zero.
Non-finite inputs are left out: the quantizer sends blocks holding a NaN or an
infinity to its comparison encoder, never to the hardware conversion.

The file's name makes it the last GPU test to run: it takes tens of seconds of
host time (the oracle encodes every pattern, on all host cores)."""
import ctypes
import os
import shutil
import subprocess
import tempfile
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHUNK = 1 << 22                       # fp32 patterns per launch


def _build(tmp):
    src = os.path.join(ROOT, "tests", "native", "conversion_sweep.cu")
    so = os.path.join(tmp, "conversion_sweep.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-o", so, src],
                   check=True, capture_output=True, text=True)
    lib = ctypes.CDLL(so)
    lib.sweep_encode_patterns.argtypes = [ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    lib.sweep_encode_patterns.restype = ctypes.c_int
    lib.sweep_decode_bytes.argtypes = [ctypes.c_void_p]
    lib.sweep_decode_bytes.restype = ctypes.c_int
    return lib


def _compare_chunk(first, got_e2m1, got_e4m3):
    """Mismatch counts and first examples (pattern, device byte, oracle byte)
    of one chunk, finite patterns only."""
    bits = np.arange(first, first + CHUNK, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    finite = (bits & np.uint32(0x7F800000)) != np.uint32(0x7F800000)
    out = []
    for got, want in ((got_e2m1, oracle.e2m1_encode(v)), (got_e4m3, oracle.e4m3_encode(v))):
        bad = np.flatnonzero((got != want) & finite)
        out.append((bad.size, [(hex(int(bits[i])), int(got[i]), int(want[i])) for i in bad[:5]]))
    return out


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_sweep_library_builds_and_exports_its_calls():
    # CPU: the GPU sweep's library compiles and loads (no device call)
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build(tmp)
        assert lib.sweep_encode_patterns and lib.sweep_decode_bytes


def test_sweep_comparison_finds_planted_mismatches():
    # CPU: the host half of the sweep, given the oracle's own bytes with one
    # wrong byte per format planted in a finite pattern and one in a NaN
    first = 0x3F000000
    bits = np.arange(first, first + CHUNK, dtype=np.uint64).astype(np.uint32)
    e2m1, e4m3 = oracle.e2m1_encode(bits.view(np.float32)), oracle.e4m3_encode(bits.view(np.float32))
    assert [n for n, _ in _compare_chunk(first, e2m1, e4m3)] == [0, 0]
    e2m1[77] ^= 0x1
    e4m3[CHUNK - 1] ^= 0x80
    (n1, ex1), (n2, ex2) = _compare_chunk(first, e2m1, e4m3)
    assert (n1, n2) == (1, 1) and ex1[0][0] == hex(first + 77) and ex2[0][0] == hex(first + CHUNK - 1)
    nan_first = 0x7FC00000
    nan_bits = np.arange(nan_first, nan_first + CHUNK, dtype=np.uint64).astype(np.uint32)
    e2m1 = oracle.e2m1_encode(nan_bits.view(np.float32))
    e2m1[5] ^= 0x1
    assert _compare_chunk(nan_first, e2m1, oracle.e4m3_encode(nan_bits.view(np.float32)))[0][0] == 0


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_hardware_conversions_match_oracle_on_every_finite_float():
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build(tmp)
        torch.cuda.init()

        # the 256 E4M3 bytes through the f16 decode, bit for bit (NaN bytes: NaN)
        d_dec = torch.empty(256, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        assert lib.sweep_decode_bytes(d_dec.data_ptr()) == 0
        got = d_dec.cpu().numpy()
        want = np.array([oracle.e4m3_value(b) for b in range(256)], np.float32)
        nan = np.isnan(want)
        assert np.array_equal(np.isnan(got), nan)
        np.testing.assert_array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))

        # every fp32 pattern through both encoders; the host compares each
        # chunk with the oracle on a pool of threads (the oracle's calls
        # release the interpreter lock) while the device converts the next
        d_e2m1 = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
        d_e4m3 = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        n_threads = max(1, min(32, os.cpu_count() or 1))
        counts = [0, 0]
        examples = [[], []]

        def collect(fut):
            for k, (n, ex) in enumerate(fut.result()):
                counts[k] += n
                if len(examples[k]) < 10:
                    examples[k].extend(ex)

        with ThreadPoolExecutor(n_threads) as pool:
            pending = []
            for first in range(0, 1 << 32, CHUNK):
                rc = lib.sweep_encode_patterns(first, CHUNK, d_e2m1.data_ptr(), d_e4m3.data_ptr())
                assert rc == 0, "sweep launch failed with %d at pattern %#x" % (rc, first)
                pending.append(pool.submit(_compare_chunk, first, d_e2m1.cpu().numpy(), d_e4m3.cpu().numpy()))
                while len(pending) >= 2 * n_threads:
                    collect(pending.pop(0))
            for fut in pending:
                collect(fut)
    assert counts == [0, 0], {"e2m1 (pattern, device, oracle)": examples[0],
                              "e4m3 (pattern, device, oracle)": examples[1], "counts": counts}
