"""The format conversions the kernels use, against the oracle's encoders over
every fp32 bit pattern, on the GPU.

tests/native/conversion_sweep.cu is compiled into a shared library that runs
the kernels' own conversion helpers from nvfp4kv_device.cuh:

* hardware: the E2M1 encode of the quantizer's fast path
  (cvt.rn.satfinite.e2m1x2.f32), the E4M3 encode of the attention kernels'
  query and probability splits (cvt.rn.satfinite.e4m3x2.f32), and the exact
  E4M3 -> f16 decode (cvt.rn.f16x2.e4m3x2), all 256 bytes;
* software: e2m1_from_float and e4m3_from_float (the quantizer's general path,
  its scale bytes, the dequant tables), e4m3_to_float and e2m1_magnitude.

Every byte must equal the oracle's -- round to nearest even, saturation at
the largest finite value, the sign of zero.  The software encoders are
compared on all 2^32 patterns (NaN and infinities included: they take them);
the hardware encoders on the 2^32 - 2^24 finite ones, the only inputs the
kernels give them (the quantizer sends blocks holding a NaN or an infinity to
its software encoder).

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
    lib.sweep_encode_patterns.argtypes = [ctypes.c_uint32, ctypes.c_uint64] + [ctypes.c_void_p] * 4
    lib.sweep_encode_patterns.restype = ctypes.c_int
    lib.sweep_decode_bytes.argtypes = [ctypes.c_void_p]
    lib.sweep_decode_bytes.restype = ctypes.c_int
    return lib


NAMES = ("hardware e2m1", "hardware e4m3", "software e2m1", "software e4m3")


def _compare_chunk(first, hw_e2m1, hw_e4m3, sw_e2m1, sw_e4m3):
    """Mismatch counts and first examples (pattern, device byte, oracle byte)
    of one chunk, per conversion in NAMES order: the hardware ones on finite
    patterns, the software ones on every pattern."""
    bits = np.arange(first, first + CHUNK, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    finite = (bits & np.uint32(0x7F800000)) != np.uint32(0x7F800000)
    want_e2m1, want_e4m3 = oracle.e2m1_encode(v), oracle.e4m3_encode(v)
    out = []
    for got, want, mask in ((hw_e2m1, want_e2m1, finite), (hw_e4m3, want_e4m3, finite),
                            (sw_e2m1, want_e2m1, None), (sw_e4m3, want_e4m3, None)):
        diff = got != want
        if mask is not None:
            diff &= mask
        bad = np.flatnonzero(diff)
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
    # wrong byte planted per conversion; in a NaN chunk only the software
    # conversions' plants count
    for first, want_counts in ((0x3F000000, [1, 1, 1, 1]), (0x7FC00000, [0, 0, 1, 1])):
        bits = np.arange(first, first + CHUNK, dtype=np.uint64).astype(np.uint32)
        e2m1, e4m3 = oracle.e2m1_encode(bits.view(np.float32)), oracle.e4m3_encode(bits.view(np.float32))
        got = [e2m1.copy(), e4m3.copy(), e2m1.copy(), e4m3.copy()]
        assert [n for n, _ in _compare_chunk(first, *got)] == [0, 0, 0, 0]
        at = [77, CHUNK - 1, 0, 12345]
        for k in range(4):
            got[k][at[k]] ^= 0x1
        res = _compare_chunk(first, *got)
        assert [n for n, _ in res] == want_counts
        for k in range(4):
            if want_counts[k]:
                assert res[k][1][0][0] == hex(first + at[k])


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_hardware_conversions_match_oracle_on_every_finite_float():
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build(tmp)
        torch.cuda.init()

        # the 256 E4M3 bytes through the hardware f16 decode and through
        # e4m3_to_float, bit for bit (NaN bytes: NaN from the hardware, not
        # taken by the software decoder), and the 8 E2M1 magnitudes
        d_dec = torch.empty(520, dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        assert lib.sweep_decode_bytes(d_dec.data_ptr()) == 0
        dec = d_dec.cpu().numpy()
        want = np.array([oracle.e4m3_value(b) for b in range(256)], np.float32)
        nan = np.isnan(want)
        assert np.array_equal(np.isnan(dec[:256]), nan)
        np.testing.assert_array_equal(dec[:256][~nan].view(np.uint32), want[~nan].view(np.uint32))
        np.testing.assert_array_equal(dec[256:512][~nan].view(np.uint32), want[~nan].view(np.uint32))
        np.testing.assert_array_equal(dec[512:520], np.array([oracle.e2m1_value(c) for c in range(8)], np.float32))

        # every fp32 pattern through the four encoders; the host compares each
        # chunk with the oracle on a pool of threads (the oracle's calls
        # release the interpreter lock) while the device converts the next
        bufs = [torch.empty(CHUNK, dtype=torch.uint8, device="cuda") for _ in range(4)]
        torch.cuda.synchronize()
        n_threads = max(1, min(32, os.cpu_count() or 1))
        counts = [0] * 4
        examples = [[] for _ in range(4)]

        def collect(fut):
            for k, (n, ex) in enumerate(fut.result()):
                counts[k] += n
                if len(examples[k]) < 10:
                    examples[k].extend(ex)

        with ThreadPoolExecutor(n_threads) as pool:
            pending = []
            for first in range(0, 1 << 32, CHUNK):
                rc = lib.sweep_encode_patterns(first, CHUNK, *[b.data_ptr() for b in bufs])
                assert rc == 0, "sweep launch failed with %d at pattern %#x" % (rc, first)
                pending.append(pool.submit(_compare_chunk, first, *[b.cpu().numpy() for b in bufs]))
                while len(pending) >= 2 * n_threads:
                    collect(pending.pop(0))
            for fut in pending:
                collect(fut)
    assert counts == [0] * 4, {NAMES[k] + " (pattern, device, oracle)": examples[k] for k in range(4)}
