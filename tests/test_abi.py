"""The C-ABI library loads, exports every symbol include/*.h declares, and its
host-only logic (sizes, argument validation) behaves as documented.  No
kernel is launched here: every call below returns before reaching the GPU.
"""
import ctypes
import glob
import os
import re
import shutil
import subprocess

import pytest

import oracle
from bit_decode_attention_b200 import _native
from bit_decode_attention_b200 import build as native_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    native_build.build()
    return _native.lib()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b((?:nvfp4|mxfp4)_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_native.EXPORTS)


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.nvfp4_version()
    assert lib.nvfp4_status_string(0) == b"ok"
    assert lib.nvfp4_status_string(3) == b"sequence past cache capacity"
    assert lib.nvfp4_status_string(99) == b"unknown status"


def test_cache_bytes_matches_oracle_memory_model(lib):
    # one plane = B*H*S*D elements at 4.5 bits; K and V together follow the
    # KV-memory formula of the pages with 4.5-bit elements
    for B, H, S, D in [(8, 8, 4096, 128), (1, 8, 65536, 128), (3, 2, 48, 64)]:
        plane = lib.nvfp4_cache_bytes(B, H, S, D)
        assert plane == B * H * S * (D // 2 + D // 16)
        assert 2 * plane == oracle.kv_bytes(1, H, D, S, B, oracle.nvfp4_bits_per_element())
    assert lib.nvfp4_cache_bytes(1, 0, 16, 128) == 0
    assert lib.nvfp4_cache_bytes(1, 1, 16, 40) == 0
    # MXFP4: 4.25 bits per element (one E8M0 byte per 32 elements)
    for B, H, S, D in [(8, 8, 4096, 128), (3, 2, 48, 64)]:
        plane = lib.mxfp4_cache_bytes(B, H, S, D)
        assert plane == B * H * S * (D // 2 + D // 32)
        assert 2 * plane == oracle.kv_bytes(1, H, D, S, B, oracle.mxfp4_bits_per_element())
    assert lib.mxfp4_cache_bytes(1, 1, 16, 48) == 0


def test_workspace_size(lib):
    assert lib.nvfp4_decode_attention_workspace(8, 32, 8, 128) > 0
    assert lib.nvfp4_decode_attention_workspace(8, 30, 8, 128) == 0   # H_q % H_kv
    assert lib.nvfp4_decode_attention_workspace(8, 8 * 17, 8, 128) == 0  # group > 16
    assert lib.nvfp4_decode_attention_workspace(8, 32, 8, 96) == 0     # head_dim


def _plane(B=1, H=1, S=16, D=128, codes=16, scales=16):
    return _native.KVPlaneStruct(codes, scales, B, H, S, D)


def test_argument_validation_without_gpu(lib):
    p = _plane()
    bad_s = _plane(S=24)
    bad_d = _plane(D=96)
    misaligned = _plane(codes=17)
    dev = ctypes.c_void_p(64)  # never dereferenced: every call below fails validation
    INVALID, WS = _native.NVFP4_ERR_INVALID_ARG, _native.NVFP4_ERR_WORKSPACE
    qa = lib.nvfp4_kv_quantize_append
    assert qa(dev, 0, 1, dev, None, dev, ctypes.byref(bad_s), None, None) == INVALID
    assert qa(dev, 0, 1, dev, None, dev, ctypes.byref(bad_d), None, None) == INVALID
    assert qa(dev, 0, 1, dev, None, dev, ctypes.byref(misaligned), None, None) == INVALID
    assert qa(dev, 7, 1, dev, None, dev, ctypes.byref(p), None, None) == INVALID   # dtype
    assert qa(dev, 0, 1, dev, dev, dev, ctypes.byref(p), None, None) == INVALID    # aliasing
    assert qa(ctypes.c_void_p(72), 0, 1, dev, None, dev, ctypes.byref(p), None, None) == INVALID
    assert qa(dev, 0, 0, dev, None, dev, ctypes.byref(p), None, None) == 0         # no-op
    qkv = lib.nvfp4_kv_quantize_append_kv
    kv_other = _plane(S=32)
    assert qkv(dev, dev, 0, 1, dev, None, dev, dev, ctypes.byref(p), ctypes.byref(kv_other), None, None) == INVALID
    assert qkv(dev, dev, 0, 1, dev, None, None, dev, ctypes.byref(p), ctypes.byref(p), None, None) == INVALID
    assert qkv(dev, ctypes.c_void_p(72), 0, 1, dev, None, dev, dev, ctypes.byref(p), ctypes.byref(p),
               None, None) == INVALID                                                  # V misaligned
    assert qkv(dev, dev, 0, 0, dev, None, dev, dev, ctypes.byref(p), ctypes.byref(p), None, None) == 0
    dq = lib.nvfp4_kv_dequant_fp8
    assert dq(ctypes.byref(p), None, dev, dev, None, None) == INVALID
    assert dq(ctypes.byref(p), dev, dev, ctypes.c_void_p(65), None, None) == INVALID
    at = lib.nvfp4_decode_attention
    k, v = _plane(B=2, H=2), _plane(B=2, H=2)
    v_other = _plane(B=2, H=2, S=32)
    args = lambda hq, kk, vv, ws, nbytes: (dev, 0, hq, ctypes.byref(kk), ctypes.byref(vv), dev, dev,
                                           dev, ctypes.c_float(0.0), dev, ws, nbytes, None, None)
    assert at(*args(3, k, v, dev, 1 << 30)) == INVALID            # H_q % H_kv
    assert at(*args(4, k, v_other, dev, 1 << 30)) == INVALID      # planes disagree
    assert at(*args(2 * 17, k, v, dev, 1 << 30)) == _native.NVFP4_ERR_UNSUPPORTED
    # 2^10 KV heads x 2^21 tokens = 2^26 tiles of 32 tokens per sequence: fits
    # 32-bit tile counts for one sequence, not for 2^6 of them
    big1, big64 = _plane(B=1, H=1 << 10, S=1 << 21), _plane(B=64, H=1 << 10, S=1 << 21)
    assert at(*args(1 << 10, big64, big64, dev, 1 << 30)) == _native.NVFP4_ERR_UNSUPPORTED
    assert at(*args(1 << 10, big1, big1, dev, 16)) == WS           # passes the tile check
    assert at(dev, 0, 4, ctypes.byref(k), ctypes.byref(v), dev, dev, dev, ctypes.c_float(0.0),
              ctypes.c_void_p(68), dev, 1 << 30, None, None) == INVALID   # out misaligned
    assert at(*args(4, k, v, None, 0)) == WS
    assert at(*args(4, k, v, dev, 16)) == WS
    mx = lib.mxfp4_kv_quantize_append
    mxp = _plane(D=128, scales=32)
    assert mx(dev, 0, 1, dev, None, ctypes.byref(bad_s), None, None) == INVALID
    assert mx(dev, 7, 1, dev, None, ctypes.byref(mxp), None, None) == INVALID       # dtype
    assert mx(dev, 0, 1, dev, dev, ctypes.byref(mxp), None, None) == INVALID        # aliasing
    assert mx(ctypes.c_void_p(72), 0, 1, dev, None, ctypes.byref(mxp), None, None) == INVALID
    assert mx(dev, 0, 1, None, None, ctypes.byref(mxp), None, None) == INVALID      # no start
    assert mx(dev, 0, 0, dev, None, ctypes.byref(mxp), None, None) == 0             # no-op
    # paged planes: page_tokens a multiple of 128, a block table, a shared table for K and V
    PP = _native.PagedPlaneStruct
    tbl = ctypes.c_void_p(256)
    pg = PP(16, 16, tbl, 4, 2, 128, 128, 2, 3)
    pg_other = PP(16, 16, ctypes.c_void_p(512), 4, 2, 128, 128, 2, 3)
    bad_pages = [PP(16, 16, tbl, 4, 2, 96, 128, 2, 3),      # page not a multiple of 128
                 PP(16, 16, None, 4, 2, 128, 128, 2, 3),     # no block table
                 PP(16, 16, tbl, 0, 2, 128, 128, 2, 3),      # empty pool
                 PP(16, 16, tbl, 4, 2, 128, 96, 2, 3),       # head_dim
                 PP(16, 16, tbl, 4, 2, 1 << 24, 128, 2, 1 << 10),   # capacity past 2^31
                 PP(17, 16, tbl, 4, 2, 128, 128, 2, 3)]      # misaligned codes
    qp = lib.nvfp4_kv_quantize_append_paged
    for bp in bad_pages:
        assert qp(dev, 0, 1, dev, None, dev, ctypes.byref(bp), None, None) == INVALID
    assert qp(dev, 0, 1, dev, None, None, ctypes.byref(pg), None, None) == INVALID     # no scale
    assert qp(dev, 0, 0, dev, None, dev, ctypes.byref(pg), None, None) == 0            # no-op
    ap = lib.nvfp4_decode_attention_paged
    pargs = lambda kk, vv, ws, nbytes: (dev, 0, 4, ctypes.byref(kk), ctypes.byref(vv), dev, dev, dev,
                                        ctypes.c_float(0.0), dev, ws, nbytes, None, None)
    for bp in bad_pages:
        assert ap(*pargs(bp, bp, dev, 1 << 30)) == INVALID
    assert ap(*pargs(pg, pg_other, dev, 1 << 30)) == INVALID     # K and V tables differ
    assert ap(*pargs(pg, pg, dev, 16)) == WS
    # chunked prefill: head_dim 128 and bf16 queries only; checks before any launch
    pf = lib.nvfp4_prefill_attention
    k128, v128 = _plane(B=2, H=2), _plane(B=2, H=2)
    k64 = _plane(B=2, H=2, D=64)
    pfa = lambda q, dt, C, hq, kk, vv, st, scale, out: (q, dt, C, hq, ctypes.byref(kk), ctypes.byref(vv), dev,
                                                        dev, st, ctypes.c_float(scale), out, None, None)
    UNSUP = _native.NVFP4_ERR_UNSUPPORTED
    assert pf(*pfa(dev, 0, 16, 3, k128, v128, dev, 0.0, dev)) == INVALID        # H_q % H_kv
    assert pf(*pfa(dev, 0, 16, 4, k128, v_other, dev, 0.0, dev)) == INVALID     # planes disagree
    assert pf(*pfa(dev, 0, -1, 4, k128, v128, dev, 0.0, dev)) == INVALID        # negative chunk
    assert pf(*pfa(dev, 0, 16, 4, k128, v128, None, 0.0, dev)) == INVALID       # no start positions
    assert pf(*pfa(dev, 0, 16, 4, k128, v128, dev, -1.0, dev)) == INVALID       # softmax scale
    assert pf(*pfa(dev, 7, 16, 4, k128, v128, dev, 0.0, dev)) == INVALID        # dtype
    assert pf(*pfa(dev, 1, 16, 4, k128, v128, dev, 0.0, dev)) == UNSUP          # fp32 queries
    assert pf(*pfa(dev, 0, 16, 4, k64, k64, dev, 0.0, dev)) == UNSUP            # head_dim 64
    assert pf(*pfa(ctypes.c_void_p(72), 0, 16, 4, k128, v128, dev, 0.0, dev)) == INVALID   # q misaligned
    assert pf(*pfa(dev, 0, 16, 4, k128, v128, dev, 0.0, None)) == INVALID       # no output
    assert pf(*pfa(dev, 0, 0, 4, k128, v128, dev, 0.0, dev)) == 0               # empty chunk: no-op
    cal = lib.nvfp4_calib_tensor_scale
    assert cal(dev, 0, -1, dev, None, None) == INVALID
    assert cal(dev, 0, 10, None, None, None) == INVALID
    assert cal(ctypes.c_void_p(65), 0, 10, dev, None, None) == INVALID   # bf16 misaligned


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_plain_c_and_links(lib, tmp_path):
    # the boundary is a C ABI: a C99 program (-pedantic, no C++) includes the
    # header, links the library and calls its host-only entry points
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "nvfp4kv.h"\n'
        '#include <stdio.h>\n'
        'int main(void) {\n'
        '    nvfp4_kv_plane p = {0};\n'
        '    nvfp4_kv_paged_plane q = {0};\n'
        '    (void)p; (void)q;\n'
        '    printf("%zu %zu %s\\n", nvfp4_cache_bytes(2, 8, 4096, 128), mxfp4_cache_bytes(2, 8, 4096, 128),\n'
        '           nvfp4_status_string(NVFP4_ERR_CAPACITY));\n'
        '    return 0;\n'
        '}\n')
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_native.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lnvfp4kv",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) == 2 * 8 * 4096 * (64 + 8)
    assert int(out[1]) == 2 * 8 * 4096 * (64 + 4)
    assert len(out) > 2


def test_missing_library_raises_and_cpu_tensors_are_refused(lib, monkeypatch):
    # no CPU path: without the built library every call raises, and host
    # tensors are refused before anything reaches the library
    import torch

    import bit_decode_attention_b200 as nv
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", os.path.join(ROOT, "no", "such", "libnvfp4kv.so"))
    with pytest.raises(RuntimeError, match="not built"):
        _native.lib()
    monkeypatch.undo()
    x = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16)
    plane = nv.KVPlane(torch.zeros(1, 1, 16, 64, dtype=torch.uint8), torch.zeros(1, 1, 16, 8, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA"):
        nv.nvfp4_kv_quantize_append(x, torch.zeros(1, dtype=torch.int32), torch.ones(1), plane)
    with pytest.raises(ValueError, match="CUDA"):
        nv.nvfp4_calib_tensor_scale(x)
