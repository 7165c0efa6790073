"""nvfp4_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (the library supplies the scratch from a built-in
device buffer).  Collected last on purpose: if it fails, every other test has
already run.  Its GPU check calls the entry point through the C ABI and
compares with nvfp4_decode_attention on two calls in a row."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic
from bit_decode_attention_b200 import _native


def _plane_struct(plane):
    return plane.struct()


def test_noalloc_rejects_shapes_past_its_buffer():
    lib = _native.lib()
    # counters alone (B * H_kv int32) would need 32 MiB: rejected before any GPU work
    kp = _native.KVPlaneStruct(256, 512, 1 << 20, 8, 16, 128)
    vp = _native.KVPlaneStruct(768, 1024, 1 << 20, 8, 16, 128)
    rc = lib.nvfp4_decode_attention_noalloc(ctypes.c_void_p(64), 0, 32, ctypes.byref(kp),
                                            ctypes.byref(vp), ctypes.c_void_p(64), ctypes.c_void_p(64),
                                            ctypes.c_void_p(64), ctypes.c_float(0.0),
                                            ctypes.c_void_p(64), None, None)
    assert rc == _native.NVFP4_ERR_WORKSPACE


def test_noalloc_checks_arguments_like_the_workspace_entry_point():
    lib = _native.lib()
    kp = _native.KVPlaneStruct(256, 512, 2, 2, 16, 128)
    vp = _native.KVPlaneStruct(768, 1024, 2, 2, 16, 128)
    p = ctypes.c_void_p(64)

    def call(H_q, q=p, out=p, scale=0.0, dtype=0):
        return lib.nvfp4_decode_attention_noalloc(q, dtype, H_q, ctypes.byref(kp), ctypes.byref(vp), p, p,
                                                  p, ctypes.c_float(scale), out, None, None)
    # a GQA group past 16 is a valid request this build does not handle, as for
    # nvfp4_decode_attention (checked before any GPU work)
    assert call(34) == _native.NVFP4_ERR_UNSUPPORTED
    assert call(3) == _native.NVFP4_ERR_INVALID_ARG                   # H_q not a multiple of H_kv
    assert call(4, q=ctypes.c_void_p(72)) == _native.NVFP4_ERR_INVALID_ARG   # misaligned q
    assert call(4, out=None) == _native.NVFP4_ERR_INVALID_ARG
    assert call(4, scale=float("nan")) == _native.NVFP4_ERR_INVALID_ARG
    assert call(4, dtype=7) == _native.NVFP4_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    from cases import ATOL_MAX, ATOL_MEAN, Case
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=3, Hq=16, Hkv=4), lens=[700, 33, 1500])
    want = c.gpu_attention().cpu().numpy()              # existing entry point, own workspace
    lib = _native.lib()
    kp, vp = _plane_struct(c.k), _plane_struct(c.v)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):                                   # two calls in a row share the buffer
        out = torch.full_like(c.q_dev, float("nan"), dtype=torch.float32)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = lib.nvfp4_decode_attention_noalloc(
            ctypes.c_void_p(c.q_dev.data_ptr()), _native.NVFP4_IN_BF16, c.w.Hq, ctypes.byref(kp),
            ctypes.byref(vp), ctypes.c_void_p(c.sk.data_ptr()), ctypes.c_void_p(c.sv.data_ptr()),
            ctypes.c_void_p(c.seq_lens.data_ptr()), ctypes.c_float(0.0),
            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(status.data_ptr()), stream)
        assert rc == _native.NVFP4_OK
        torch.cuda.synchronize()
        assert status.item() == 0
        err = np.abs(out.cpu().numpy().astype(np.float64) - want)
        assert np.all(np.isfinite(err))
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN


@pytest.mark.gpu
def test_noalloc_largest_group_fills_most_of_the_buffer():
    """GQA group 16 at head_dim 128: the split partials take most of the 8 MiB
    buffer; results still match the workspace entry point."""
    from cases import ATOL_MAX, ATOL_MEAN, Case
    c = Case(synthetic.shrink(synthetic.get("gqa"), B=2, Hq=32, Hkv=2), lens=[9000, 300])
    want = c.gpu_attention().cpu().numpy()
    import bit_decode_attention_b200 as nv
    assert nv.nvfp4_decode_attention_workspace(2, 32, 2, 128) > 4 << 20
    for _ in range(2):
        got = nv.nvfp4_decode_attention_noalloc(c.q_dev, c.k, c.v, c.sk, c.sv, c.seq_lens).cpu().numpy()
        err = np.abs(got.astype(np.float64) - want)
        assert np.all(np.isfinite(err))
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN
