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
