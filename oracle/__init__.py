"""CPU oracle for the NVFP4 KV-cache path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``bit_decode_attention_b200``) never imports it, and the two
share no code.  The arithmetic lives in ``nvfp4_oracle.c``; this module only
marshals numpy arrays through ctypes.

Each wrapper names the page passage its C function follows; see the C file.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode_array.argtypes = [f32p, ctypes.c_int64, u8p]
        L.oracle_e4m3_encode_array.argtypes = [f32p, ctypes.c_int64, u8p]
        L.oracle_tensor_scale.argtypes = [f32p, ctypes.c_int64, f32p]
        L.oracle_tensor_scale.restype = ctypes.c_int
        L.oracle_quantize_block.argtypes = [f32p, ctypes.c_float, u8p, u8p]
        L.oracle_quantize_append.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, i32p, ctypes.c_float, u8p, u8p,
                                             ctypes.c_int]
        L.oracle_quantize_append.restype = ctypes.c_int
        L.oracle_dequant_fp8.argtypes = [ctypes.c_uint8, ctypes.c_uint8, ctypes.c_float]
        L.oracle_dequant_fp8.restype = ctypes.c_uint8
        L.oracle_dequant_planes.argtypes = [u8p, u8p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_float, i32p, u8p]
        L.oracle_decode_attention_fp8.argtypes = [f32p, u8p, u8p, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  i32p, ctypes.c_double, f64p]
        L.oracle_decode_attention_nvfp4.argtypes = [f32p, u8p, u8p, u8p, u8p, ctypes.c_float,
                                                    ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    i32p, ctypes.c_double, f64p]
        L.oracle_kv_bytes.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_double]
        L.oracle_nvfp4_reconstruct_planes.argtypes = [u8p, u8p, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                                      i32p, f64p]
        L.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_value.restype = ctypes.c_double
        L.oracle_mxfp4_quantize_block.argtypes = [f32p, u8p, u8p]
        L.oracle_mxfp4_quantize_block.restype = ctypes.c_int
        L.oracle_mxfp4_quantize_append.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, i32p, u8p, u8p, ctypes.c_int]
        L.oracle_mxfp4_quantize_append.restype = ctypes.c_int
        L.oracle_mxfp4_reconstruct_planes.argtypes = [u8p, u8p, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_int, i32p, f64p]
        L.oracle_prefill_attention_nvfp4.argtypes = [f32p, u8p, u8p, u8p, u8p, ctypes.c_float,
                                                     ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, i32p, ctypes.c_double, f64p]
        L.oracle_mxfp4_bits_per_element.argtypes = []
        L.oracle_mxfp4_bits_per_element.restype = ctypes.c_double
        L.oracle_kv_bytes.restype = ctypes.c_double
        L.oracle_nvfp4_bits_per_element.argtypes = []
        L.oracle_nvfp4_bits_per_element.restype = ctypes.c_double
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_get_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---- formats ----------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(code)


def e4m3_value(byte: int) -> float:
    return lib().oracle_e4m3_value(byte)


def e2m1_encode(v) -> np.ndarray:
    v = _f32(v).ravel()
    out = np.empty(v.size, np.uint8)
    lib().oracle_e2m1_encode_array(_p(v, ctypes.c_float), v.size, _p(out, ctypes.c_uint8))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = _f32(v).ravel()
    out = np.empty(v.size, np.uint8)
    lib().oracle_e4m3_encode_array(_p(v, ctypes.c_float), v.size, _p(out, ctypes.c_uint8))
    return out


# ---- calibration ------------------------------------------------------------
def tensor_scale(x):
    """Return (status, s_tensor) for the whole array x (fp32 values)."""
    x = _f32(x).ravel()
    s = np.zeros(1, np.float32)
    st = lib().oracle_tensor_scale(_p(x, ctypes.c_float), x.size, _p(s, ctypes.c_float))
    return int(st), np.float32(s[0])


# ---- quantize ---------------------------------------------------------------
def quantize_block(x16, s_tensor):
    x16 = _f32(x16).ravel()
    assert x16.size == 16
    packed = np.zeros(8, np.uint8)
    sb = np.zeros(1, np.uint8)
    lib().oracle_quantize_block(_p(x16, ctypes.c_float), np.float32(s_tensor),
                                _p(packed, ctypes.c_uint8), _p(sb, ctypes.c_uint8))
    return packed, int(sb[0])


def new_planes(B, H_kv, S_max, D):
    codes = np.zeros((B, H_kv, S_max, D // 2), np.uint8)
    scales = np.zeros((B, H_kv, S_max, D // 16), np.uint8)
    return codes, scales


def quantize_append(x_new, start, s_tensor, codes, scales):
    """x_new fp32 [B][n_new][H_kv][D]; codes/scales are updated in place."""
    x_new = _f32(x_new)
    B, n_new, H_kv, D = x_new.shape
    S_max = codes.shape[2]
    start = np.ascontiguousarray(start, np.int32)
    assert codes.flags.c_contiguous and scales.flags.c_contiguous
    return int(lib().oracle_quantize_append(
        _p(x_new, ctypes.c_float), B, n_new, H_kv, D, _p(start, ctypes.c_int32),
        np.float32(s_tensor), _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), S_max))


# ---- dequant ----------------------------------------------------------------
def dequant_fp8(code: int, scale_byte: int, s_tensor) -> int:
    return int(lib().oracle_dequant_fp8(code, scale_byte, np.float32(s_tensor)))


def dequant_planes(codes, scales, s_tensor, seq_lens):
    B, H_kv, S_max, Dh = codes.shape
    D = 2 * Dh
    seq_lens = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, H_kv, S_max, D), np.uint8)
    lib().oracle_dequant_planes(_p(np.ascontiguousarray(codes), ctypes.c_uint8),
                                _p(np.ascontiguousarray(scales), ctypes.c_uint8),
                                B, H_kv, S_max, D, np.float32(s_tensor),
                                _p(seq_lens, ctypes.c_int32), _p(out, ctypes.c_uint8))
    return out


def nvfp4_reconstruct_planes(codes, scales, s_tensor, seq_lens):
    """fp64 x^ = value(code) * value(sb) * s_tensor, [B][H_kv][S_max][D] (unset slots 0)."""
    B, H_kv, S_max, Dh = codes.shape
    D = 2 * Dh
    seq_lens = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, H_kv, S_max, D), np.float64)
    lib().oracle_nvfp4_reconstruct_planes(_p(np.ascontiguousarray(codes), ctypes.c_uint8),
                                          _p(np.ascontiguousarray(scales), ctypes.c_uint8),
                                          B, H_kv, S_max, D, np.float32(s_tensor),
                                          _p(seq_lens, ctypes.c_int32), _p(out, ctypes.c_double))
    return out


# ---- MXFP4 ("MXFP4との比較": 32-element blocks, E8M0 scales) -------------------
def e8m0_value(byte: int) -> float:
    return lib().oracle_e8m0_value(byte)


def mxfp4_quantize_block(x32):
    """Return (status, packed 16 bytes, E8M0 scale byte) for 32 fp32 values."""
    x32 = _f32(x32).ravel()
    assert x32.size == 32
    packed = np.zeros(16, np.uint8)
    sb = np.zeros(1, np.uint8)
    st = lib().oracle_mxfp4_quantize_block(_p(x32, ctypes.c_float), _p(packed, ctypes.c_uint8),
                                           _p(sb, ctypes.c_uint8))
    return int(st), packed, int(sb[0])


def new_mxfp4_planes(B, H_kv, S_max, D):
    codes = np.zeros((B, H_kv, S_max, D // 2), np.uint8)
    scales = np.zeros((B, H_kv, S_max, D // 32), np.uint8)
    return codes, scales


def mxfp4_quantize_append(x_new, start, codes, scales):
    """x_new fp32 [B][n_new][H_kv][D]; codes/scales are updated in place."""
    x_new = _f32(x_new)
    B, n_new, H_kv, D = x_new.shape
    S_max = codes.shape[2]
    start = np.ascontiguousarray(start, np.int32)
    assert codes.flags.c_contiguous and scales.flags.c_contiguous
    return int(lib().oracle_mxfp4_quantize_append(
        _p(x_new, ctypes.c_float), B, n_new, H_kv, D, _p(start, ctypes.c_int32),
        _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), S_max))


def mxfp4_reconstruct_planes(codes, scales, seq_lens):
    """fp64 x^ = value(code) * 2^(e8m0 - 127), [B][H_kv][S_max][D] (unset slots 0)."""
    B, H_kv, S_max, Dh = codes.shape
    D = 2 * Dh
    seq_lens = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, H_kv, S_max, D), np.float64)
    lib().oracle_mxfp4_reconstruct_planes(_p(np.ascontiguousarray(codes), ctypes.c_uint8),
                                          _p(np.ascontiguousarray(scales), ctypes.c_uint8),
                                          B, H_kv, S_max, D, _p(seq_lens, ctypes.c_int32),
                                          _p(out, ctypes.c_double))
    return out


def mxfp4_bits_per_element() -> float:
    return lib().oracle_mxfp4_bits_per_element()


# ---- attention --------------------------------------------------------------
def decode_attention_fp8(q, k8, v8, seq_lens, softmax_scale=0.0):
    """q fp32 [B][H_q][D]; k8/v8 E4M3 bytes [B][H_kv][S_max][D] -> fp64 [B][H_q][D]."""
    q = _f32(q)
    B, H_q, D = q.shape
    _, H_kv, S_max, _ = k8.shape
    seq_lens = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, H_q, D), np.float64)
    lib().oracle_decode_attention_fp8(_p(q, ctypes.c_float),
                                      _p(np.ascontiguousarray(k8), ctypes.c_uint8),
                                      _p(np.ascontiguousarray(v8), ctypes.c_uint8),
                                      B, H_q, H_kv, S_max, D, _p(seq_lens, ctypes.c_int32),
                                      float(softmax_scale), _p(out, ctypes.c_double))
    return out


def decode_attention_nvfp4(q, k_codes, k_scales, v_codes, v_scales, s_tensor_k, s_tensor_v,
                           seq_lens, softmax_scale=0.0):
    q = _f32(q)
    B, H_q, D = q.shape
    _, H_kv, S_max, _ = k_codes.shape
    seq_lens = np.ascontiguousarray(seq_lens, np.int32)
    out = np.zeros((B, H_q, D), np.float64)
    c = np.ascontiguousarray
    lib().oracle_decode_attention_nvfp4(
        _p(q, ctypes.c_float), _p(c(k_codes), ctypes.c_uint8), _p(c(k_scales), ctypes.c_uint8),
        _p(c(v_codes), ctypes.c_uint8), _p(c(v_scales), ctypes.c_uint8),
        np.float32(s_tensor_k), np.float32(s_tensor_v), B, H_q, H_kv, S_max, D,
        _p(seq_lens, ctypes.c_int32), float(softmax_scale), _p(out, ctypes.c_double))
    return out


def prefill_attention_nvfp4(q, k_codes, k_scales, v_codes, v_scales, s_tensor_k, s_tensor_v,
                            start, softmax_scale=0.0):
    """q fp32 [B][C][H_q][D] at positions start[b] + i -> fp64 [B][C][H_q][D] (causal)."""
    q = _f32(q)
    B, C, H_q, D = q.shape
    _, H_kv, S_max, _ = k_codes.shape
    start = np.ascontiguousarray(start, np.int32)
    assert np.all(start >= 0) and np.all(start + C <= S_max)
    out = np.zeros((B, C, H_q, D), np.float64)
    c = np.ascontiguousarray
    lib().oracle_prefill_attention_nvfp4(
        _p(q, ctypes.c_float), _p(c(k_codes), ctypes.c_uint8), _p(c(k_scales), ctypes.c_uint8),
        _p(c(v_codes), ctypes.c_uint8), _p(c(v_scales), ctypes.c_uint8),
        np.float32(s_tensor_k), np.float32(s_tensor_v), B, C, H_q, H_kv, S_max, D,
        _p(start, ctypes.c_int32), float(softmax_scale), _p(out, ctypes.c_double))
    return out


# ---- memory model -----------------------------------------------------------
def nvfp4_bits_per_element() -> float:
    return lib().oracle_nvfp4_bits_per_element()


def kv_bytes(layers, n_h, d_h, s, b, bits_per_element) -> float:
    return lib().oracle_kv_bytes(layers, n_h, d_h, s, b, float(bits_per_element))
