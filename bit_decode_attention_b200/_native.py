"""ctypes loader for libnvfp4kv.so (the C ABI in include/nvfp4kv.h).

The shared library is built in-tree by ``bit_decode_attention_b200.build``.
There is no fallback: if the library is missing or fails to load, every call
raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4kv.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_UNSUPPORTED = 2
NVFP4_ERR_CAPACITY = 3
NVFP4_ERR_NONFINITE = 4
NVFP4_ERR_CUDA = 5
NVFP4_ERR_TIMEOUT = 6
NVFP4_ERR_WORKSPACE = 7

NVFP4_IN_BF16 = 0
NVFP4_IN_F32 = 1

# every symbol the header declares
EXPORTS = (
    "nvfp4_status_string",
    "nvfp4_version",
    "nvfp4_cache_bytes",
    "nvfp4_calib_tensor_scale",
    "nvfp4_kv_quantize_append",
    "nvfp4_kv_quantize_append_kv",
    "nvfp4_kv_dequant_fp8",
    "nvfp4_decode_attention_workspace",
    "nvfp4_decode_attention",
    "nvfp4_decode_attention_noalloc",
    "mxfp4_cache_bytes",
    "mxfp4_kv_quantize_append",
    "nvfp4_kv_quantize_append_paged",
    "nvfp4_decode_attention_paged",
    "nvfp4_decode_attention_append",
    "nvfp4_set_wait_limit",
    "nvfp4_prefill_attention",
)


class KVPlaneStruct(ctypes.Structure):
    """nvfp4_kv_plane: host struct pointing at device code and scale arrays."""
    _fields_ = [
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("B", ctypes.c_int32),
        ("H_kv", ctypes.c_int32),
        ("S_max", ctypes.c_int32),
        ("D", ctypes.c_int32),
    ]


class PagedPlaneStruct(ctypes.Structure):
    """nvfp4_kv_paged_plane: host struct pointing at a device page pool and block table."""
    _fields_ = [
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("num_pages", ctypes.c_int32),
        ("H_kv", ctypes.c_int32),
        ("page_tokens", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("B", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
    ]


class NativeError(RuntimeError):
    def __init__(self, func, status, text):
        super().__init__("%s failed: %s (status %d)" % (func, text, status))
        self.status = status


_lib = None


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libnvfp4kv.so is not built (expected at %s); run "
            "`python -m bit_decode_attention_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    plane_p = ctypes.POINTER(KVPlaneStruct)
    L.nvfp4_status_string.argtypes = [i32]
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_version.argtypes = []
    L.nvfp4_version.restype = ctypes.c_char_p
    L.nvfp4_cache_bytes.argtypes = [i32, i32, i32, i32]
    L.nvfp4_cache_bytes.restype = sz
    L.nvfp4_calib_tensor_scale.argtypes = [vp, i32, i64, vp, vp, vp]
    L.nvfp4_calib_tensor_scale.restype = i32
    L.nvfp4_kv_quantize_append.argtypes = [vp, i32, i32, vp, vp, vp, plane_p, vp, vp]
    L.nvfp4_kv_quantize_append.restype = i32
    L.nvfp4_kv_quantize_append_kv.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp, plane_p, plane_p, vp, vp]
    L.nvfp4_kv_quantize_append_kv.restype = i32
    L.nvfp4_kv_dequant_fp8.argtypes = [plane_p, vp, vp, vp, vp, vp]
    L.nvfp4_kv_dequant_fp8.restype = i32
    L.nvfp4_decode_attention_workspace.argtypes = [i32, i32, i32, i32]
    L.nvfp4_decode_attention_workspace.restype = sz
    L.nvfp4_decode_attention.argtypes = [vp, i32, i32, plane_p, plane_p, vp, vp, vp, f32, vp, vp,
                                         sz, vp, vp]
    L.nvfp4_decode_attention.restype = i32
    L.nvfp4_decode_attention_noalloc.argtypes = [vp, i32, i32, plane_p, plane_p, vp, vp, vp, f32, vp,
                                                 vp, vp]
    L.nvfp4_decode_attention_noalloc.restype = i32
    L.mxfp4_cache_bytes.argtypes = [i32, i32, i32, i32]
    L.mxfp4_cache_bytes.restype = sz
    L.mxfp4_kv_quantize_append.argtypes = [vp, i32, i32, vp, vp, plane_p, vp, vp]
    L.mxfp4_kv_quantize_append.restype = i32
    paged_p = ctypes.POINTER(PagedPlaneStruct)
    L.nvfp4_kv_quantize_append_paged.argtypes = [vp, i32, i32, vp, vp, vp, paged_p, vp, vp]
    L.nvfp4_kv_quantize_append_paged.restype = i32
    L.nvfp4_decode_attention_paged.argtypes = [vp, i32, i32, paged_p, paged_p, vp, vp, vp, f32, vp, vp,
                                               sz, vp, vp]
    L.nvfp4_decode_attention_paged.restype = i32
    L.nvfp4_decode_attention_append.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, plane_p, plane_p, vp, vp,
                                                f32, vp, vp, sz, vp, vp]
    L.nvfp4_decode_attention_append.restype = i32
    L.nvfp4_set_wait_limit.argtypes = [i64]
    L.nvfp4_set_wait_limit.restype = None
    L.nvfp4_prefill_attention.argtypes = [vp, i32, i32, i32, plane_p, plane_p, vp, vp, vp, f32, vp, vp, vp]
    L.nvfp4_prefill_attention.restype = i32
    _lib = L
    return L


def check(func_name, status):
    if status != NVFP4_OK:
        text = lib().nvfp4_status_string(status).decode()
        raise NativeError(func_name, status, text)
