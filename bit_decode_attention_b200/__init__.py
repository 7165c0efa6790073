"""bit_decode_attention_b200 -- NVFP4 KV cache with fused NVFP4 -> FP8 decode
attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of libnvfp4kv.so (include/nvfp4kv.h).
The functions below carry the C names and only marshal arguments: torch
tensors supply device memory and the current CUDA stream, every step of the
computation runs in the library's kernels.  There is no CPU path.

Formats and flow follow "NVIDIA解説: NVFP4 KV Cacheで長コンテキストLLM推論を最適化"
(sections "E2M1 + 2レベルスケーリング" and "量子化・逆量子化フロー").
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _native
from ._native import (NVFP4_ERR_CAPACITY, NVFP4_ERR_INVALID_ARG, NVFP4_ERR_NONFINITE,  # noqa: F401
                      NVFP4_ERR_TIMEOUT, NVFP4_ERR_UNSUPPORTED, NVFP4_ERR_WORKSPACE, NVFP4_OK,
                      NativeError)

__all__ = [
    "KVPlane", "nvfp4_cache_bytes", "nvfp4_calib_tensor_scale", "nvfp4_kv_quantize_append",
    "nvfp4_kv_quantize_append_kv",
    "nvfp4_kv_dequant_fp8", "nvfp4_decode_attention_workspace", "nvfp4_decode_attention",
    "nvfp4_version", "NativeError", "nvfp4_decode_attention_noalloc",
    "mxfp4_cache_bytes", "mxfp4_kv_quantize_append",
    "PagedKVPlane", "nvfp4_kv_quantize_append_paged", "nvfp4_decode_attention_paged",
    "nvfp4_prefill_attention", "nvfp4_decode_attention_append", "nvfp4_set_wait_limit",
]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _native.NVFP4_IN_BF16
    if t.dtype == torch.float32:
        return _native.NVFP4_IN_F32
    raise TypeError("inputs must be bfloat16 or float32, got %s" % t.dtype)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


@dataclasses.dataclass
class KVPlane:
    """One NVFP4 cache plane (K or V) in device memory.

    codes  uint8 [B][H_kv][S_max][D/2]  (element 2j low nibble of byte j)
    scales uint8 [B][H_kv][S_max][D/16] (one E4M3 byte per 16 elements)
    """
    codes: torch.Tensor
    scales: torch.Tensor

    @classmethod
    def allocate(cls, B: int, H_kv: int, S_max: int, D: int, device="cuda") -> "KVPlane":
        codes = torch.zeros(B, H_kv, S_max, D // 2, dtype=torch.uint8, device=device)
        scales = torch.zeros(B, H_kv, S_max, D // 16, dtype=torch.uint8, device=device)
        return cls(codes, scales)

    @classmethod
    def allocate_mxfp4(cls, B: int, H_kv: int, S_max: int, D: int, device="cuda") -> "KVPlane":
        """An MXFP4 plane: the same codes, scales uint8 [B][H_kv][S_max][D/32] (E8M0)."""
        codes = torch.zeros(B, H_kv, S_max, D // 2, dtype=torch.uint8, device=device)
        scales = torch.zeros(B, H_kv, S_max, D // 32, dtype=torch.uint8, device=device)
        return cls(codes, scales)

    @property
    def shape(self):
        B, H, S, Dh = self.codes.shape
        return B, H, S, 2 * Dh

    def struct(self) -> _native.KVPlaneStruct:
        B, H, S, D = self.shape
        return _native.KVPlaneStruct(self.codes.data_ptr(), self.scales.data_ptr(), B, H, S, D)


@dataclasses.dataclass
class PagedKVPlane:
    """One paged NVFP4 cache plane: a page pool and the block table.

    codes       uint8 [num_pages][H_kv][page_tokens][D/2]
    scales      uint8 [num_pages][H_kv][page_tokens][D/16]
    block_table int32 [B][max_pages]; token t of sequence b lives in page
                block_table[b][t // page_tokens], slot t % page_tokens
    K and V planes of one cache share the block table.
    """
    codes: torch.Tensor
    scales: torch.Tensor
    block_table: torch.Tensor

    @classmethod
    def allocate(cls, num_pages: int, H_kv: int, page_tokens: int, D: int, block_table: torch.Tensor,
                 device="cuda") -> "PagedKVPlane":
        codes = torch.zeros(num_pages, H_kv, page_tokens, D // 2, dtype=torch.uint8, device=device)
        scales = torch.zeros(num_pages, H_kv, page_tokens, D // 16, dtype=torch.uint8, device=device)
        return cls(codes, scales, block_table)

    def struct(self) -> _native.PagedPlaneStruct:
        P, H, T, Dh = self.codes.shape
        B, M = self.block_table.shape
        return _native.PagedPlaneStruct(self.codes.data_ptr(), self.scales.data_ptr(),
                                        self.block_table.data_ptr(), P, H, T, 2 * Dh, B, M)


def nvfp4_version() -> str:
    return _native.lib().nvfp4_version().decode()


def nvfp4_set_wait_limit(polls: int) -> None:
    """Testing hook: pipeline-wait give-up limit of the tensor-core attention
    kernel (sleeping polls; 0 = give up unless already complete; < 0 = default)."""
    _native.lib().nvfp4_set_wait_limit(int(polls))


def nvfp4_cache_bytes(B: int, H_kv: int, S_max: int, D: int) -> int:
    return int(_native.lib().nvfp4_cache_bytes(B, H_kv, S_max, D))


def nvfp4_calib_tensor_scale(x: torch.Tensor, s_tensor: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-tensor scale fl32(amax / 2688) as a 1-element device float tensor."""
    _need_cuda(x)
    if s_tensor is None:
        s_tensor = torch.empty(1, dtype=torch.float32, device=x.device)
    st = _native.lib().nvfp4_calib_tensor_scale(_ptr(x), _dtype_code(x), x.numel(), _ptr(s_tensor),
                                                _ptr(status), _stream(stream))
    _native.check("nvfp4_calib_tensor_scale", st)
    return s_tensor


def nvfp4_kv_quantize_append(x_new: torch.Tensor, start_pos: torch.Tensor, s_tensor: torch.Tensor,
                             plane: KVPlane, new_lens: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Quantize x_new [B][n_new][H_kv][D] and write it at slots start_pos[b]... of `plane`."""
    _need_cuda(x_new, start_pos, s_tensor, new_lens, status)
    n_new = x_new.shape[1]
    pl = plane.struct()
    st = _native.lib().nvfp4_kv_quantize_append(_ptr(x_new), _dtype_code(x_new), n_new,
                                                _ptr(start_pos), _ptr(new_lens), _ptr(s_tensor),
                                                ctypes.byref(pl), _ptr(status), _stream(stream))
    _native.check("nvfp4_kv_quantize_append", st)


def nvfp4_kv_quantize_append_paged(x_new: torch.Tensor, start_pos: torch.Tensor, s_tensor: torch.Tensor,
                                   plane: PagedKVPlane, new_lens: Optional[torch.Tensor] = None,
                                   status: Optional[torch.Tensor] = None, stream=None) -> None:
    """nvfp4_kv_quantize_append into a paged plane (slots found through its block table)."""
    _need_cuda(x_new, start_pos, s_tensor, new_lens, status, plane.block_table)
    pl = plane.struct()
    st = _native.lib().nvfp4_kv_quantize_append_paged(_ptr(x_new), _dtype_code(x_new), x_new.shape[1],
                                                      _ptr(start_pos), _ptr(new_lens), _ptr(s_tensor),
                                                      ctypes.byref(pl), _ptr(status), _stream(stream))
    _native.check("nvfp4_kv_quantize_append_paged", st)


def nvfp4_kv_quantize_append_kv(x_k: torch.Tensor, x_v: torch.Tensor, start_pos: torch.Tensor,
                                s_tensor_k: torch.Tensor, s_tensor_v: torch.Tensor, k: KVPlane, v: KVPlane,
                                new_lens: Optional[torch.Tensor] = None,
                                status: Optional[torch.Tensor] = None, stream=None) -> None:
    """nvfp4_kv_quantize_append for K into `k` and V into `v` in one launch."""
    _need_cuda(x_k, x_v, start_pos, s_tensor_k, s_tensor_v, new_lens, status)
    if x_k.shape != x_v.shape or x_k.dtype != x_v.dtype:
        raise ValueError("x_k and x_v must have the same shape and dtype")
    n_new = x_k.shape[1]
    pk, pv = k.struct(), v.struct()
    st = _native.lib().nvfp4_kv_quantize_append_kv(_ptr(x_k), _ptr(x_v), _dtype_code(x_k), n_new,
                                                   _ptr(start_pos), _ptr(new_lens), _ptr(s_tensor_k),
                                                   _ptr(s_tensor_v), ctypes.byref(pk), ctypes.byref(pv),
                                                   _ptr(status), _stream(stream))
    _native.check("nvfp4_kv_quantize_append_kv", st)


def mxfp4_cache_bytes(B: int, H_kv: int, S_max: int, D: int) -> int:
    return int(_native.lib().mxfp4_cache_bytes(B, H_kv, S_max, D))


def mxfp4_kv_quantize_append(x_new: torch.Tensor, start_pos: torch.Tensor, plane: KVPlane,
                             new_lens: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Quantize x_new [B][n_new][H_kv][D] to MXFP4 (32-element blocks, E8M0
    scales) and write it at slots start_pos[b]... of an MXFP4 `plane`."""
    _need_cuda(x_new, start_pos, new_lens, status)
    B, H, S, D = plane.shape
    if plane.scales.shape[-1] != D // 32:
        raise ValueError("an MXFP4 plane holds D/32 scale bytes per token (KVPlane.allocate_mxfp4)")
    pl = plane.struct()
    st = _native.lib().mxfp4_kv_quantize_append(_ptr(x_new), _dtype_code(x_new), x_new.shape[1],
                                                _ptr(start_pos), _ptr(new_lens), ctypes.byref(pl),
                                                _ptr(status), _stream(stream))
    _native.check("mxfp4_kv_quantize_append", st)


def nvfp4_kv_dequant_fp8(plane: KVPlane, s_tensor: torch.Tensor, seq_lens: torch.Tensor,
                         out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """E4M3 bytes [B][H_kv][S_max][D] for the first seq_lens[b] slots."""
    _need_cuda(s_tensor, seq_lens, out, status)
    B, H, S, D = plane.shape
    if out is None:
        out = torch.zeros(B, H, S, D, dtype=torch.uint8, device=plane.codes.device)
    pl = plane.struct()
    st = _native.lib().nvfp4_kv_dequant_fp8(ctypes.byref(pl), _ptr(s_tensor), _ptr(seq_lens),
                                            _ptr(out), _ptr(status), _stream(stream))
    _native.check("nvfp4_kv_dequant_fp8", st)
    return out


def nvfp4_decode_attention_workspace(B: int, H_q: int, H_kv: int, D: int) -> int:
    return int(_native.lib().nvfp4_decode_attention_workspace(B, H_q, H_kv, D))


def new_workspace(B: int, H_q: int, H_kv: int, D: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace for nvfp4_decode_attention (reusable across calls)."""
    n = nvfp4_decode_attention_workspace(B, H_q, H_kv, D)
    if n == 0:
        raise ValueError("unsupported attention shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def nvfp4_prefill_attention(q: torch.Tensor, k: KVPlane, v: KVPlane, s_tensor_k: torch.Tensor,
                            s_tensor_v: torch.Tensor, start_pos: torch.Tensor, softmax_scale: float = 0.0,
                            out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """Causal attention of a prompt chunk over the NVFP4 cache (the chunk's K/V
    already appended at start_pos); q [B][C][H_q][128] -> fp32 [B][C][H_q][128]."""
    _need_cuda(q, s_tensor_k, s_tensor_v, start_pos, out, status)
    B, C, H_q, D = q.shape
    if out is None:
        out = torch.empty(B, C, H_q, D, dtype=torch.float32, device=q.device)
    kp, vp = k.struct(), v.struct()
    st = _native.lib().nvfp4_prefill_attention(
        _ptr(q), _dtype_code(q), C, H_q, ctypes.byref(kp), ctypes.byref(vp), _ptr(s_tensor_k),
        _ptr(s_tensor_v), _ptr(start_pos), ctypes.c_float(softmax_scale), _ptr(out), _ptr(status),
        _stream(stream))
    _native.check("nvfp4_prefill_attention", st)
    return out


def nvfp4_decode_attention(q: torch.Tensor, k: KVPlane, v: KVPlane, s_tensor_k: torch.Tensor,
                           s_tensor_v: torch.Tensor, seq_lens: torch.Tensor,
                           softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """softmax(q K^T * scale) V over the NVFP4 cache; q [B][H_q][D] -> fp32 [B][H_q][D]."""
    _need_cuda(q, s_tensor_k, s_tensor_v, seq_lens, out, workspace, status)
    B, H_q, D = q.shape
    Bk, H_kv, S, Dk = k.shape
    if out is None:
        out = torch.empty(B, H_q, D, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, H_q, H_kv, D, device=q.device)
    kp, vp = k.struct(), v.struct()
    st = _native.lib().nvfp4_decode_attention(
        _ptr(q), _dtype_code(q), H_q, ctypes.byref(kp), ctypes.byref(vp), _ptr(s_tensor_k),
        _ptr(s_tensor_v), _ptr(seq_lens), ctypes.c_float(softmax_scale), _ptr(out),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _native.check("nvfp4_decode_attention", st)
    return out


def nvfp4_decode_attention_append(q: torch.Tensor, x_k_new: torch.Tensor, x_v_new: torch.Tensor,
                                  start_pos: torch.Tensor, k: KVPlane, v: KVPlane, s_tensor_k: torch.Tensor,
                                  s_tensor_v: torch.Tensor, softmax_scale: float = 0.0,
                                  out: Optional[torch.Tensor] = None, new_lens: Optional[torch.Tensor] = None,
                                  workspace: Optional[torch.Tensor] = None,
                                  status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Append one token per sequence (x_k_new / x_v_new [B][1][H_kv][D]) at slot
    start_pos[b], then attend over start_pos[b] + 1 tokens; fp32 [B][H_q][D]."""
    _need_cuda(q, x_k_new, x_v_new, start_pos, s_tensor_k, s_tensor_v, out, new_lens, workspace, status)
    if x_k_new.shape != x_v_new.shape or x_k_new.dtype != x_v_new.dtype:
        raise ValueError("x_k_new and x_v_new must have the same shape and dtype")
    B, H_q, D = q.shape
    Bk, H_kv, S, Dk = k.shape
    if tuple(x_k_new.shape) != (Bk, 1, H_kv, Dk):
        raise ValueError("x_k_new must be [B][1][H_kv][D]")
    if out is None:
        out = torch.empty(B, H_q, D, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, H_q, H_kv, D, device=q.device)
    kp, vp = k.struct(), v.struct()
    st = _native.lib().nvfp4_decode_attention_append(
        _ptr(q), _dtype_code(q), H_q, _ptr(x_k_new), _ptr(x_v_new), _dtype_code(x_k_new), _ptr(start_pos),
        _ptr(new_lens), ctypes.byref(kp), ctypes.byref(vp), _ptr(s_tensor_k), _ptr(s_tensor_v),
        ctypes.c_float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream))
    _native.check("nvfp4_decode_attention_append", st)
    return out


def nvfp4_decode_attention_paged(q: torch.Tensor, k: PagedKVPlane, v: PagedKVPlane,
                                 s_tensor_k: torch.Tensor, s_tensor_v: torch.Tensor,
                                 seq_lens: torch.Tensor, softmax_scale: float = 0.0,
                                 out: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None,
                                 status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """nvfp4_decode_attention over paged K/V planes that share one block table."""
    _need_cuda(q, s_tensor_k, s_tensor_v, seq_lens, out, workspace, status, k.block_table)
    B, H_q, D = q.shape
    H_kv = k.codes.shape[1]
    if out is None:
        out = torch.empty(B, H_q, D, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, H_q, H_kv, D, device=q.device)
    kp, vp = k.struct(), v.struct()
    st = _native.lib().nvfp4_decode_attention_paged(
        _ptr(q), _dtype_code(q), H_q, ctypes.byref(kp), ctypes.byref(vp), _ptr(s_tensor_k),
        _ptr(s_tensor_v), _ptr(seq_lens), ctypes.c_float(softmax_scale), _ptr(out),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _native.check("nvfp4_decode_attention_paged", st)
    return out


def nvfp4_decode_attention_noalloc(q: torch.Tensor, k: KVPlane, v: KVPlane, s_tensor_k: torch.Tensor,
                                   s_tensor_v: torch.Tensor, seq_lens: torch.Tensor,
                                   softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                   status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """nvfp4_decode_attention without a workspace, for callers that may not
    allocate device memory: scratch is the library's built-in device buffer
    (shared by all calls on a device; calls must not overlap on the GPU)."""
    _need_cuda(q, s_tensor_k, s_tensor_v, seq_lens, out, status)
    B, H_q, D = q.shape
    if out is None:
        out = torch.empty(B, H_q, D, dtype=torch.float32, device=q.device)
    kp, vp = k.struct(), v.struct()
    st = _native.lib().nvfp4_decode_attention_noalloc(
        _ptr(q), _dtype_code(q), H_q, ctypes.byref(kp), ctypes.byref(vp), _ptr(s_tensor_k),
        _ptr(s_tensor_v), _ptr(seq_lens), ctypes.c_float(softmax_scale), _ptr(out), _ptr(status),
        _stream(stream))
    _native.check("nvfp4_decode_attention_noalloc", st)
    return out
