"""Seeded synthetic workloads shared by the tests, the bench and the oracle legs.

This module holds NO arithmetic of the method (no scaling, quantization or
attention): it only draws random numbers with the shapes and value
distributions of the workloads below, on a CPU ``torch.Generator`` so that the
CUDA path and the oracle receive bit-identical inputs.

Workloads (sizes and distributions of the NVFP4 KV-cache use cases: long
context, large batch, GQA decode, large-MoE-shaped attention):

  tiny       B1  Hq1  Hkv1 D64  L256      fp32 K/V ~ N(0,1), channels 7 and 40
                                          scaled x20; q ~ N(0,1) fp32
  gqa        B8  Hq32 Hkv8 D128 L4096     bf16 K/V ~ N(0,1) * LogNormal(0,1)
                                          per (kv head, channel); q ~ N(0,1)
  long64k    B1  Hq64 Hkv8 D128 L65536    as gqa, plus 0.1% of elements
                                          replaced by N(0, 30) outliers
  ragged     B128 Hq32 Hkv8 D128 L~U[1024,8192]  N(0,1) * LogNormal(0,0.5)
  moe128k    B1  Hq96 Hkv8 D128 L131072   N(0,1) * LogNormal(0,1); GQA group 12

Seeds are 1000 + the workload's index in the list above.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    D: int
    L: Optional[int]            # uniform length (None for ragged)
    L_range: Optional[tuple]    # inclusive (lo, hi) for ragged lengths
    dtype: str                  # "f32" or "bf16" for K/V/q inputs
    lognormal_sigma: float      # 0 for plain N(0,1)
    outlier_channels: tuple     # channels scaled by outlier_channel_gain
    outlier_channel_gain: float
    outlier_frac: float         # fraction of elements replaced by N(0, outlier_std)
    outlier_std: float
    chunk: Optional[int] = None  # prefill append chunk (tokens), None = one call

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = [
    Workload("tiny", 0, B=1, Hq=1, Hkv=1, D=64, L=256, L_range=None, dtype="f32",
             lognormal_sigma=0.0, outlier_channels=(7, 40), outlier_channel_gain=20.0,
             outlier_frac=0.0, outlier_std=0.0),
    Workload("gqa", 1, B=8, Hq=32, Hkv=8, D=128, L=4096, L_range=None, dtype="bf16",
             lognormal_sigma=1.0, outlier_channels=(), outlier_channel_gain=1.0,
             outlier_frac=0.0, outlier_std=0.0),
    Workload("long64k", 2, B=1, Hq=64, Hkv=8, D=128, L=65536, L_range=None, dtype="bf16",
             lognormal_sigma=1.0, outlier_channels=(), outlier_channel_gain=1.0,
             outlier_frac=0.001, outlier_std=30.0),
    Workload("ragged", 3, B=128, Hq=32, Hkv=8, D=128, L=None, L_range=(1024, 8192),
             dtype="bf16", lognormal_sigma=0.5, outlier_channels=(), outlier_channel_gain=1.0,
             outlier_frac=0.0, outlier_std=0.0),
    Workload("moe128k", 4, B=1, Hq=96, Hkv=8, D=128, L=131072, L_range=None, dtype="bf16",
             lognormal_sigma=1.0, outlier_channels=(), outlier_channel_gain=1.0,
             outlier_frac=0.0, outlier_std=0.0, chunk=2048),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def get(name: str) -> Workload:
    return BY_NAME[name]


def shrink(w: Workload, **kw) -> Workload:
    """Same distributions, other sizes (for oracle-sized parity cases)."""
    return dataclasses.replace(w, **kw)


def generator(w: Workload, stream: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed * 7919 + stream)
    return g


def seq_lens(w: Workload) -> List[int]:
    """Per-sequence lengths; ragged lengths are uniform integers in L_range."""
    if w.L is not None:
        return [w.L] * w.B
    lo, hi = w.L_range
    g = generator(w, stream=1)
    return torch.randint(lo, hi + 1, (w.B,), generator=g).tolist()


def channel_scales(w: Workload):
    """(scale_k, scale_v), each fp32 [Hkv][D]: LogNormal(0, sigma) per channel,
    drawn separately for K and V and shared over batch and tokens."""
    g = generator(w, stream=2)
    out = []
    for _ in range(2):
        if w.lognormal_sigma > 0:
            s = torch.exp(torch.randn(w.Hkv, w.D, generator=g) * w.lognormal_sigma)
        else:
            s = torch.ones(w.Hkv, w.D)
        for c in w.outlier_channels:
            s[:, c] *= w.outlier_channel_gain
        out.append(s)
    return out[0], out[1]


def _round_dtype(x: torch.Tensor, w: Workload) -> torch.Tensor:
    """Round to the workload's input dtype and return the exact fp32 widening."""
    return x.to(w.torch_dtype()).to(torch.float32)


def kv_tokens(w: Workload, n_tokens: int, which: str, stream: int = 0,
              batch: Optional[int] = None) -> torch.Tensor:
    """K or V inputs, fp32 values exactly representable in w.dtype,
    shape [B][n_tokens][Hkv][D] (token-major, as appended)."""
    assert which in ("k", "v")
    B = w.B if batch is None else batch
    sk, sv = channel_scales(w)
    scale = sk if which == "k" else sv
    g = generator(w, stream=10 + (0 if which == "k" else 1) + 2 * stream)
    x = torch.randn(B, n_tokens, w.Hkv, w.D, generator=g)
    x = x * scale.view(1, 1, w.Hkv, w.D)
    if w.outlier_frac > 0:
        mask = torch.rand(B, n_tokens, w.Hkv, w.D, generator=g) < w.outlier_frac
        vals = torch.randn(B, n_tokens, w.Hkv, w.D, generator=g) * w.outlier_std
        x = torch.where(mask, vals, x)
    return _round_dtype(x, w)


def queries(w: Workload, stream: int = 0, batch: Optional[int] = None) -> torch.Tensor:
    """Decode queries ~ N(0,1), fp32 values exactly representable in w.dtype,
    shape [B][Hq][D]."""
    B = w.B if batch is None else batch
    g = generator(w, stream=100 + stream)
    return _round_dtype(torch.randn(B, w.Hq, w.D, generator=g), w)


def prefill_queries(w: Workload, C: int, stream: int = 0) -> torch.Tensor:
    """Queries of a C-token prompt chunk ~ N(0,1), fp32 values exactly
    representable in w.dtype, shape [B][C][Hq][D]."""
    g = generator(w, stream=300 + stream)
    return _round_dtype(torch.randn(w.B, C, w.Hq, w.D, generator=g), w)


def capacity(max_len: int, extra: int = 0) -> int:
    """Cache capacity S_max for a workload: max_len + extra rounded up to 16."""
    n = max_len + extra
    return (n + 15) // 16 * 16


def random_planes(seed: int, B: int, H_kv: int, S_max: int, D: int, max_scale_byte: int = 0x7E):
    """Uniformly random NVFP4 planes (every code nibble, scale bytes 0..max),
    uint8 tensors [B][H_kv][S_max][D/2] and [B][H_kv][S_max][D/16]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    codes = torch.randint(0, 256, (B, H_kv, S_max, D // 2), generator=g, dtype=torch.int32)
    scales = torch.randint(0, max_scale_byte + 1, (B, H_kv, S_max, D // 16), generator=g,
                           dtype=torch.int32)
    return codes.to(torch.uint8), scales.to(torch.uint8)


def special_blocks(D: int = 128) -> torch.Tensor:
    """A handful of hand-picked token rows [n][D] that hit the corner cases of
    block quantization: all-zero and signed-zero blocks, one-hot blocks, exact
    grid midpoints, tiny values, and values far beyond the calibrated range."""
    rows = []
    z = torch.zeros(D)
    rows.append(z.clone())
    r = z.clone(); r[1::2] = -0.0; rows.append(r)
    r = z.clone(); r[0] = 1.0; r[17] = -3.0; rows.append(r)
    r = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * (D // 8)); rows.append(r)
    r = torch.tensor([-0.25, 0.5, -1.0, 1.5, -2.0, 3.0, -4.0, 6.0] * (D // 8)); rows.append(r)
    r = torch.full((D,), 1e-30); r[::3] = -2e-38; rows.append(r)
    r = torch.linspace(-50.0, 50.0, D); rows.append(r)
    r = torch.linspace(-1e4, 3e4, D); rows.append(r)
    # one float either side of every grid midpoint, in blocks whose amax is 6
    # (with s_tensor = 1 the block's divisor is exactly 1)
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    below = torch.nextafter(mids, torch.zeros(7))
    above = torch.nextafter(mids, torch.full((7,), 8.0))
    blk = torch.cat([below, above, torch.tensor([6.0, -6.0])])
    r = torch.cat([blk, -blk] * (D // 32)); rows.append(r)
    # small values of both signs that round to a signed zero or the first code
    r = torch.tensor([-1e-3, 1e-3, -0.2, 0.2, -0.26, 0.26, -0.0, 6.0] * (D // 8)); rows.append(r)
    return torch.stack(rows)


def nonfinite_blocks(D: int = 128) -> torch.Tensor:
    """Token rows [n][D] with a NaN or an infinity inside blocks of ordinary
    values (the quantizer's path for blocks it cannot divide by correction)."""
    r = torch.linspace(-3.0, 3.0, D)
    r[5] = float("nan")
    r[40] = float("inf")
    r[41] = -float("inf")
    r2 = torch.linspace(-1.0, 1.0, D)
    r2[16:32] = float("nan")
    return torch.stack([r, r2])
