"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws seeded random
tensors and builds the per-head slope vector (an input array of the method),
so that the CUDA path and the CPU oracle are fed identical values.

Recipe: a CPU ``torch.Generator`` seeded with ``seed + t`` (t = 0 for Q,
1 for K, 2 for V, 3 for dO), fp32 N(0, 1) draws, multiplied by ``scale``,
then cast to the I/O dtype. The oracle consumes the cast values (upcast).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


def normal(shape, seed: int, scale: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def qkv(B: int, N: int, H: int, Hkv: int, d: int, seed: int = 0, scale: float = 1.0,
        dtype=torch.bfloat16, with_dout: bool = False):
    """Q [B,N,H,d], K/V [B,N,Hkv,d] (and dO [B,N,H,d] ~ N(0,1) if asked)."""
    q = normal((B, N, H, d), seed + 0, scale, dtype)
    k = normal((B, N, Hkv, d), seed + 1, scale, dtype)
    v = normal((B, N, Hkv, d), seed + 2, scale, dtype)
    if with_dout:
        do = normal((B, N, H, d), seed + 3, 1.0, dtype)
        return q, k, v, do
    return q, k, v


def balanced_alibi_slopes(H: int) -> torch.Tensor:
    """Balanced ALiBi slopes ("SWAT" page, section "Balanced ALiBi"): the first
    H/2 heads are forward-looking with s = -2^-k, the other H/2 backward-looking
    with s = +2^-k, k = 1 .. H/2 (geometric spacing, one temporal scale per head).
    """
    if H % 2 != 0:
        raise ValueError("balanced ALiBi needs an even number of heads")
    half = H // 2
    mags = [2.0 ** -(k + 1) for k in range(half)]
    return torch.tensor([-m for m in mags] + mags, dtype=torch.float32)


def geometric_alibi_slopes(H: int) -> torch.Tensor:
    """The tiny-config rule "slopes 2^(-8h/H)", h = 1..H (1-based), with the
    first half of the heads forward-looking (negative) and the second half
    backward-looking (positive)."""
    if H % 2 != 0:
        raise ValueError("balanced ALiBi needs an even number of heads")
    mags = [2.0 ** (-8.0 * h / H) for h in range(1, H + 1)]
    return torch.tensor([-m if h < H // 2 else m for h, m in enumerate(mags)],
                        dtype=torch.float32)


def forward_only_slopes(H: int) -> torch.Tensor:
    """SWAT(-): every head forward-looking, s = -2^-k over the heads of each half."""
    half = max(H // 2, 1)
    mags = [2.0 ** -((h % half) + 1) for h in range(H)]
    return torch.tensor([-m for m in mags], dtype=torch.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    window: int
    n_sink: int
    mode: int          # 0 sigmoid, 1 softmax
    rope_base: float
    scale: float       # multiplier on N(0,1) inputs
    slopes: str        # "balanced", "geometric", "none"
    dtype: str         # "bf16" or "f32"

    def slope_tensor(self):
        if self.slopes == "balanced":
            return balanced_alibi_slopes(self.H)
        if self.slopes == "geometric":
            return geometric_alibi_slopes(self.H)
        if self.slopes == "forward":
            return forward_only_slopes(self.H)
        return None

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


# The pages' workload shapes (340M SWAT layer, long sequence, SWA(64,4), ring decode).
TINY_F32 = Workload("tiny_swat_fwd_f32", 1, 2, 2, 128, 64, 16, 0, 0, 1e4, 1.0, "geometric", "f32")
SWAT_340M = Workload("swat_340m_layer", 8, 16, 16, 4096, 64, 512, 0, 0, 1e4, 1.0 / math.sqrt(64),
                     "balanced", "bf16")
SWAT_LONG = Workload("swat_long_64k", 1, 32, 32, 65536, 128, 4096, 0, 0, 1e4, 1.0, "balanced", "bf16")
SWA_SINK = Workload("swa_64_4_gqa", 2, 32, 8, 32768, 128, 64, 4, 1, 5e5, 1.0, "none", "bf16")


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    Hkv: int
    d: int
    window: int
    n_sink: int
    mode: int
    rope_base: float
    slopes: str
    start_pos: int

    def slope_tensor(self):
        if self.slopes == "balanced":
            return balanced_alibi_slopes(self.H)
        return None


DECODE_SIGMOID = DecodeWorkload("ring_decode_sigmoid", 64, 32, 8, 128, 4096, 0, 0, 1e4, "balanced", 32768)
DECODE_SOFTMAX = DecodeWorkload("ring_decode_softmax_sink4", 64, 32, 8, 128, 4096, 4, 1, 5e5, "none", 32768)


def decode_step_inputs(B: int, H: int, Hkv: int, d: int, step: int, dtype=torch.bfloat16):
    """Per-step q [B,H,d], k_new / v_new [B,Hkv,d] from seed 1000 + step."""
    base = 1000 + step
    g = torch.Generator(device="cpu")
    g.manual_seed(base)
    q = torch.randn(B, H, d, generator=g, dtype=torch.float32)
    kn = torch.randn(B, Hkv, d, generator=g, dtype=torch.float32)
    vn = torch.randn(B, Hkv, d, generator=g, dtype=torch.float32)
    return q.to(dtype), kn.to(dtype), vn.to(dtype)
