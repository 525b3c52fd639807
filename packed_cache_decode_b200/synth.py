"""Seeded synthetic attention inputs shaped like the layers the method is evaluated on.

This module only draws numbers. It holds none of the method's arithmetic (no energy
score, no rate allocation, no rotation, no quantisation, no attention); it feeds both
the CUDA path and the CPU oracle, which therefore see identical inputs.

Recipe (the abstract of "Block-GTQ: RoPE-Block Rate Allocation for KV-Cache
Quantization" evaluates on Llama-3.1-8B, Qwen2.5-3B and 70B-class models; none of
their weights exist here, so these draws stand in for their activations):

* per head, per RoPE block j (coordinates j and j+64), one scale drawn log-uniform in
  [0.1, 10] multiplies both coordinates; q heads and k heads draw their scales
  independently, v only when ``scale_v`` is set (the tiny single-head case);
* per KV head, 4 distinct outlier channels (uniform over the 128 coordinates) are
  multiplied by 8 in k and in every query head that maps to that KV head;
* the scaled vectors are N(0,1) draws; q and k then get rotate-half RoPE at their
  positions with base ``theta`` (values are fp32; callers cast to bf16 where the
  configuration says so).

Every (batch row, head) slice has its own generator seed, so any slice can be redrawn
alone without drawing the whole tensor.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

HEAD_DIM = 128
N_BLOCKS = HEAD_DIM // 2

_TAG_MODEL, _TAG_Q, _TAG_K, _TAG_V = 11, 23, 37, 41


def _slice_seed(*parts: int) -> int:
    s = 0x5EED
    for p in parts:
        s = (s * 1000003 + int(p) + 0x9E37) % (1 << 62)
    return s


def _gen(*parts: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_slice_seed(*parts))
    return g


@dataclass
class LayerModel:
    """Fixed per-layer statistics of the synthetic activations."""

    h_q: int
    h_kv: int
    seed: int
    q_scale: torch.Tensor            # [h_q, 64] fp32
    k_scale: torch.Tensor            # [h_kv, 64] fp32
    v_scale: torch.Tensor | None     # [h_kv, 64] fp32 or None
    outliers: torch.Tensor           # [h_kv, n_outliers] int64
    outlier_gain: float = 8.0

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv


def make_layer_model(h_q: int, h_kv: int, seed: int, scale_v: bool = False,
                     n_outliers: int = 4, outlier_gain: float = 8.0,
                     scale_lo: float = 0.1, scale_hi: float = 10.0) -> LayerModel:
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    g = _gen(seed, _TAG_MODEL)
    lo, hi = math.log(scale_lo), math.log(scale_hi)

    def scales(n):
        return torch.exp(lo + (hi - lo) * torch.rand(n, N_BLOCKS, generator=g, dtype=torch.float64)).float()

    q_scale = scales(h_q)
    k_scale = scales(h_kv)
    v_scale = scales(h_kv) if scale_v else None
    outliers = torch.stack([torch.randperm(HEAD_DIM, generator=g)[:n_outliers] for _ in range(h_kv)])
    return LayerModel(h_q, h_kv, seed, q_scale, k_scale, v_scale, outliers, outlier_gain)


def rope_rotate_half(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half RoPE over the last dimension (pairs j, j+64), computed in fp64."""
    half = x.shape[-1] // 2
    inv = theta ** (-torch.arange(half, dtype=torch.float64) * 2.0 / x.shape[-1])
    ang = pos.to(torch.float64)[:, None] * inv[None, :]          # [n, 64]
    shape = [1] * (x.dim() - 2)
    c = torch.cos(ang).view(*shape, *ang.shape) if shape else torch.cos(ang)
    s = torch.sin(ang).view(*shape, *ang.shape) if shape else torch.sin(ang)
    xd = x.to(torch.float64)
    a, b = xd[..., :half], xd[..., half:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1).to(x.dtype)


def _blockscale(scale_row: torch.Tensor) -> torch.Tensor:
    return torch.cat([scale_row, scale_row])  # coordinate j and j+64 share block j's scale


def key_slice(m: LayerModel, b: int, h: int, n: int, start: int, seed: int, theta: float) -> torch.Tensor:
    """Post-RoPE keys of KV head h of batch row b at positions start..start+n-1, [n, 128] fp32."""
    x = torch.randn(n, HEAD_DIM, generator=_gen(seed, _TAG_K, b, h), dtype=torch.float32)
    x *= _blockscale(m.k_scale[h])
    x[:, m.outliers[h]] *= m.outlier_gain
    return rope_rotate_half(x, torch.arange(start, start + n), theta)


def value_slice(m: LayerModel, b: int, h: int, n: int, seed: int) -> torch.Tensor:
    x = torch.randn(n, HEAD_DIM, generator=_gen(seed, _TAG_V, b, h), dtype=torch.float32)
    if m.v_scale is not None:
        x *= _blockscale(m.v_scale[h])
        x[:, m.outliers[h]] *= m.outlier_gain
    return x


def query_slice(m: LayerModel, b: int, hq: int, n: int, start: int, seed: int, theta: float) -> torch.Tensor:
    x = torch.randn(n, HEAD_DIM, generator=_gen(seed, _TAG_Q, b, hq), dtype=torch.float32)
    x *= _blockscale(m.q_scale[hq])
    x[:, m.outliers[hq // m.group]] *= m.outlier_gain
    return rope_rotate_half(x, torch.arange(start, start + n), theta)


def make_cache_inputs(m: LayerModel, batch: int, length: int, seed: int, theta: float,
                      dtype: torch.dtype = torch.float32):
    """q [B, h_q, 128] at position length-1 and k, v [B, length, h_kv, 128]."""
    k = torch.empty(batch, length, m.h_kv, HEAD_DIM, dtype=dtype)
    v = torch.empty_like(k)
    q = torch.empty(batch, m.h_q, HEAD_DIM, dtype=dtype)
    for b in range(batch):
        for h in range(m.h_kv):
            k[b, :, h] = key_slice(m, b, h, length, 0, seed, theta).to(dtype)
            v[b, :, h] = value_slice(m, b, h, length, seed).to(dtype)
        for hq in range(m.h_q):
            q[b, hq] = query_slice(m, b, hq, 1, length - 1, seed, theta)[0].to(dtype)
    return q, k, v


def make_calibration(m: LayerModel, n: int, seed: int, theta: float):
    """n calibration queries [n, h_q, 128] and keys [n, h_kv, 128] at positions 0..n-1."""
    q = torch.stack([query_slice(m, 0, hq, n, 0, seed, theta) for hq in range(m.h_q)], dim=1)
    k = torch.stack([key_slice(m, 0, h, n, 0, seed, theta) for h in range(m.h_kv)], dim=1)
    return q, k


@dataclass
class Workload:
    """One attention layer shape of the evaluation, with its coding rates."""

    name: str
    h_q: int
    h_kv: int
    batch: int
    length: int
    k_bits: int          # average logical key bits per coordinate
    v_bits: int
    theta: float
    dtype: torch.dtype
    seed: int
    scale_v: bool = False
    layers: int = 1      # model depth: one cache per layer when a step covers the model
    allowed: tuple = (1, 2, 3, 4)
    notes: str = field(default="")


WORKLOADS = {
    "tiny": Workload("tiny single-head 1x1 d128 L1024 fp32 K2V2", 1, 1, 1, 1024, 2, 2, 5e5,
                     torch.float32, 0, scale_v=True, layers=1),
    "llama8b": Workload("llama-3.1-8b-shaped 32q/8kv d128 B1 L32768 bf16 K2V2", 32, 8, 1, 32768, 2, 2,
                        5e5, torch.bfloat16, 1, layers=32),
    "qwen3b": Workload("qwen2.5-3b-shaped 16q/2kv d128 B1 L131072 bf16 K3V3", 16, 2, 1, 131072, 3, 3,
                       1e6, torch.bfloat16, 2, layers=36),
    "llama70b": Workload("llama-70b-shaped 64q/8kv d128 B4 L131072 bf16 K2V2", 64, 8, 4, 131072, 2, 2,
                         5e5, torch.bfloat16, 3, layers=80),
}


def sweep_workloads():
    """The 32q/8kv sweep: contexts x batch x rates."""
    out = []
    for length in (4096, 16384, 65536, 262144):
        for batch in (1, 8, 32):
            for kb, vb in ((2, 2), (3, 2), (3, 3), (4, 4)):
                out.append(Workload(f"sweep 32q/8kv L{length} B{batch} K{kb}V{vb}", 32, 8, batch, length,
                                    kb, vb, 5e5, torch.bfloat16, 4))
    return out


def bf16_round(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).to(torch.float32)


def to_numpy64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()
