"""Seeded synthetic inputs for the PM-KVQ hot path.

This module only draws numbers: Gaussian keys, values and queries shaped like
the long-CoT models the PM-KVQ note evaluates (DeepSeek-R1-Distill Qwen 7B and
32B, Llama 70B heads), with a few fixed outlier channels in the Keys and the
rotate-half RoPE those models apply.  It holds none of the method's
arithmetic (no migration factor, quantizer, shift or attention), so that the
CPU oracle and the CUDA path can both consume it without sharing any of the
method's code.

Recipe (one KV-cache block = one transformer layer):
  * K ~ N(0, 1) per channel; a fixed set of outlier channels (chosen by the
    seed, the same for every head and token) is multiplied by 20 before RoPE.
    The PM-KVQ note (current pain points; key design 3) places the outliers
    in fixed Key channels.
  * V ~ N(0, 1), no outliers, no RoPE.
  * Q ~ N(0, 1), RoPE at the decode position.
  * RoPE: rotate-half pairs (i, i + d/2), angle pos * theta^(-2i/d),
    theta = 1e4.  With d = 128 the slowest pair has a period of
    2 pi 10^(4 * 126/128) = 54,410 tokens, the figure the note quotes for
    DeepSeek-R1-Distill-Qwen-7B (current pain points).
Every draw comes from its own torch.Generator seeded from (seed, stream tag,
layer, position), so a chunk can be regenerated on its own, on the CPU or on
a GPU (the two devices give different numbers; tests that compare against
the oracle draw on the CPU).
"""
from __future__ import annotations

import math

import torch

HEAD_DIM = 128
ROPE_THETA = 1.0e4
OUTLIER_GAIN = 20.0


def rope_inv_freq(d: int = HEAD_DIM, theta: float = ROPE_THETA) -> torch.Tensor:
    """theta^(-2i/d) for the d/2 rotation pairs (fp64)."""
    i = torch.arange(d // 2, dtype=torch.float64)
    return theta ** (-2.0 * i / d)


def lowest_period(d: int = HEAD_DIM, theta: float = ROPE_THETA) -> float:
    """Period, in tokens, of the slowest RoPE pair: 2 pi / min_i theta^(-2i/d)."""
    return 2.0 * math.pi / float(rope_inv_freq(d, theta).min())


def apply_rope(x: torch.Tensor, positions: torch.Tensor) -> torch.Tensor:
    """Rotate-half RoPE.  x: [..., n, heads, d] (fp32), positions: [n] ints."""
    d = x.shape[-1]
    inv = rope_inv_freq(d).to(x.device)
    ang = positions.to(torch.float64)[:, None] * inv[None, :]  # [n, d/2]
    cos = torch.cos(ang).to(torch.float32)[:, None, :]  # [n, 1, d/2]
    sin = torch.sin(ang).to(torch.float32)[:, None, :]
    x1, x2 = x[..., : d // 2], x[..., d // 2 :]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def _gen(seed: int, tag: int, layer: int, pos: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tag * 7_919 + layer * 104_729 + pos * 13) % (2**63 - 1))
    return g


def outlier_channels(seed: int, layer: int, count: int, d: int = HEAD_DIM) -> torch.Tensor:
    """`count` distinct channels (sorted) chosen by (seed, layer)."""
    g = _gen(seed, 1, layer, 0, "cpu")
    return torch.randperm(d, generator=g)[:count].sort().values


def keys_values(seed: int, layer: int, batch: int, n: int, kv_heads: int, pos0: int,
                n_outliers: int, dtype=torch.bfloat16, device="cpu"):
    """K, V: [batch][n][kv_heads][128] for positions pos0 .. pos0+n-1."""
    g = _gen(seed, 2, layer, pos0, device)
    k = torch.randn((batch, n, kv_heads, HEAD_DIM), generator=g, device=device)
    v = torch.randn((batch, n, kv_heads, HEAD_DIM), generator=g, device=device)
    if n_outliers:
        ch = outlier_channels(seed, layer, n_outliers).to(device)
        k[..., ch] *= OUTLIER_GAIN
    pos = torch.arange(pos0, pos0 + n, device=device)
    k = apply_rope(k, pos)
    return k.to(dtype), v.to(dtype)


def queries(seed: int, layer: int, step: int, batch: int, q_heads: int, pos: int,
            dtype=torch.bfloat16, device="cpu"):
    """Q: [batch][q_heads][128] at decode position `pos`."""
    g = _gen(seed, 3, layer, step, device)
    q = torch.randn((batch, 1, q_heads, HEAD_DIM), generator=g, device=device)
    q = apply_rope(q, torch.tensor([pos], device=device))
    return q[:, 0].to(dtype)


def outliers_for(kv_heads: int, pct: float = 0.01, minimum: int = 1) -> int:
    """Outlier channels per head from a fraction of a layer's kv_heads*128 channels."""
    return max(minimum, round(pct * kv_heads * HEAD_DIM))
