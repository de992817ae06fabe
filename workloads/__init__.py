"""Seeded synthetic KV/Q workloads shaped like the pages' next-scale models.

This module only draws random numbers and arranges them into tensors. It holds
none of the quantizer's or the attention's arithmetic, so both the CUDA path and
the CPU oracle can be fed from it without sharing any method code.

Shapes follow the model families named in "VAR-Q results data (Tables 2-4)":
VAR-d16/d20/d30 (Table 2a, ImageNet 256x256, 10 scales, 680 tokens) and
Infinity-2B (Table 2b, 13 scales, 10521 tokens). The value distribution follows
the cache statistics described in "VAR-Q: Tuning-Free KV Cache Quantization ...",
Abstract paragraph 2: a few massive-value channels, magnitudes persistent within
a (block, channel) cell and shifting across cells, caused by projection bias and
RoPE-induced scattering. No trained weights or datasets are involved.

Layout of every generated tensor: [batch][heads][tokens][head_dim], contiguous,
tokens of block s occupying [prefix(s), prefix(s) + n_s).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    heads: int
    head_dim: int
    batch: int
    sides: Tuple[int, ...]          # scale side lengths r_s; block s has r_s**2 tokens
    kv_dtype: str                   # "f32" or "bf16"
    n_outlier: int                  # massive channels per head
    outlier_style: str              # "fixed30" (x30, per-block offset) or "massive" (x U(20,50) per cell + bias)
    rope_k: bool                    # pairwise rotation of K channels (RoPE scattering)
    bits: Tuple[int, ...]           # precisions exercised on this workload
    chunks: Tuple[int, ...] = ()    # explicit block sizes (next-frame video); empty: r_s**2 per scale

    @property
    def block_tokens(self) -> Tuple[int, ...]:
        return tuple(self.chunks) if self.chunks else tuple(r * r for r in self.sides)

    @property
    def num_blocks(self) -> int:
        return len(self.block_tokens)

    @property
    def tokens(self) -> int:
        return sum(self.block_tokens)

    def prefix(self, s: int) -> int:
        """Token offset of block s in the flattened sequence."""
        return sum(self.block_tokens[:s])

    def describe(self) -> str:
        return (f"{self.name}: L={self.layers} H={self.heads} D={self.head_dim} B={self.batch} "
                f"blocks={self.num_blocks} N={self.tokens} kv={self.kv_dtype} bits={self.bits}")


VAR_SIDES = (1, 2, 3, 4, 5, 6, 8, 10, 13, 16)
INFINITY_SIDES = (1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64)

# Next-frame video ("VAR-Q results data (Tables 2-4)", Table 4: Self-Forcing
# 1.3B, 5-second clips, batch 12; LongLive 1.3B, 30-second clips, batch 20).
# The pages give no schedule. Assumed here: a 1.3B video model of 30 layers,
# 12 heads x 128 (hidden 1536), latent frames of 30 x 52 = 1560 tokens,
# generated in chunks of 3 frames (4680 tokens) that attend block-causally to
# the cached chunks. Self-Forcing: 21 latent frames, 7 chunks, 32760 tokens
# (the BF16 KV of Table 4, 67.49 GiB, is 30 * 2 * N * 1536 * 2 B * 12 with
# N = 32760 to within 0.01 GiB). LongLive: a cache window of 12 frames, 4
# chunks, 18720 tokens (its BF16 KV, 64.28 GiB at batch 20, gives N = 18720).
VIDEO_CHUNK = 3 * 1560

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1, 64, 1, (1, 2, 3, 4), "f32", 2, "fixed30", False, (4, 3)),
    "var_d16": Workload("var_d16", 16, 16, 64, 8, VAR_SIDES, "bf16", 6, "massive", False, (4, 3)),
    "var_d20": Workload("var_d20", 20, 20, 64, 128, VAR_SIDES, "bf16", 6, "massive", True, (4, 3)),
    "var_d30": Workload("var_d30", 30, 30, 64, 128, VAR_SIDES, "bf16", 6, "massive", True, (3,)),
    "infinity_2b": Workload("infinity_2b", 32, 16, 128, 8, INFINITY_SIDES, "bf16", 8, "massive", True, (4, 3)),
    "video_self_forcing": Workload("video_self_forcing", 30, 12, 128, 12, (), "bf16", 8, "massive", True, (6, 4),
                                   chunks=(VIDEO_CHUNK,) * 7),
    "video_longlive": Workload("video_longlive", 30, 12, 128, 20, (), "bf16", 8, "massive", True, (6, 4),
                               chunks=(VIDEO_CHUNK,) * 4),
}


def substream_seed(seed: int, layer: int, which: str) -> int:
    """Per-(layer, tensor) seed: seed + 1000*layer + {K: 0, V: 1, Q: 2}."""
    return seed + 1000 * layer + {"k": 0, "v": 1, "q": 2}[which]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draw_kv(w: Workload, layer: int, which: str, seed: int, device) -> torch.Tensor:
    """One layer's K or V in fp32, [B][H][N][D]."""
    g = _gen(device, substream_seed(seed, layer, which))
    B, H, N, D = w.batch, w.heads, w.tokens, w.head_dim
    S = w.num_blocks
    n_s = torch.tensor(w.block_tokens, device=device)
    block_of_token = torch.repeat_interleave(torch.arange(S, device=device), n_s)  # [N]

    x = torch.randn((B, H, N, D), generator=g, device=device, dtype=torch.float32)
    # outlier channel positions: fixed per (layer, head)
    pos = torch.stack([torch.randperm(D, generator=g, device=device)[: w.n_outlier] for _ in range(H)])  # [H, n_out]
    if w.outlier_style == "fixed30":
        mult = torch.ones((B, H, S, D), device=device)
        for h in range(H):
            mult[:, h, :, pos[h]] = 30.0
        offset = (torch.rand((B, H, S), generator=g, device=device) * 10.0 - 5.0)  # U(-5, 5) per block
        x = x * mult[:, :, block_of_token, :] + offset[:, :, block_of_token].unsqueeze(-1)
    else:
        mag = 20.0 + 30.0 * torch.rand((B, H, S, w.n_outlier), generator=g, device=device)  # U(20,50) per cell
        mult = torch.ones((B, H, S, D), device=device)
        for h in range(H):
            mult[:, h, :, pos[h]] = mag[:, h]
        bias = 2.0 * torch.randn((H, D), generator=g, device=device)  # projection bias, std 2, fixed over blocks
        x = x * mult[:, :, block_of_token, :] + bias.view(1, H, 1, D)
        if w.rope_k and which == "k":
            t = torch.arange(N, device=device, dtype=torch.float32)
            inv_freq = torch.pow(10000.0, -torch.arange(0, D, 2, device=device, dtype=torch.float32) / D)
            ang = t[:, None] * inv_freq[None, :]                    # [N, D/2]
            c, s_ = torch.cos(ang), torch.sin(ang)
            x0, x1 = x[..., 0::2], x[..., 1::2]
            r0 = x0 * c - x1 * s_
            r1 = x0 * s_ + x1 * c
            x = torch.stack((r0, r1), dim=-1).reshape(B, H, N, D)
    return x


def make_kv(w: Workload, layer: int, seed: int = 0, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """K and V of one layer, [B][H][N][D], fp32 (tiny) or bf16 (round-to-nearest-even cast)."""
    out = []
    for which in ("k", "v"):
        x = _draw_kv(w, layer, which, seed, device)
        out.append(x if w.kv_dtype == "f32" else x.to(torch.bfloat16))
    return out[0], out[1]


def make_q(w: Workload, layer: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Queries of one layer, [B][H][N][D] bf16, N(0,1), no rotation."""
    g = _gen(device, substream_seed(seed, layer, "q"))
    q = torch.randn((w.batch, w.heads, w.tokens, w.head_dim), generator=g, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16)


def default_softmax_scale(w: Workload) -> float:
    return 1.0 / math.sqrt(w.head_dim)
