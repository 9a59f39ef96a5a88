"""Seeded synthetic workloads shaped like the pages' video latents.

This module holds shapes and random-number generation only: none of the method's arithmetic.
Both the CUDA path (tests, bench) and the CPU oracle take their inputs from here, so both see
identical bf16 bits.

Shapes (latent grids after a 1x2x2 patchify):
  * CogVideoX, 49 frames of 480x720 through a 4x8x8 causal VAE: 13 x 30 x 45 tokens, with a
    226-token text prefix ("CogVideoX" section 2: text and video concatenated).
  * Open-Sora Plan, 93x480x640 through a 4x8x8 VAE: 24 x 30 x 40.
  * Open-Sora Plan v1.5, 121x576x1024 through an 8x8x8 VAE: 16 x 36 x 64.
Values: q, k, v ~ N(0, 1), drawn in fp32 by torch's CPU generator and rounded to bf16 (RNE);
seeds q = s, k = s + 1, v = s + 2 with s = 1000 + the config's index below.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    heads: int
    head_dim: int
    grid: tuple            # (T, H, W)
    text_len: int
    split: tuple           # RoPE channels (d_t, d_h, d_w)
    skiparse_k: int = 0    # 0: no Skiparse case for this workload
    theta: float = 10000.0
    ops: tuple = field(default=("dense",))

    @property
    def n_video(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def seq_len(self) -> int:
        return self.text_len + self.n_video

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def dense_flops(self) -> float:
        """4 * B * heads * N^2 * d (QK^T and PV, 2 flops per multiply-add)."""
        return 4.0 * self.B * self.heads * self.seq_len ** 2 * self.head_dim

    def skiparse_flops(self, k: int | None = None) -> float:
        k = k or self.skiparse_k
        return 4.0 * self.B * self.heads * self.n_video ** 2 * self.head_dim / k

    def rope_bytes(self) -> int:
        """q and k, read and written, over the video tokens (text tokens are untouched)."""
        return 2 * 2 * self.B * self.n_video * self.heads * self.head_dim * 2

    def describe(self) -> dict:
        T, H, W = self.grid
        return {"workload": self.name, "B": self.B, "heads": self.heads, "head_dim": self.head_dim,
                "grid": f"{T}x{H}x{W}", "text_len": self.text_len, "seq_len": self.seq_len,
                "rope_split": "/".join(str(s) for s in self.split), "theta": self.theta}


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", 0, 1, 2, 64, (4, 8, 8), 0, (16, 24, 24), skiparse_k=2,
                 ops=("dense", "single", "group")),
        Workload("cogvideox_2b", 1, 1, 30, 64, (13, 30, 45), 226, (16, 24, 24)),
        Workload("open_sora_plan", 2, 1, 24, 96, (24, 30, 40), 0, (32, 32, 32), skiparse_k=4,
                 ops=("dense", "single", "group")),
        Workload("cogvideox_5b", 3, 2, 48, 64, (13, 30, 45), 226, (16, 24, 24)),
        Workload("long_video", 4, 1, 32, 128, (16, 36, 64), 0, (32, 48, 48), skiparse_k=4,
                 ops=("dense", "single", "group")),
    ]
}


def randn_bf16(shape, seed: int) -> torch.Tensor:
    """N(0,1) fp32 from torch's CPU generator with ``seed``, rounded to bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_qkv(w: Workload, seed: int | None = None):
    """q, k, v as CPU bf16 tensors [B, N, heads, head_dim] (BSHD, contiguous)."""
    s = w.seed if seed is None else seed
    shape = (w.B, w.seq_len, w.heads, w.head_dim)
    return randn_bf16(shape, s), randn_bf16(shape, s + 1), randn_bf16(shape, s + 2)


def custom(name: str, B: int, heads: int, head_dim: int, grid, text_len: int, split,
           skiparse_k: int = 0, index: int = 100) -> Workload:
    """An ad-hoc workload (tests use these for ragged and edge-case shapes)."""
    return Workload(name, index, B, heads, head_dim, tuple(grid), text_len, tuple(split), skiparse_k)


@dataclass(frozen=True)
class PackedWorkload:
    """A packed batch of samples of different shapes (CogVideoX section 3.1, Multi-Resolution
    Frame Pack): each sample is (text_len, T, H, W); all share heads and head_dim."""
    name: str
    index: int
    heads: int
    head_dim: int
    samples: tuple          # ((text_len, T, H, W), ...)
    split: tuple
    theta: float = 10000.0

    @property
    def lengths(self) -> list:
        return [L + T * H * W for L, T, H, W in self.samples]

    @property
    def total(self) -> int:
        return sum(self.lengths)

    @property
    def bounds(self) -> list:
        out = [0]
        for n in self.lengths:
            out.append(out[-1] + n)
        return out

    @property
    def seed(self) -> int:
        return 2000 + self.index

    def flops(self) -> float:
        """4 * heads * d * sum_i N_i^2 (block-diagonal attention, QK^T and PV)."""
        return 4.0 * self.heads * self.head_dim * sum(n * n for n in self.lengths)

    def describe(self) -> dict:
        return {"workload": self.name, "heads": self.heads, "head_dim": self.head_dim,
                "samples": ["%d+%dx%dx%d" % s for s in self.samples], "tokens": self.total,
                "rope_split": "/".join(str(s) for s in self.split)}


# CogVideoX-2B-shaped heads; 49- and 25-frame clips at 480x720, a 49-frame clip at 384x640, a
# 960x1440 image and a 480x720 image, each with a 226-token prompt
PACKED_WORKLOADS = {
    w.name: w for w in [
        PackedWorkload("frame_pack_cog2b", 0, 30, 64,
                       ((226, 13, 30, 45), (226, 7, 30, 45), (226, 13, 24, 40), (226, 1, 60, 90), (226, 1, 30, 45)),
                       (16, 24, 24)),
    ]
}


def make_packed_qkv(heads: int, head_dim: int, total: int, seed: int, total_kv: int | None = None):
    """q [1, total, heads, d] and k, v [1, total_kv (default total), heads, d], CPU bf16."""
    nkv = total if total_kv is None else total_kv
    return (randn_bf16((1, total, heads, head_dim), seed), randn_bf16((1, nkv, heads, head_dim), seed + 1),
            randn_bf16((1, nkv, heads, head_dim), seed + 2))
