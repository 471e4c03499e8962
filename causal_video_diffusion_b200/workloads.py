"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module holds shapes, schedules and random-number draws only -- none of the layer's
arithmetic -- so that the CUDA path and the CPU oracle can be fed identical inputs without sharing
any computation.

Shapes follow the paper "UnStep: Training-Free Acceleration of Causal Video Diffusion with Fewer
Steps Than Distillation" (arXiv 2609.32518), Table 3: an 81-frame 832x480 clip is a 1x21x16x60x104
latent (21 latent frames) generated as seven causal chunks of three latent frames; the first chunk
takes four denoising steps and each later chunk two (UnStep), each chunk adding one clean-cache
forward, so a clip costs 23 DiT forwards (35 for the original four-step schedule).  The 60x104
latent grid patchified 2x2 gives 30x52 = 1560 tokens per latent frame.  Head count, head width
and the RoPE split (12 x 128, 44/42/42, theta 10000) are the Wan2.1-1.3B-shaped layer.

Inputs are i.i.d. N(0, 1) draws in fp32 from a seeded torch generator, rounded to bf16 (RNE) --
the unit-variance activations a projected q/k/v stream looks like.  The benchmark the pages
measure quality on (VBench) has no tensors of its own; these draws stand in for the DiT
activations at its shape.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch


@dataclass(frozen=True)
class LayerShape:
    """One attention layer: batch of streams, heads, head width, token grid, RoPE split."""
    B: int
    H: int
    D: int
    Hg: int
    Wg: int
    d_t: int
    d_h: int
    d_w: int
    theta: float = 10000.0
    chunk_frames: int = 3

    @property
    def Tf(self) -> int:
        return self.Hg * self.Wg

    @property
    def L(self) -> int:
        return self.chunk_frames * self.Tf


@dataclass(frozen=True)
class Workload:
    """A layer shape plus how a stream is driven through it."""
    name: str
    shape: LayerShape
    cap: int                 # ring capacity in latent frames
    window: int              # attention window in latent frames
    chunks: int              # chunks streamed
    layers: int = 1
    # forwards per chunk (denoising steps + one clean-cache pass); None = one forward per chunk
    forwards_per_chunk: Optional[Tuple[int, ...]] = None
    start_frame: int = 0

    def forwards(self, chunk: int) -> int:
        if self.forwards_per_chunk is None:
            return 1
        return self.forwards_per_chunk[chunk]

    def frame_idx(self, chunk: int) -> int:
        return self.start_frame + chunk * self.shape.chunk_frames

    def keys_for_chunk(self, chunk: int) -> int:
        f_end = self.frame_idx(chunk) + self.shape.chunk_frames - 1
        first = max(self.start_frame, f_end - self.window + 1)
        return (f_end - first + 1) * self.shape.Tf

    def attn_flops(self, chunk: int) -> int:
        """4 * B * H * L * Lk * D: the two contractions, counted on true (unpadded) keys."""
        s = self.shape
        return 4 * s.B * s.H * s.L * self.keys_for_chunk(chunk) * s.D

    def rope_bytes(self, rotate_q: bool = True) -> int:
        """Algorithmic bytes of one RoPE+append call: read q, k, v; write q, K, V (bf16).
        Without ``rotate_q`` (queries rotated inside the attention): read k, v; write K, V."""
        s = self.shape
        return (6 if rotate_q else 4) * s.B * s.L * s.H * s.D * 2


WAN = dict(H=12, D=128, Hg=30, Wg=52, d_t=44, d_h=42, d_w=42)

# Table 3: four denoising steps for the first chunk, two for each later chunk (UnStep), plus one
# clean-cache forward per chunk -> 5, 3, 3, 3, 3, 3, 3 = 23 forwards.
UNSTEP_FORWARDS = (5, 3, 3, 3, 3, 3, 3)
# the original four-step schedule: 7 x (4 + 1) = 35 forwards.
SELF_FORCING_FORWARDS = (5, 5, 5, 5, 5, 5, 5)

WORKLOADS = {
    # tiny oracle case: 2 heads x 64 (24/20/20), 4x6 grid, chunk 3 frames, window 6, 3 chunks
    "tiny": Workload("tiny", LayerShape(B=1, H=2, D=64, Hg=4, Wg=6, d_t=24, d_h=20, d_w=20),
                     cap=6, window=6, chunks=3),
    # Wan-1.3B-shaped layer, full causal cache: the last chunk of a 21-frame clip sees 21 frames
    "wan_full": Workload("wan_full", LayerShape(B=1, **WAN), cap=21, window=21, chunks=7),
    # the same layer with the limited window W = 9, 7 chunks streamed with eviction
    "wan_window": Workload("wan_window", LayerShape(B=1, **WAN), cap=9, window=9, chunks=7),
    # the 5-s clip schedule through 30 layers, windowed W = 9 (23 forwards per layer)
    "clip30": Workload("clip30", LayerShape(B=1, **WAN), cap=9, window=9, chunks=7, layers=30,
                       forwards_per_chunk=UNSTEP_FORWARDS),
    # 4 independent streams of 120 latent frames (40 chunks), W = 9
    "long_b4": Workload("long_b4", LayerShape(B=4, **WAN), cap=9, window=9, chunks=40),
    # profiling case: the full-cache layer with 8 of its 12 heads (same kernel, same key count,
    # inputs still larger than L2, two thirds of the device memory)
    "wan_full_h8": Workload("wan_full_h8", LayerShape(B=1, **dict(WAN, H=8)), cap=21,
                            window=21, chunks=7),
}


def qkv_seed(base: int, layer: int = 0, forward: int = 0, chunk: int = 0) -> int:
    """Seed of one (layer, chunk, forward) draw; distinct for every call of a workload."""
    return int(base) * 1_000_003 + layer * 10_007 + chunk * 101 + forward


def gen_qkv(seed: int, shape: LayerShape, device: str = "cpu"):
    """q, k, v as bf16 tensors ``[B][L][H][D]``: N(0,1) fp32 draws rounded to bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    dims = (shape.B, shape.L, shape.H, shape.D)
    out = []
    for _ in range(3):
        x = torch.randn(dims, generator=g, dtype=torch.float32, device=device)
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def bits(t: torch.Tensor):
    """The raw bf16 bit patterns of a (CPU) bf16 tensor as a numpy uint16 array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def from_bits(a) -> torch.Tensor:
    """A bf16 CPU tensor from a numpy uint16 array of bit patterns."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


# the truncated-SVD projections of the same layer: 1536 = 12 heads x 128 channels
MODEL_DIM = 12 * 128


def gen_weight(seed: int, d_out: int, d_in: int) -> torch.Tensor:
    """A synthetic fp32 projection weight [d_out][d_in], i.i.d. N(0, 1/d_in) (unit-variance
    outputs for unit-variance inputs), from a seeded CPU generator."""
    g = torch.Generator()
    g.manual_seed(int(seed))
    return torch.randn((d_out, d_in), generator=g, dtype=torch.float32) / (d_in ** 0.5)


def gen_act(seed: int, rows: int, cols: int, device: str = "cpu") -> torch.Tensor:
    """bf16 activations [rows][cols] from N(0, 1) fp32 draws."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn((rows, cols), generator=g, dtype=torch.float32,
                       device=device).to(torch.bfloat16)
