"""Shared drivers for the GPU parity tests: run the same seeded stream through the CUDA library
and through the oracle, and compare element by element."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import numpy as np
import torch

import oracle
from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import workloads as W

# the layer's stated tolerance for unit-variance inputs (GPU bf16 output vs exact fp64)
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (normal range; subnormal spacing below 2^-126)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    e = np.floor(np.log2(ax))
    return np.exp2(e - 7)


def rope_error_bound(exact: np.ndarray, src: np.ndarray) -> np.ndarray:
    """Bound on |bf16(fp32 rotation) - exact|: half a bf16 ulp of the result (one binade of
    slack) plus the fp32 evaluation error of a*c - b*s with fp32 cos/sin, <= 4*2^-24*(|a|+|b|)."""
    a = np.abs(src[..., 0::2])
    b = np.abs(src[..., 1::2])
    pair = np.repeat(a + b, 2, axis=-1)
    return 0.5 * bf16_ulp(np.abs(exact) * (1 + 2.0 ** -7)) + 4 * 2.0 ** -24 * pair + 1e-38


def gpu_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def make_cache(shape: W.LayerShape, cap: int, max_pos_t: int, use_scratch: bool = True,
               scratch=None) -> binding.LayerCache:
    return binding.LayerCache(shape.B, shape.H, shape.D, shape.Hg, shape.Wg, shape.d_t,
                              shape.d_h, shape.d_w, cap_frames=cap, max_pos_t=max_pos_t,
                              theta=shape.theta, use_scratch=use_scratch, scratch=scratch)


def make_oracle(shape: W.LayerShape, cap: int, heads=None) -> oracle.OracleLayer:
    return oracle.OracleLayer(shape.B, shape.H, shape.Hg, shape.Wg,
                              oracle.RopeSpec(shape.d_t, shape.d_h, shape.d_w, shape.theta), cap,
                              heads=heads)


@dataclass
class Errors:
    max_abs: float
    mean_abs: float
    rel_rms: float
    n: int

    def ok(self) -> bool:
        return self.max_abs <= MAX_ABS and self.mean_abs <= MEAN_ABS


def attn_errors(got: np.ndarray, want: np.ndarray) -> Errors:
    d = np.abs(got - want)
    rms = math.sqrt(float(np.mean((got - want) ** 2)))
    ref = math.sqrt(float(np.mean(want ** 2))) or 1.0
    return Errors(float(d.max()), float(d.mean()), rms / ref, int(d.size))


def sample_rows(L: int, Tf: int, n_random: int, rng: np.random.Generator) -> List[int]:
    """Query rows at tile (128) and frame boundaries, the whole last tile, plus random rows."""
    rows = set()
    for t in range(0, L, 128):
        rows.update(x for x in (t - 1, t, t + 1, t + 127) if 0 <= x < L)
    for f in range(0, L, Tf):
        rows.update(x for x in (f - 1, f, f + 1) if 0 <= x < L)
    rows.update(range((L - 1) // 128 * 128, L))
    rows.update(int(x) for x in rng.integers(0, L, size=n_random))
    return sorted(rows)


def compare_cache(cache: binding.LayerCache, ol: oracle.OracleLayer, heads: Sequence[int]):
    """slot_frame bit-exact; V rows bit-exact copies; K rows within the RoPE bound."""
    sf = cache.slot_frame.cpu().numpy().tolist()
    assert sf == ol.slot_frame, (sf, ol.slot_frame)
    filled = [s for s in range(ol.cap) if ol.slot_frame[s] >= 0]
    rows = np.concatenate([np.arange(s * ol.Tf, (s + 1) * ol.Tf) for s in filled])
    hs = list(heads)
    kd = gpu_to_f64(cache.k_cache[:, hs][:, :, rows])
    vd = gpu_to_f64(cache.v_cache[:, hs][:, :, rows])
    kx = ol.K[:, :, rows]
    vx = ol.V[:, :, rows]
    assert np.array_equal(vd, vx), "V cache rows are not bit-exact copies"
    err = np.abs(kd - kx)
    # bound from the exact value alone (the source pair is not kept by the oracle's ring):
    # half an ulp plus a generous fp32 evaluation term relative to the pair's norm
    a = np.abs(kx[..., 0::2]) + np.abs(kx[..., 1::2])
    pair = np.repeat(a, 2, axis=-1) * 1.5
    bound = 0.5 * bf16_ulp(np.abs(kx) * (1 + 2.0 ** -7)) + 4 * 2.0 ** -24 * pair + 1e-38
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} K elements beyond the rounding bound"
    exact_rne = float(np.mean(kd == oracle.bf16_to_f64(oracle.f64_to_bf16(kx))))
    return exact_rne
