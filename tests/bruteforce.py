"""Brute-force restatement of the layer, used only to pin the oracle on tiny inputs.

It is built differently from the oracle on purpose, so that a slip in one does not repeat in the
other:

* RoPE is an explicit block-diagonal D x D rotation matrix per token, assembled from per-axis
  frequency vectors and applied as a matrix-vector product (the oracle rotates pair by pair);
* the cache is not a ring: every frame ever written is kept, and the temporal window is an
  explicit boolean mask over the whole sequence of frames (the oracle gathers ring slots);
* the softmax is a dense masked softmax over all keys in numpy; ``torch`` fp64
  ``scaled_dot_product_attention`` with the same mask is a library cross-check.
"""
from __future__ import annotations

import math
from typing import Dict, List, Tuple

import numpy as np
import torch


def freq_vector(D: int, d_t: int, d_h: int, d_w: int, theta: float):
    """Per-pair inverse frequency and the axis (0 = t, 1 = h, 2 = w) each pair reads."""
    inv = []
    axis = []
    for a, d in enumerate((d_t, d_h, d_w)):
        inv.append(theta ** (-np.arange(0, d, 2, dtype=np.float64) / d))
        axis.append(np.full(d // 2, a))
    inv = np.concatenate(inv)
    axis = np.concatenate(axis)
    assert inv.shape[0] == D // 2
    return inv, axis


def rotation_matrix(D, d_t, d_h, d_w, theta, f, y, x) -> np.ndarray:
    inv, axis = freq_vector(D, d_t, d_h, d_w, theta)
    pos = np.array([f, y, x], dtype=np.float64)[axis]
    ang = pos * inv
    R = np.zeros((D, D))
    for p in range(D // 2):
        c, s = math.cos(ang[p]), math.sin(ang[p])
        R[2 * p:2 * p + 2, 2 * p:2 * p + 2] = [[c, -s], [s, c]]
    return R


def brute_rope(x: np.ndarray, frame_idx: int, Hg: int, Wg: int, split, theta) -> np.ndarray:
    """x: fp64 [B][L][H][D] of one chunk -> rotated copy."""
    B, L, H, D = x.shape
    Tf = Hg * Wg
    out = np.empty_like(x)
    for l in range(L):
        i, tok = divmod(l, Tf)
        y, xx = divmod(tok, Wg)
        R = rotation_matrix(D, *split, theta, frame_idx + i, y, xx)
        out[:, l] = np.einsum("de,bhe->bhd", R, x[:, l])
    return out


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


class BruteStream:
    """Keeps every frame ever written; the window is a mask over all of them."""

    def __init__(self, Hg, Wg, split, theta, window):
        self.Hg, self.Wg, self.split, self.theta, self.window = Hg, Wg, split, theta, window
        self.frames: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}
        self.first = None

    def forward(self, q_bf16, k_bf16, v_bf16, frame_idx, frames) -> Tuple[np.ndarray, ...]:
        Tf = self.Hg * self.Wg
        q = brute_rope(to_f64(q_bf16), frame_idx, self.Hg, self.Wg, self.split, self.theta)
        k = brute_rope(to_f64(k_bf16), frame_idx, self.Hg, self.Wg, self.split, self.theta)
        v = to_f64(v_bf16)
        if self.first is None:
            self.first = frame_idx
        for i in range(frames):
            self.frames[frame_idx + i] = (k[:, i * Tf:(i + 1) * Tf], v[:, i * Tf:(i + 1) * Tf])
        f_end = frame_idx + frames - 1
        order = sorted(self.frames)
        K = np.concatenate([self.frames[f][0] for f in order], axis=1)   # [B][Nall][H][D]
        V = np.concatenate([self.frames[f][1] for f in order], axis=1)
        key_frame = np.repeat(np.array(order), Tf)
        lo = max(self.first, f_end - self.window + 1)
        allowed = (key_frame >= lo) & (key_frame <= f_end)              # same for every query
        D = q.shape[-1]
        s = np.einsum("blhd,bnhd->bhln", q, K) / math.sqrt(D)
        s = np.where(allowed[None, None, None, :], s, -np.inf)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        o = np.einsum("bhln,bnhd->blhd", p, V)
        return q, o, K, V, allowed


def sdpa_check(q: np.ndarray, K: np.ndarray, V: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """torch fp64 scaled_dot_product_attention with the same boolean key mask."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)          # [B][H][L][D]
    kt = torch.from_numpy(K).permute(0, 2, 1, 3)
    vt = torch.from_numpy(V).permute(0, 2, 1, 3)
    mask = torch.from_numpy(allowed)[None, None, None, :].expand(qt.shape[0], qt.shape[1],
                                                                  qt.shape[2], -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    return o.permute(0, 2, 1, 3).numpy()
