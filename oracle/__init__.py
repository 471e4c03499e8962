"""fp64 CPU oracle of the UnStep chunk-causal attention layer.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the product library never does, and the two share no code.

What it computes follows "UnStep: Training-Free Acceleration of Causal Video Diffusion with Fewer
Steps Than Distillation" (arXiv 2609.32518): the abstract's runtime stack (RoPE with cached
coefficients, KV indexing, a temporal window limit on the attention KV cache) and Table 1 row C4
(the attention window limit added).  The pages print no formulas, so the oracle writes out the
textbook definitions:

* ``rope3d`` -- 3D rotary embedding, channel blocks (t, h, w) of widths (d_t, d_h, d_w), adjacent
  channel pairs, angle ``pos * theta**(-2j/d_a)``, rotation by ``+angle``; arithmetic in C
  (``unstep_oracle.c``).
* ``OracleLayer`` -- a KV cache that keeps the last ``cap`` latent frames, frame ``f`` living in
  slot ``f mod cap``; every forward of a chunk writes its frames (a re-forward of the same chunk
  overwrites them) and then its queries attend to the frames
  ``[max(f_first, f_end - window + 1), f_end]`` (the current chunk included; ``f_first`` is the
  stream's first frame, 0 unless the stream starts at a later position), softmax scale
  ``1/sqrt(D)``; the softmax is the two-pass definition in C.

Outputs are exact fp64 functions of the bf16 inputs; ``stored`` copies (bf16 RNE of the fp64
value) mirror what a bf16 cache holds.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import build as _build

_LIB = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the C part of the oracle."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        ip = ctypes.POINTER(ctypes.c_int)
        L.orc_rope3d.argtypes = [u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, dp]
        L.orc_rope3d.restype = ctypes.c_int
        L.orc_attention_rows.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, dp, dp, ctypes.c_int, ip, ip, ip,
                                         ctypes.c_int, ctypes.c_double, dp]
        L.orc_attention_rows.restype = ctypes.c_int
        L.orc_bf16_array_to_f64.argtypes = [u16p, ctypes.c_long, dp]
        L.orc_bf16_array_to_f64.restype = ctypes.c_int
        L.orc_f64_array_to_bf16.argtypes = [dp, ctypes.c_long, u16p]
        L.orc_f64_array_to_bf16.restype = ctypes.c_int
        L.orc_rope_angle.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        L.orc_rope_angle.restype = ctypes.c_double
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


# --------------------------------------------------------------------------------------------
# bf16 conversions (exact widening; RNE narrowing straight from fp64)
# --------------------------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    rc = lib().orc_bf16_array_to_f64(_ptr(bits, ctypes.c_uint16), bits.size,
                                     _ptr(out, ctypes.c_double))
    assert rc == 0
    return out


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    rc = lib().orc_f64_array_to_bf16(_ptr(x, ctypes.c_double), x.size,
                                     _ptr(out, ctypes.c_uint16))
    assert rc == 0
    return out


# --------------------------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class RopeSpec:
    """Channel split and base of the 3D rotary embedding (t block first, then h, then w)."""
    d_t: int
    d_h: int
    d_w: int
    theta: float = 10000.0

    @property
    def D(self) -> int:
        return self.d_t + self.d_h + self.d_w


def rope_angle(pos: int, j: int, d_a: int, theta: float) -> float:
    """Angle of pair ``j`` of a block of width ``d_a`` at position ``pos``."""
    return float(lib().orc_rope_angle(int(pos), int(j), int(d_a), float(theta)))


def rope3d(x_bits: np.ndarray, frame_idx: int, frames: int, Hg: int, Wg: int,
           spec: RopeSpec) -> np.ndarray:
    """Exact fp64 3D RoPE of one chunk. ``x_bits``: bf16 bits ``[B][L][H][D]``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    B, L, H, D = x_bits.shape
    out = np.empty(x_bits.shape, dtype=np.float64)
    rc = lib().orc_rope3d(_ptr(x_bits, ctypes.c_uint16), B, L, H, D, int(frame_idx), int(frames),
                          int(Hg), int(Wg), spec.d_t, spec.d_h, spec.d_w, float(spec.theta),
                          _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"orc_rope3d rejected its arguments (rc={rc})")
    return out


# --------------------------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------------------------

def attention_rows(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                   rows: Sequence[Tuple[int, int, int]], scale: float) -> np.ndarray:
    """Softmax attention of the selected rows.

    ``q``: fp64 ``[B][L][H][D]``; ``K``, ``V``: fp64 ``[B][H][Nk][D]``; ``rows``: (b, l, h).
    Returns fp64 ``[len(rows)][D]``.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    B, L, H, D = q.shape
    assert K.shape[:2] == (B, H) and K.shape[3] == D and V.shape == K.shape
    Nk = K.shape[2]
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    rb = np.ascontiguousarray(rows[:, 0])
    rl = np.ascontiguousarray(rows[:, 1])
    rh = np.ascontiguousarray(rows[:, 2])
    out = np.empty((rows.shape[0], D), dtype=np.float64)
    rc = lib().orc_attention_rows(_ptr(q, ctypes.c_double), B, L, H, D,
                                  _ptr(K, ctypes.c_double), _ptr(V, ctypes.c_double), Nk,
                                  _ptr(rb, ctypes.c_int), _ptr(rl, ctypes.c_int),
                                  _ptr(rh, ctypes.c_int), rows.shape[0], float(scale),
                                  _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"orc_attention_rows failed (rc={rc})")
    return out


# --------------------------------------------------------------------------------------------
# Ring-buffer KV cache with a temporal window
# --------------------------------------------------------------------------------------------

class FrameOrderError(ValueError):
    pass


class WindowError(ValueError):
    pass


@dataclass
class OracleLayer:
    """One attention layer's cache as the method defines it.

    The cache keeps the last ``cap`` latent frames; frame ``f`` lives in slot ``f mod cap`` and
    its ``Hg*Wg`` tokens occupy rows ``slot*T_f .. slot*T_f + T_f - 1``.  ``heads`` restricts the
    state kept (and the rows that can be attended) to a subset of heads, which is how large
    workloads are sampled; the arithmetic per head does not change.
    """

    B: int
    H: int
    Hg: int
    Wg: int
    spec: RopeSpec
    cap: int
    heads: Optional[Sequence[int]] = None
    slot_frame: List[int] = field(default_factory=list)
    frames_written: int = 0
    last_chunk_start: int = -1
    last_chunk_frames: int = 0
    first_frame: int = 0

    def __post_init__(self):
        self.heads = list(range(self.H)) if self.heads is None else list(self.heads)
        self.D = self.spec.D
        self.Tf = self.Hg * self.Wg
        hs = len(self.heads)
        rows = self.cap * self.Tf
        self.K = np.zeros((self.B, hs, rows, self.D), dtype=np.float64)
        self.V = np.zeros((self.B, hs, rows, self.D), dtype=np.float64)
        self.slot_frame = [-1] * self.cap

    # the cache's indexing rule (bit-exact contract)
    def slot_of(self, f: int) -> int:
        return f % self.cap

    def check_frame_order(self, frame_idx: int, frames: int) -> bool:
        """Returns True for a new chunk, False for a re-forward of the latest chunk."""
        if frames < 1 or frames > self.cap:
            raise WindowError(f"a chunk of {frames} frames does not fit a cache of {self.cap}")
        if self.last_chunk_frames == 0:
            if frame_idx < 0:
                raise FrameOrderError("frame_idx must be >= 0")
            return True     # the stream may start at any temporal position
        if frame_idx == self.frames_written:
            return True
        if frame_idx == self.last_chunk_start and frames == self.last_chunk_frames:
            return False
        raise FrameOrderError(
            f"frame_idx {frame_idx}: expected {self.frames_written} (next chunk) or "
            f"{self.last_chunk_start} (re-forward of the latest chunk)")

    def append(self, q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
               frame_idx: int, frames: int) -> np.ndarray:
        """Rotate q and k of one chunk, write rotated k and v to the ring; return rotated q."""
        B, L, H, D = q_bits.shape
        assert (B, H, D) == (self.B, self.H, self.D) and L == frames * self.Tf
        new = self.check_frame_order(frame_idx, frames)
        q_rot = rope3d(q_bits, frame_idx, frames, self.Hg, self.Wg, self.spec)
        k_rot = rope3d(k_bits, frame_idx, frames, self.Hg, self.Wg, self.spec)
        v = bf16_to_f64(v_bits)
        hs = self.heads
        for i in range(frames):
            f = frame_idx + i
            s = self.slot_of(f)
            rows = slice(s * self.Tf, (s + 1) * self.Tf)
            toks = slice(i * self.Tf, (i + 1) * self.Tf)
            # [B][T_f][H][D] -> [B][Hs][T_f][D]
            self.K[:, :, rows, :] = np.transpose(k_rot[:, toks][:, :, hs, :], (0, 2, 1, 3))
            self.V[:, :, rows, :] = np.transpose(v[:, toks][:, :, hs, :], (0, 2, 1, 3))
            self.slot_frame[s] = f
        if new:
            if self.last_chunk_frames == 0:
                self.first_frame = frame_idx
            self.frames_written = frame_idx + frames
        self.last_chunk_start = frame_idx
        self.last_chunk_frames = frames
        return q_rot

    def fill_zero_frames(self, frame_idx: int, frames: int) -> None:
        """Record a chunk whose rotated keys and values are all zero (no arithmetic: used to
        bring a cache to a late position quickly when only timing or coverage matters)."""
        new = self.check_frame_order(frame_idx, frames)
        for i in range(frames):
            f = frame_idx + i
            s = self.slot_of(f)
            self.K[:, :, s * self.Tf:(s + 1) * self.Tf, :] = 0.0
            self.V[:, :, s * self.Tf:(s + 1) * self.Tf, :] = 0.0
            self.slot_frame[s] = f
        if new:
            if self.last_chunk_frames == 0:
                self.first_frame = frame_idx
            self.frames_written = frame_idx + frames
        self.last_chunk_start = frame_idx
        self.last_chunk_frames = frames

    def window_frames(self, window: int) -> List[int]:
        """Frames the latest chunk attends to, oldest first."""
        if self.last_chunk_frames == 0:
            raise WindowError("no chunk has been appended")
        if window < self.last_chunk_frames or window > self.cap:
            raise WindowError(f"window {window} outside [{self.last_chunk_frames}, {self.cap}]")
        f_end = self.last_chunk_start + self.last_chunk_frames - 1
        return list(range(max(self.first_frame, f_end - window + 1), f_end + 1))

    def window_kv(self, window: int) -> Tuple[np.ndarray, np.ndarray]:
        """Keys and values of the window in logical frame order, ``[B][Hs][Nk][D]``."""
        frames = self.window_frames(window)
        idx = []
        for f in frames:
            s = self.slot_of(f)
            if self.slot_frame[s] != f:
                raise WindowError(f"frame {f} is no longer resident")
            idx.extend(range(s * self.Tf, (s + 1) * self.Tf))
        idx = np.asarray(idx, dtype=np.int64)
        return self.K[:, :, idx, :], self.V[:, :, idx, :]

    def attend(self, q_rot: np.ndarray, window: int,
               rows: Optional[Iterable[Tuple[int, int, int]]] = None) -> np.ndarray:
        """Attention of the latest chunk's rotated queries over the window.

        ``rows``: (b, l, h) with h among ``heads``; default every row of every kept head.
        Returns ``[nrows][D]`` in the order of ``rows``.
        """
        K, V = self.window_kv(window)
        hs = self.heads
        hpos = {h: i for i, h in enumerate(hs)}
        B, L = q_rot.shape[:2]
        if rows is None:
            rows = [(b, l, h) for b in range(B) for h in hs for l in range(L)]
        rows = [(int(b), int(l), hpos[int(h)]) for (b, l, h) in rows]
        q_sub = np.ascontiguousarray(q_rot[:, :, hs, :])
        return attention_rows(q_sub, K, V, rows, 1.0 / math.sqrt(self.D))

    def stored_k(self) -> np.ndarray:
        """The rotated keys as a bf16 cache holds them (RNE of the fp64 rotation)."""
        return f64_to_bf16(self.K)


# --------------------------------------------------------------------------------------------
# Truncated-SVD projections (abstract; Figure 11 / Table 5: V/O rank retention 0.92)
# --------------------------------------------------------------------------------------------

def matmul_bt(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """C = A B^T in fp64 from bf16 bit patterns (A [M][K], B [N][K])."""
    return bf16_to_f64(a_bits) @ bf16_to_f64(b_bits).T


def lowrank_linear(x_bits, w1_bits, w2_bits, round_t: bool = False) -> np.ndarray:
    """y = (x w1^T) w2^T in fp64; with round_t the rank-space product is rounded to bf16 (RNE)
    first, as a bf16 intermediate buffer holds it."""
    t = matmul_bt(x_bits, w1_bits)
    if round_t:
        t = bf16_to_f64(f64_to_bf16(t))
    return t @ bf16_to_f64(w2_bits).T


def svd_truncate(W: np.ndarray, rank: int):
    """Factors of the rank-`rank` truncation of W [d_out][d_in] by numpy's SVD:
    (w1 = (V_r S_r)^T [rank][d_in], w2 = U_r [d_out][rank], singular values)."""
    U, S, Vh = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return (S[:rank, None] * Vh[:rank]), U[:, :rank], S


# --------------------------------------------------------------------------------------------
# Renoise (abstract; Tables 4 and 5: renoise the generated latent to sigma* before the clean pass)
# --------------------------------------------------------------------------------------------

def renoise(x0_bits: np.ndarray, eps_bits: np.ndarray, sigma: float) -> np.ndarray:
    """(1 - sigma) x0 + sigma eps in fp64 from bf16 bit patterns."""
    return (1.0 - sigma) * bf16_to_f64(x0_bits) + sigma * bf16_to_f64(eps_bits)


# --------------------------------------------------------------------------------------------
# Causal 3D convolution of the VAE decoder (abstract and Table 1 row C2: the decoder is sped up
# through its memory layout, precision and convolution kernels)
# --------------------------------------------------------------------------------------------

def conv3d_causal(x_bits: np.ndarray, w_bits: np.ndarray,
                  bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Causal 3x3x3 convolution in fp64 from bf16 bit patterns, channels-last.

    x: [B][T + 2][H][W][C_in] -- each stream's first two frames are its causal history (the
    frames the previous chunk ended with, zeros at a stream's start); w: [C_out][3][3][3][C_in]
    indexed by the taps (dt, dy, dx); bias: [C_out] (fp64) or None.  Output [B][T][H][W][C_out]:

        y[b, t, h, x, o] = bias[o] + sum over dt, dy, dx, c of
                           w[o, dt, dy, dx, c] * in[b, t + dt, h + dy - 1, x + dx - 1, c]

    with positions outside the frame reading 0 (one position of zero padding in h and w), so that
    output frame t sees input frames t .. t + 2 (its own frame and the two before it).  Written
    as the sum over the 27 taps of a shifted slice times the tap's [C_in][C_out] matrix.
    """
    x = bf16_to_f64(x_bits)
    wt = bf16_to_f64(w_bits)
    B, Tin, H, W, Ci = x.shape
    Co = wt.shape[0]
    assert wt.shape == (Co, 3, 3, 3, Ci) and Tin >= 3
    T = Tin - 2
    xp = np.zeros((B, Tin, H + 2, W + 2, Ci))
    xp[:, :, 1:H + 1, 1:W + 1, :] = x
    y = np.zeros((B, T, H, W, Co))
    for dt in range(3):
        for dy in range(3):
            for dx in range(3):
                y += xp[:, dt:dt + T, dy:dy + H, dx:dx + W, :] @ wt[:, dt, dy, dx, :].T
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64)
    return y
