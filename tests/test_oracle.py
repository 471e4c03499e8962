"""Pins of the fp64 oracle against things other than itself (CPU only).

* bf16 narrowing against exact rational rounding;
* RoPE closed forms (identity at position 0, known angles on each axis), against an explicit
  rotation-matrix brute force, and the two invariants the method's RoPE fixes (pair norms kept,
  scores depend only on position differences);
* the ring cache + window attention against a brute force that keeps all frames and masks, and
  against torch's fp64 ``scaled_dot_product_attention``;
* closed forms of attention: constant V, q = 0 gives the plain mean of V over exactly the window;
* the key order: the ring's physical slot order gives the oldest-first result.
"""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import workloads as W
from tests.bruteforce import BruteStream, brute_rope, sdpa_check, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------
# bf16 conversions
# ------------------------------------------------------------------------------------------

def _bf16_value(bits: int) -> Fraction:
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return sign * Fraction(m, 1 << 7) * Fraction(1, 1 << 126)
    return sign * (1 + Fraction(m, 1 << 7)) * Fraction(2) ** (e - 127)


def _nearest_bf16_exact(x: float) -> int:
    """RNE by exhaustive comparison of exact rationals among neighbouring bf16 values."""
    fx = Fraction(x)
    f32 = np.float32(x)
    base = int(np.array([f32], dtype=np.float32).view(np.uint32)[0] >> 16)
    cands = []
    for d in range(-2, 3):
        b = base + d
        if b < 0 or (b & 0x7F80) == 0x7F80:
            continue
        if (b ^ base) & 0x8000:
            continue
        cands.append(b)
    best = min(cands, key=lambda b: (abs(_bf16_value(b) - fx), b & 1))
    return best


def test_bf16_widening_is_exact_roundtrip():
    allbits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = allbits[(allbits & 0x7F80) != 0x7F80]
    back = oracle.f64_to_bf16(oracle.bf16_to_f64(finite))
    # -0 and +0 both keep their sign; every finite pattern survives
    assert np.array_equal(back, finite)


def test_bf16_rne_ties_and_double_rounding():
    cases = {
        1.0 + 2.0 ** -8: 0x3F80,               # tie -> even (1.0)
        1.0 + 3 * 2.0 ** -8: 0x3F82,           # tie -> even (1 + 2^-6)
        1.0 + 2.0 ** -8 + 2.0 ** -40: 0x3F81,  # just above the tie: binary32 first would tie
        -(1.0 + 2.0 ** -8 + 2.0 ** -40): 0xBF81,
        2.0 ** -130: 0x0008,                   # bf16 subnormal
    }
    for x, want in cases.items():
        got = int(oracle.f64_to_bf16(np.array([x]))[0])
        assert got == want, (x, hex(got), hex(want))


def test_bf16_rne_against_exact_rationals():
    rng = random.Random(7)
    xs = [rng.gauss(0, 1) * 10 ** rng.uniform(-6, 6) for _ in range(3000)]
    got = oracle.f64_to_bf16(np.array(xs))
    for x, g in zip(xs, got):
        assert int(g) == _nearest_bf16_exact(x), x


# ------------------------------------------------------------------------------------------
# RoPE
# ------------------------------------------------------------------------------------------

SPEC64 = oracle.RopeSpec(24, 20, 20, 10000.0)
SPEC128 = oracle.RopeSpec(44, 42, 42, 10000.0)


def _unit_pair_input(D, pair, H=1):
    x = np.zeros((1, 1, H, D), dtype=np.float64)
    x[..., 2 * pair] = 1.0
    return oracle.f64_to_bf16(x)


def test_rope_identity_at_position_zero():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(1, 1, 4, 128, generator=g).to(torch.bfloat16)
    out = oracle.rope3d(W.bits(x), 0, 1, 1, 1, SPEC128)     # f = y = x = 0
    assert np.array_equal(out, to_f64(x))


@pytest.mark.parametrize("pair,frame,yx,expect_angle", [
    (0, 1, (0, 0), 1.0),        # temporal pair 0: theta^0 = 1 -> angle = f
    (11, 100, (0, 0), 1.0),     # temporal pair 11 of 22: theta^(-1/2) = 0.01 -> 100 * 0.01
    (21, 1, (0, 0), 10000.0 ** (-42.0 / 44.0)),
    (22, 5, (1, 0), 1.0),       # first height pair: angle = y (frame position must not leak in)
    (43, 5, (0, 1), 1.0),       # first width pair: angle = x
    (63, 0, (0, 3), 3 * 10000.0 ** (-40.0 / 42.0)),   # last width pair
])
def test_rope_closed_form_angles(pair, frame, yx, expect_angle):
    Hg, Wg = 4, 4
    y, xx = yx
    D = 128
    x = np.zeros((1, Hg * Wg, 1, D))
    l = y * Wg + xx
    x[0, l, 0, 2 * pair] = 1.0
    out = oracle.rope3d(oracle.f64_to_bf16(x), frame, 1, Hg, Wg, SPEC128)
    a, b = out[0, l, 0, 2 * pair], out[0, l, 0, 2 * pair + 1]
    assert a == pytest.approx(math.cos(expect_angle), abs=1e-14)
    assert b == pytest.approx(math.sin(expect_angle), abs=1e-14)     # +angle rotation
    others = np.delete(out[0, l, 0], [2 * pair, 2 * pair + 1])
    assert np.all(others == 0)


@pytest.mark.parametrize("D,split,Hg,Wg,frames,f0", [
    (64, (24, 20, 20), 4, 6, 3, 0),
    (64, (24, 20, 20), 4, 6, 3, 117),
    (128, (44, 42, 42), 3, 5, 2, 7),
    (8, (4, 2, 2), 2, 3, 3, 5),
    (12, (0, 6, 6), 2, 2, 1, 3),
])
def test_rope_matches_rotation_matrix_bruteforce(D, split, Hg, Wg, frames, f0):
    g = torch.Generator().manual_seed(D * 31 + f0)
    x = torch.randn(2, frames * Hg * Wg, 3, D, generator=g).to(torch.bfloat16)
    spec = oracle.RopeSpec(*split, 10000.0)
    got = oracle.rope3d(W.bits(x), f0, frames, Hg, Wg, spec)
    want = brute_rope(to_f64(x), f0, Hg, Wg, split, 10000.0)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_rope_preserves_pair_norms():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(1, 3 * 24, 2, 64, generator=g).to(torch.bfloat16)
    out = oracle.rope3d(W.bits(x), 9, 3, 4, 6, SPEC64)
    xin = to_f64(x)
    n_in = xin[..., 0::2] ** 2 + xin[..., 1::2] ** 2
    n_out = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-14, atol=1e-15)


def test_rope_scores_depend_only_on_position_difference():
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 24, 1, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 24, 1, 64, generator=g).to(torch.bfloat16)
    for c in (1, 17, 100):
        s0 = np.einsum("ld,md->lm", oracle.rope3d(W.bits(q), 2, 1, 4, 6, SPEC64)[0, :, 0],
                       oracle.rope3d(W.bits(k), 0, 1, 4, 6, SPEC64)[0, :, 0])
        s1 = np.einsum("ld,md->lm", oracle.rope3d(W.bits(q), 2 + c, 1, 4, 6, SPEC64)[0, :, 0],
                       oracle.rope3d(W.bits(k), 0 + c, 1, 4, 6, SPEC64)[0, :, 0])
        np.testing.assert_allclose(s1, s0, rtol=0, atol=1e-12)


def test_rope_rejects_bad_split():
    x = np.zeros((1, 4, 1, 8), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.rope3d(x, 0, 1, 2, 2, oracle.RopeSpec(3, 3, 2))
    with pytest.raises(ValueError):
        oracle.rope3d(x, 0, 2, 2, 2, oracle.RopeSpec(4, 2, 2))   # L != frames*Hg*Wg


# ------------------------------------------------------------------------------------------
# Ring cache + window attention against the brute force
# ------------------------------------------------------------------------------------------

def _stream(shape, cap, window, schedule, seed, start=0, heads=None):
    """Drive the oracle and the brute force through the same sequence of forwards."""
    ol = oracle.OracleLayer(shape.B, shape.H, shape.Hg, shape.Wg,
                            oracle.RopeSpec(shape.d_t, shape.d_h, shape.d_w, shape.theta), cap,
                            heads=heads)
    bf = BruteStream(shape.Hg, shape.Wg, (shape.d_t, shape.d_h, shape.d_w), shape.theta, window)
    results = []
    for n, (frame_idx, frames) in enumerate(schedule):
        q, k, v = W.gen_qkv(seed + n, shape)
        q_rot = ol.append(W.bits(q), W.bits(k), W.bits(v), frame_idx, frames)
        got = ol.attend(q_rot, window)
        hs = ol.heads
        got = got.reshape(shape.B, len(hs), shape.L, shape.D).transpose(0, 2, 1, 3)
        bq, bo, bK, bV, allowed = bf.forward(q, k, v, frame_idx, frames)
        results.append((ol, got, bq, bo, bK, bV, allowed))
    return results


def test_tiny_workload_matches_bruteforce_and_sdpa():
    wl = W.WORKLOADS["tiny"]
    s = wl.shape
    sched = [(wl.frame_idx(c), s.chunk_frames) for c in range(wl.chunks)]
    for ol, got, bq, bo, bK, bV, allowed in _stream(s, wl.cap, wl.window, sched, seed=100):
        np.testing.assert_allclose(got, bo, rtol=0, atol=1e-12)
        np.testing.assert_allclose(sdpa_check(bq, bK, bV, allowed), bo, rtol=0, atol=1e-12)
    # the last chunk (frames 6..8) with cap = window = 6 sees frames 3..8 only
    assert ol.window_frames(wl.window) == [3, 4, 5, 6, 7, 8]
    assert ol.slot_frame == [6, 7, 8, 3, 4, 5]


@pytest.mark.parametrize("cap,window,frames,chunks,start", [
    (4, 4, 2, 5, 0),       # wraps twice
    (5, 3, 1, 7, 0),       # window smaller than the cache
    (6, 4, 2, 4, 11),      # stream starting at a later temporal position
    (9, 9, 3, 3, 0),       # window covers everything: plain block-causal attention
])
def test_ring_window_matches_bruteforce(cap, window, frames, chunks, start):
    shape = W.LayerShape(B=2, H=2, D=8, Hg=2, Wg=3, d_t=4, d_h=2, d_w=2, chunk_frames=frames)
    sched = []
    for c in range(chunks):
        f = start + c * frames
        sched.append((f, frames))
        if c % 2 == 1:
            sched.append((f, frames))            # a re-forward of the same chunk overwrites it
    for ol, got, bq, bo, *_ in _stream(shape, cap, window, sched, seed=cap * 7 + window):
        np.testing.assert_allclose(got, bo, rtol=0, atol=1e-12)


def test_head_subset_is_the_same_arithmetic():
    wl = W.WORKLOADS["tiny"]
    s = wl.shape
    sched = [(wl.frame_idx(c), s.chunk_frames) for c in range(wl.chunks)]
    full = _stream(s, wl.cap, wl.window, sched, seed=5)
    part = _stream(s, wl.cap, wl.window, sched, seed=5, heads=[1])
    for a, b in zip(full, part):
        np.testing.assert_array_equal(a[1][:, :, 1:2], b[1])


def test_shift_invariance_of_outputs():
    shape = W.LayerShape(B=1, H=2, D=8, Hg=2, Wg=2, d_t=4, d_h=2, d_w=2, chunk_frames=2)
    a = _stream(shape, 4, 4, [(0, 2), (2, 2), (4, 2)], seed=1)
    b = _stream(shape, 4, 4, [(13, 2), (15, 2), (17, 2)], seed=1, start=13)
    for ra, rb in zip(a, b):
        np.testing.assert_allclose(ra[1], rb[1], rtol=0, atol=1e-12)


def test_full_window_equals_block_causal_with_sdpa_is_causal():
    """Window covering every frame and one-frame chunks: block-causal = per-frame causal mask."""
    shape = W.LayerShape(B=1, H=1, D=8, Hg=1, Wg=1, d_t=4, d_h=2, d_w=2, chunk_frames=1)
    n = 6
    ol = oracle.OracleLayer(1, 1, 1, 1, oracle.RopeSpec(4, 2, 2), cap=n)
    qs, ks, vs, outs = [], [], [], []
    for f in range(n):
        q, k, v = W.gen_qkv(40 + f, shape)
        q_rot = ol.append(W.bits(q), W.bits(k), W.bits(v), f, 1)
        outs.append(ol.attend(q_rot, n)[0])
        qs.append(q_rot[0, 0, 0])
        ks.append(ol.K[0, 0, f])
        vs.append(ol.V[0, 0, f])
    Q = torch.tensor(np.array(qs))[None, None]
    K = torch.tensor(np.array(ks))[None, None]
    V = torch.tensor(np.array(vs))[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)[0, 0]
    np.testing.assert_allclose(np.array(outs), ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------
# Closed forms of attention
# ------------------------------------------------------------------------------------------

def _layer_with_values(shape, cap, window, sched, vfun, qzero=False, seed=0):
    ol = oracle.OracleLayer(shape.B, shape.H, shape.Hg, shape.Wg,
                            oracle.RopeSpec(shape.d_t, shape.d_h, shape.d_w), cap)
    out = None
    for n, (f0, frames) in enumerate(sched):
        q, k, _ = W.gen_qkv(seed + n, shape)
        if qzero:
            q = torch.zeros_like(q)
        v = vfun(f0, shape).to(torch.bfloat16)
        q_rot = ol.append(W.bits(q), W.bits(k), W.bits(v), f0, frames)
        out = ol.attend(q_rot, window)
    return ol, out


def test_constant_values_give_constant_output():
    shape = W.WORKLOADS["tiny"].shape
    v0 = torch.linspace(-2, 2, shape.D)

    def vconst(f0, s):
        return v0.expand(s.B, s.L, s.H, s.D).clone()

    _, out = _layer_with_values(shape, 6, 6, [(0, 3), (3, 3), (6, 3)], vconst)
    want = v0.to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=1e-14)


def test_zero_query_gives_window_mean():
    """q = 0: uniform weights, so o = mean of V over exactly the window's keys.

    V[:,0] = 1, V[:,1] = frame index, V[:,2] = (token mod 256)/256: a wrong slot, a dropped or
    doubled frame or a wrong window moves columns 1 and 2 away from their closed forms.
    """
    shape = W.LayerShape(B=1, H=2, D=64, Hg=4, Wg=6, d_t=24, d_h=20, d_w=20)
    Tf = shape.Tf

    def vstruct(f0, s):
        v = torch.zeros(s.B, s.L, s.H, s.D)
        l = torch.arange(s.L)
        v[:, :, :, 0] = 1.0
        v[:, :, :, 1] = (f0 + l // Tf).float()[None, :, None]
        v[:, :, :, 2] = ((l % Tf) % 256).float()[None, :, None] / 256
        return v

    for window in (3, 4, 6):
        ol, out = _layer_with_values(shape, 6, window, [(0, 3), (3, 3), (6, 3), (9, 3)],
                                     vstruct, qzero=True)
        frames = ol.window_frames(window)
        assert frames == list(range(12 - window, 12))
        assert np.allclose(out[:, 0], 1.0, atol=1e-14)
        assert np.allclose(out[:, 1], np.mean(frames), atol=1e-12)
        assert np.allclose(out[:, 2], np.mean(np.arange(Tf) % 256) / 256, atol=1e-14)


@pytest.mark.parametrize("cap,window,chunks", [(6, 6, 5), (9, 6, 4), (9, 9, 7)])
def test_physical_slot_order_gives_the_logical_result(cap, window, chunks):
    """Attending the window's keys in the ring's physical slot order (how the cache lies in
    memory, and the order a kernel walks it) gives the oldest-first result up to rounding:
    softmax attention is a sum over keys, so the order of the keys cannot matter."""
    B, H, Hg, Wg, F, D = 1, 2, 3, 4, 3, 64
    ol = oracle.OracleLayer(B, H, Hg, Wg, oracle.RopeSpec(24, 20, 20, 10000.0), cap)
    rng = np.random.default_rng(11)
    for c in range(chunks):
        q, k, v = (oracle.f64_to_bf16(rng.normal(size=(B, F * Hg * Wg, H, D))) for _ in range(3))
        q_rot = ol.append(q, k, v, c * F, F)
    logical = ol.attend(q_rot, window)
    Tf = Hg * Wg
    slots_logical = [ol.slot_of(f) for f in ol.window_frames(window)]
    slots_physical = sorted(slots_logical)
    assert slots_physical != slots_logical        # the window wraps the ring in these cases
    idx = np.concatenate([np.arange(s * Tf, (s + 1) * Tf) for s in slots_physical])
    rows = [(b, l, h) for b in range(B) for h in range(H) for l in range(F * Tf)]
    physical = oracle.attention_rows(q_rot, ol.K[:, :, idx, :], ol.V[:, :, idx, :], rows,
                                     1.0 / math.sqrt(D))
    np.testing.assert_allclose(physical, logical, rtol=1e-12, atol=1e-14)
    # a permutation that is not a reordering of whole keys (one value row moved to another key)
    # must not pass the same check
    bad_v = ol.V[:, :, idx, :].copy()
    bad_v[:, :, [0, 1]] = bad_v[:, :, [1, 0]]
    wrong = oracle.attention_rows(q_rot, ol.K[:, :, idx, :], bad_v, rows, 1.0 / math.sqrt(D))
    assert np.max(np.abs(wrong - logical)) > 1e-6


# ------------------------------------------------------------------------------------------
# Frame-order contract and the pages' schedule
# ------------------------------------------------------------------------------------------

def test_frame_order_rules():
    ol = oracle.OracleLayer(1, 1, 1, 2, oracle.RopeSpec(4, 2, 2), cap=4)
    z = np.zeros((1, 2, 1, 8), dtype=np.uint16)
    ol.append(z, z, z, 0, 1)
    ol.append(z, z, z, 0, 1)          # re-forward
    with pytest.raises(oracle.FrameOrderError):
        ol.append(z, z, z, 2, 1)      # skips frame 1
    ol.append(z, z, z, 1, 1)
    with pytest.raises(oracle.FrameOrderError):
        ol.append(z, z, z, 0, 1)      # not the latest chunk any more
    with pytest.raises(oracle.WindowError):
        ol.window_frames(5)           # larger than the cache


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = [int(x) for x in v]
    return vals


def test_clip_schedule_matches_table3():
    g = _golden("table3_forward_counts.txt")
    wl = W.WORKLOADS["clip30"]
    assert wl.chunks == g["chunks"][0]
    assert wl.shape.chunk_frames == g["frames_per_chunk"][0]
    assert wl.chunks * wl.shape.chunk_frames == g["latent_frames"][0] == g["noise_shape"][1]
    assert sum(W.UNSTEP_FORWARDS) == g["unstep_total_forwards"][0]
    assert sum(W.SELF_FORCING_FORWARDS) == g["self_forcing_total_forwards"][0]
    clean = g["clean_cache_forwards_per_chunk"][0]
    assert W.UNSTEP_FORWARDS[0] == g["unstep_steps_first"][0] + clean
    assert all(n == g["unstep_steps_later"][0] + clean for n in W.UNSTEP_FORWARDS[1:])
    # 60x104 latent, 2x2 patches -> 30x52 tokens per latent frame
    assert (wl.shape.Hg * 2, wl.shape.Wg * 2) == tuple(g["noise_shape"][3:5])

