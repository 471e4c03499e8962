"""The C ABI without a GPU: the library loads, exports what include/unstep.h declares, and its
host-side logic (table sizes, frame-order rules, ring slots, window resolution, argument checks)
agrees with the oracle's.  No call here reaches a kernel launch."""
import ctypes
import os
import random
import struct
import subprocess

import numpy as np
import pytest

import oracle
from causal_video_diffusion_b200 import binding as B
from causal_video_diffusion_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "unstep.h")
INIT_MAGIC = 0x55535450  # the value unstep_cache_init stores in `initialized`


@pytest.fixture(scope="module")
def L():
    from causal_video_diffusion_b200 import build
    build.build()
    return B.lib()


def _cache(shape, cap, max_pos_t=128, fake_ptrs=False):
    c = B.unstep_cache_t()
    c.B, c.H, c.D, c.Hg, c.Wg = shape.B, shape.H, shape.D, shape.Hg, shape.Wg
    c.d_t, c.d_h, c.d_w, c.theta = shape.d_t, shape.d_h, shape.d_w, shape.theta
    c.cap_frames, c.max_pos_t = cap, max_pos_t
    if fake_ptrs:  # never dereferenced: only calls that fail validation are made with these
        c.k_cache, c.v_cache, c.slot_frame, c.cos_sin, c.dev_error = (
            0x100000, 0x200000, 0x300000, 0x400000, 0x500000)
    return c


def test_every_declared_symbol_is_exported(L):
    declared = B.declared_symbols(HEADER)
    assert set(declared) == set(B._SIGNATURES), declared
    nm = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = {line.split()[-1] for line in nm.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(L, s)


def test_status_strings(L):
    for code in range(-8, 1):
        assert L.unstep_status_string(code)
    assert L.unstep_status_string(-8) == b"a device-side wait timed out"
    assert L.unstep_version() == 101


def test_table_and_cache_sizes(L):
    s = W.WORKLOADS["wan_full"].shape
    c = _cache(s, 21, max_pos_t=120)
    assert L.unstep_cache_table_bytes(ctypes.byref(c)) == 8 * (120 * 22 + 30 * 21 + 52 * 21)
    assert L.unstep_cache_kv_bytes(ctypes.byref(c)) == 1 * 12 * 21 * 1560 * 128 * 2
    c.D, c.d_t = 96, 12        # split still sums to D but D is unsupported
    assert L.unstep_cache_table_bytes(ctypes.byref(c)) == 0
    c = _cache(s, 21)
    c.d_h = 41                 # odd block
    assert L.unstep_cache_table_bytes(ctypes.byref(c)) == 0
    # the attention scratch depends on the device's SM count: 0 without a usable device
    import torch
    if not torch.cuda.is_available():
        assert L.unstep_attn_scratch_bytes(ctypes.byref(_cache(s, 21))) == 0


def test_init_rejects_bad_arguments_without_touching_the_device(L):
    s = W.WORKLOADS["tiny"].shape
    c = _cache(s, 6)
    assert L.unstep_cache_init(ctypes.byref(c), None) == B.UNSTEP_ERR_ARG      # NULL pointers
    c = _cache(s, 6, fake_ptrs=True)
    c.k_cache = 0x100008                                                        # misaligned
    assert L.unstep_cache_init(ctypes.byref(c), None) == B.UNSTEP_ERR_ALIGN
    c = _cache(s, 6, fake_ptrs=True)
    c.theta = -1.0
    assert L.unstep_cache_init(ctypes.byref(c), None) == B.UNSTEP_ERR_ARG
    assert L.unstep_cache_init(None, None) == B.UNSTEP_ERR_ARG


def _sync_meta(c, ol):
    c.frames_written = ol.frames_written
    c.first_frame = ol.first_frame
    c.last_chunk_start = ol.last_chunk_start
    c.last_chunk_frames = ol.last_chunk_frames
    c.initialized = INIT_MAGIC


def test_plans_agree_with_the_oracle_ring(L):
    """Slots, new/re-forward classification and window rows, state by state."""
    rng = random.Random(3)
    for trial in range(60):
        cap = rng.randint(1, 9)
        frames = rng.randint(1, cap)
        Hg, Wg = rng.randint(1, 4), rng.randint(1, 5)
        shape = W.LayerShape(B=1, H=1, D=64, Hg=Hg, Wg=Wg, d_t=24, d_h=20, d_w=20,
                             chunk_frames=frames)
        start = rng.choice([0, 0, rng.randint(0, 40)])
        ol = oracle.OracleLayer(1, 1, Hg, Wg, oracle.RopeSpec(24, 20, 20), cap, heads=[])
        c = _cache(shape, cap, max_pos_t=400)
        _sync_meta(c, ol)
        f = start
        for step in range(rng.randint(1, 12)):
            reforward = step > 0 and rng.random() < 0.3
            fi = ol.last_chunk_start if reforward else f
            slots = (ctypes.c_int * frames)()
            rc = L.unstep_append_plan(ctypes.byref(c), fi, B.unstep_grid_t(frames, Hg, Wg), slots)
            z = np.zeros((1, frames * Hg * Wg, 1, 64), dtype=np.uint16)
            new = ol.check_frame_order(fi, frames)
            assert rc == int(new)
            assert list(slots) == [ol.slot_of(fi + i) for i in range(frames)]
            ol.append(z, z, z, fi, frames)
            _sync_meta(c, ol)
            if not reforward:
                f += frames
            for window in range(frames, cap + 1):
                plan = B.unstep_window_plan_t()
                assert L.unstep_window_plan(ctypes.byref(c), window, ctypes.byref(plan)) == 0
                want_frames = ol.window_frames(window)
                assert (plan.first_frame, plan.last_frame) == (want_frames[0], want_frames[-1])
                rows = list(range(plan.seg_row[0], plan.seg_row[0] + plan.seg_len[0])) + \
                    list(range(plan.seg_row[1], plan.seg_row[1] + plan.seg_len[1]))
                want_rows = [ol.slot_of(fr) * ol.Tf + t for fr in want_frames
                             for t in range(ol.Tf)]
                assert rows == want_rows
                assert plan.keys == len(want_rows)


def test_frame_order_and_window_errors(L):
    s = W.WORKLOADS["tiny"].shape
    c = _cache(s, 6, fake_ptrs=True)
    c.initialized = INIT_MAGIC
    c.frames_written, c.first_frame, c.last_chunk_start, c.last_chunk_frames = 6, 0, 3, 3
    g = B.unstep_grid_t(3, 4, 6)
    assert L.unstep_append_plan(ctypes.byref(c), 6, g, None) == 1      # next chunk
    assert L.unstep_append_plan(ctypes.byref(c), 3, g, None) == 0      # re-forward
    assert L.unstep_append_plan(ctypes.byref(c), 0, g, None) == B.UNSTEP_ERR_FRAME_ORDER
    assert L.unstep_append_plan(ctypes.byref(c), 9, g, None) == B.UNSTEP_ERR_FRAME_ORDER
    assert L.unstep_append_plan(ctypes.byref(c), 3, B.unstep_grid_t(2, 4, 6), None) == \
        B.UNSTEP_ERR_FRAME_ORDER                                        # re-forward, other size
    assert L.unstep_append_plan(ctypes.byref(c), 6, B.unstep_grid_t(3, 4, 5), None) == \
        B.UNSTEP_ERR_SHAPE
    assert L.unstep_append_plan(ctypes.byref(c), 6, B.unstep_grid_t(7, 4, 6), None) == \
        B.UNSTEP_ERR_WINDOW                                             # chunk > capacity
    assert L.unstep_append_plan(ctypes.byref(c), 126, g, None) == B.UNSTEP_ERR_ARG  # > max_pos_t
    plan = B.unstep_window_plan_t()
    assert L.unstep_window_plan(ctypes.byref(c), 2, ctypes.byref(plan)) == B.UNSTEP_ERR_WINDOW
    assert L.unstep_window_plan(ctypes.byref(c), 7, ctypes.byref(plan)) == B.UNSTEP_ERR_WINDOW
    # the failing calls of the product entry points return before any launch
    q = ctypes.c_void_p(0x600000)
    assert L.unstep_rope_kv_append(q, q, q, ctypes.byref(c), 0, g, None) == \
        B.UNSTEP_ERR_FRAME_ORDER
    assert L.unstep_rope_kv_append(ctypes.c_void_p(0x600004), q, q, ctypes.byref(c), 6, g,
                                   None) == B.UNSTEP_ERR_ALIGN
    assert L.unstep_rope_kv_append(None, q, q, ctypes.byref(c), 6, g, None) == B.UNSTEP_ERR_ARG
    assert L.unstep_window_attn(q, ctypes.byref(c), 7, q, None) == B.UNSTEP_ERR_WINDOW
    assert L.unstep_window_attn(ctypes.c_void_p(0x600002), ctypes.byref(c), 6, q, None) == \
        B.UNSTEP_ERR_ALIGN
    c2 = _cache(s, 6, fake_ptrs=True)           # never initialised
    assert L.unstep_window_attn(q, ctypes.byref(c2), 6, q, None) == B.UNSTEP_ERR_ARG
    # a failed call leaves the metadata unchanged
    assert (c.frames_written, c.last_chunk_start, c.last_chunk_frames) == (6, 3, 3)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_LIB", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="has not been built"):
        B.lib()


def test_exp2_polynomial_coefficients_match_their_derivation():
    """The constants in the kernel header are the Remez fit that tests/exp2_remez.py derives,
    and that fit is the minimax one: its relative error on [-1/2, 1/2] equioscillates (five
    alternating extrema of equal size for a cubic), stays below bf16's half ulp, and no
    perturbation of a coefficient lowers the maximum."""
    import re
    from tests import exp2_remez as m
    hdr = open(os.path.join(ROOT, "causal_video_diffusion_b200", "csrc", "sm100.cuh")).read()
    consts = np.array([float(v) for v in re.findall(r"kExp2C\d = ([0-9.eE+-]+)f;", hdr)])
    assert consts.size == 4
    c = m.remez_exp2()
    assert np.allclose(consts, np.float32(c), rtol=0, atol=1e-7)
    assert m.max_rel_err(consts) < 8e-5 < 2.0 ** -9
    xs = np.linspace(-0.5, 0.5, 200001)
    err = (np.polyval(c[::-1], xs) - np.exp2(xs)) / np.exp2(xs)
    ext = [0] + [i for i in range(1, xs.size - 1)
                 if abs(err[i]) >= abs(err[i - 1]) and abs(err[i]) >= abs(err[i + 1])
                 and abs(err[i]) > 0.9 * np.abs(err).max()] + [xs.size - 1]
    signs = np.sign(err[ext])
    assert len(ext) == 5 and all(signs[i] == -signs[i + 1] for i in range(4))
    assert np.ptp(np.abs(err[ext])) < 1e-3 * np.abs(err).max()
    base = m.max_rel_err(c)
    for k in range(4):
        for d in (1e-6, -1e-6):
            cc = np.array(c, dtype=np.float64)
            cc[k] += d
            assert m.max_rel_err(cc) > base


def test_multiply_high_division_method():
    """The kernels divide by run-time invariants with Granlund & Montgomery's multiply-high
    method (m = floor(2^32 (2^l - d) / d) + 1, l = ceil(log2 d), q = (umulhi(x, m) + x) >> l);
    check it against exact division over the dividend range they use (x < 2^31)."""
    rng = np.random.default_rng(9)
    ds = [1, 2, 3, 5, 7, 12, 19, 21, 24, 52, 1560, 4680, 65535, 65536, 999983, 2 ** 20 + 1]
    ds += [int(d) for d in rng.integers(1, 2 ** 24, size=40)]
    xs = np.concatenate([rng.integers(0, 2 ** 31, size=4000, dtype=np.int64),
                         np.array([0, 1, 2 ** 31 - 1, 2 ** 31 - 2], dtype=np.int64)])
    for d in ds:
        l = 0
        while (1 << l) < d:
            l += 1
        m = ((1 << 32) * ((1 << l) - d)) // d + 1
        assert m < (1 << 32)
        xs_d = np.concatenate([xs, np.arange(0, 4 * d, max(1, d // 3), dtype=np.int64)[:2000],
                               (np.arange(1, 200, dtype=np.int64) * d - 1)])
        xs_d = xs_d[(xs_d >= 0) & (xs_d < 2 ** 31)]
        hi = (xs_d.astype(object) * m) >> 32
        q = np.array([(int(h) + int(x)) >> l for h, x in zip(hi, xs_d)], dtype=np.int64)
        assert np.array_equal(q, xs_d // d), d


def test_ex_entry_points_flags_and_errors(L):
    """The flag forms of the append and the attention reject unknown flags; a deferred-q append
    ignores q (NULL or misaligned); every failing call returns before any launch."""
    s = W.WORKLOADS["tiny"].shape
    c = _cache(s, 6, fake_ptrs=True)
    c.initialized = INIT_MAGIC
    c.frames_written, c.first_frame, c.last_chunk_start, c.last_chunk_frames = 6, 0, 3, 3
    g = B.unstep_grid_t(3, 4, 6)
    q = ctypes.c_void_p(0x600000)
    odd = ctypes.c_void_p(0x600004)
    defer = B.UNSTEP_APPEND_DEFER_Q_ROPE
    assert L.unstep_rope_kv_append_ex(q, q, q, ctypes.byref(c), 6, g, 2, None) == B.UNSTEP_ERR_ARG
    assert L.unstep_rope_kv_append_ex(q, q, q, ctypes.byref(c), 6, g, 0x80000000, None) == \
        B.UNSTEP_ERR_ARG
    # with the flag, q plays no part: NULL or misaligned q reach the frame-order check
    assert L.unstep_rope_kv_append_ex(None, q, q, ctypes.byref(c), 0, g, defer, None) == \
        B.UNSTEP_ERR_FRAME_ORDER
    assert L.unstep_rope_kv_append_ex(odd, q, q, ctypes.byref(c), 0, g, defer, None) == \
        B.UNSTEP_ERR_FRAME_ORDER
    # without it q is checked first
    assert L.unstep_rope_kv_append_ex(None, q, q, ctypes.byref(c), 0, g, 0, None) == \
        B.UNSTEP_ERR_ARG
    assert L.unstep_rope_kv_append_ex(odd, q, q, ctypes.byref(c), 0, g, 0, None) == \
        B.UNSTEP_ERR_ALIGN
    # k and v are still required
    assert L.unstep_rope_kv_append_ex(None, None, q, ctypes.byref(c), 6, g, defer, None) == \
        B.UNSTEP_ERR_ARG
    assert L.unstep_rope_kv_append_ex(None, q, odd, ctypes.byref(c), 6, g, defer, None) == \
        B.UNSTEP_ERR_ALIGN
    rq = B.UNSTEP_ATTN_ROPE_Q
    assert L.unstep_window_attn_ex(q, ctypes.byref(c), 6, q, 4, None) == B.UNSTEP_ERR_ARG
    assert L.unstep_window_attn_ex(q, ctypes.byref(c), 7, q, rq, None) == B.UNSTEP_ERR_WINDOW
    assert L.unstep_window_attn_ex(None, ctypes.byref(c), 6, q, rq, None) == B.UNSTEP_ERR_ARG
    assert L.unstep_window_attn_ex(odd, ctypes.byref(c), 6, q, rq, None) == B.UNSTEP_ERR_ALIGN
    c2 = _cache(s, 6, fake_ptrs=True)           # never initialised
    assert L.unstep_window_attn_ex(q, ctypes.byref(c2), 6, q, rq, None) == B.UNSTEP_ERR_ARG
    assert L.unstep_rope_kv_append_ex(None, q, q, ctypes.byref(c2), 0, g, defer, None) == \
        B.UNSTEP_ERR_ARG
    assert (c.frames_written, c.last_chunk_start, c.last_chunk_frames) == (6, 3, 3)


def test_shard_fields_are_validated_on_the_host(L):
    """A cache may be a (stream, head) shard of larger activations; the shard must lie inside
    them (checked with the shape, before any device work)."""
    s = W.LayerShape(B=2, H=3, D=64, Hg=4, Wg=6, d_t=24, d_h=20, d_w=20)
    ok = [(0, 0, 0, 0), (0, 0, 2, 3), (1, 2, 3, 5), (0, 0, 2, 0), (0, 9, 0, 12)]
    bad = [(1, 0, 2, 3), (0, 1, 2, 3), (-1, 0, 3, 3), (0, 0, 1, 3), (0, 0, -1, 3),
           (0, 0, 1 << 16, 1 << 15)]
    for fields, want_ok in [(f, True) for f in ok] + [(f, False) for f in bad]:
        c = _cache(s, 3, max_pos_t=3)
        c.b0, c.h0, c.act_B, c.act_H = fields
        assert (L.unstep_cache_table_bytes(ctypes.byref(c)) > 0) == want_ok, fields


def _state_header(c, frames_written=6, last=(3, 3)):
    """A checkpoint header as unstep_cache_save writes it (the layout include/unstep.h gives)."""
    buf = bytearray(L_state_bytes(c))
    f = [c.B, c.H, c.D, c.Hg, c.Wg, c.d_t, c.d_h, c.d_w, c.cap_frames, c.max_pos_t,
         c.act_B or c.B, c.act_H or c.H, c.b0, c.h0]
    struct.pack_into("<2i14i", buf, 0, 0x43545355, 1, *f)
    struct.pack_into("<d4i", buf, 64, c.theta, frames_written, 0, last[0], last[1])
    return buf


def L_state_bytes(c):
    return B.lib().unstep_cache_state_bytes(ctypes.byref(c))


def test_state_buffer_size(L):
    s = W.WORKLOADS["wan_window"].shape
    c = _cache(s, 9, max_pos_t=21)
    kv = L.unstep_cache_kv_bytes(ctypes.byref(c))
    assert kv == s.B * s.H * 9 * s.Hg * s.Wg * s.D * 2
    # 128-byte header, slot_frame padded to 16 bytes, then K and V
    assert L.unstep_cache_state_bytes(ctypes.byref(c)) == 128 + 48 + 2 * kv
    c.B = 0
    assert L.unstep_cache_state_bytes(ctypes.byref(c)) == 0


def test_restore_refuses_foreign_or_damaged_state_before_any_copy(L):
    """Host-side checks only (the cache's device pointers are fake and never touched)."""
    s = W.LayerShape(B=1, H=2, D=64, Hg=4, Wg=6, d_t=24, d_h=20, d_w=20)
    c = _cache(s, 6, max_pos_t=12, fake_ptrs=True)
    c.initialized = INIT_MAGIC
    good = _state_header(c)
    n = len(good)

    def restore(buf, size=None):
        raw = (ctypes.c_ubyte * len(buf)).from_buffer(buf)
        return L.unstep_cache_restore(ctypes.byref(c), raw, n if size is None else size, None)

    bad_magic = bytearray(good)
    bad_magic[0] ^= 1
    assert restore(bad_magic) == B.UNSTEP_ERR_ARG
    bad_version = bytearray(good)
    bad_version[4] = 2
    assert restore(bad_version) == B.UNSTEP_ERR_ARG
    for off, val in [(8, 2), (12, 3), (16, 128), (40, 7), (44, 13), (56, 1)]:  # B, H, D, cap, ...
        other = bytearray(good)
        other[off:off + 4] = val.to_bytes(4, "little")
        assert restore(other) == B.UNSTEP_ERR_SHAPE, off
    theta = bytearray(good)
    theta[64:72] = struct.pack("<d", 500.0)
    assert restore(theta) == B.UNSTEP_ERR_SHAPE
    assert restore(bytearray(good), size=n - 1) == B.UNSTEP_ERR_ARG        # short buffer
    too_far = _state_header(c, frames_written=13)                          # past max_pos_t
    assert restore(too_far) == B.UNSTEP_ERR_ARG
    assert (c.frames_written, c.last_chunk_start) == (0, 0)               # cache unchanged
