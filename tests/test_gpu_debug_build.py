"""The debug build of the library (index checks compiled into the kernels) on real workloads.

libunstep_debug.so is the same source compiled with -DUNSTEP_DEBUG: the append and attention
kernels check every ring slot, cache row, table row, TMA coordinate, scratch slot and counter
index before using it, and a failed check records UNSTEP_ERR_DEVICE_BOUNDS in the cache's error
word instead of touching memory.  The tiny stream and the W = 9 Wan stream (ring wrap, stream-K
split units and their merges) must run with no check failing and with the oracle's results."""
import importlib.util
import os

import numpy as np
import pytest
import torch

from causal_video_diffusion_b200 import build as cuda_build
from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    """A second instance of the binding module, bound to the debug library."""
    path = cuda_build.build(debug=True)
    spec = importlib.util.spec_from_file_location(
        "binding_debug", os.path.join(cuda_build.PKG, "binding.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.LIB_PATH = path
    mod._LIB = None
    assert os.path.basename(mod.lib()._name) == "libunstep_debug.so"
    return mod


def _stream(dbg, name, rows_per_chunk=None, seed=21):
    wl = W.WORKLOADS[name]
    s = wl.shape
    cache = dbg.LayerCache(s.B, s.H, s.D, s.Hg, s.Wg, s.d_t, s.d_h, s.d_w, cap_frames=wl.cap,
                           max_pos_t=wl.frame_idx(wl.chunks), theta=s.theta)
    heads = [0, s.H - 1] if s.H > 2 else list(range(s.H))
    ol = P.make_oracle(s, wl.cap, heads=heads)
    rng = np.random.default_rng(seed)
    for c in range(wl.chunks):
        q, k, v = W.gen_qkv(W.qkv_seed(seed, chunk=c), s, device="cuda")
        src = [W.bits(t.cpu()) for t in (q, k, v)]
        cache.rope_kv_append(q, k, v, wl.frame_idx(c), s.chunk_frames)
        out = cache.window_attn(q, wl.window)
        torch.cuda.synchronize()
        assert cache.device_error() == 0, (name, c)
        q_rot = ol.append(*src, wl.frame_idx(c), s.chunk_frames)
        ls = range(s.L) if rows_per_chunk is None else P.sample_rows(s.L, s.Tf, rows_per_chunk,
                                                                      rng)
        rows = [(b, l, h) for b in range(s.B) for h in heads for l in ls]
        want = ol.attend(q_rot, wl.window, rows)
        got = out.cpu().double().numpy()
        e = P.attn_errors(np.stack([got[b, l, h] for (b, l, h) in rows]), want)
        assert e.max_abs <= P.MAX_ABS and e.mean_abs <= P.MEAN_ABS, (name, c, e)
    P.compare_cache(cache, ol, heads)


def test_debug_build_tiny_stream(dbg):
    _stream(dbg, "tiny")


def test_debug_build_wan_window_stream(dbg):
    _stream(dbg, "wan_window", rows_per_chunk=32)


def test_debug_build_reports_its_status_text(dbg):
    assert dbg.lib().unstep_status_string(dbg.UNSTEP_ERR_DEVICE_BOUNDS) == (
        b"a device-side index check failed (debug build)")


def test_debug_build_one_valid_key_tiles(dbg):
    """129 tokens a frame, one-frame chunks over a 3-frame ring: a 1-row second query tile and
    ring segments that end in key tiles with a single valid key, with every index check on."""
    shape = W.LayerShape(B=1, H=2, D=128, Hg=3, Wg=43, d_t=44, d_h=42, d_w=42, chunk_frames=1)
    cap = window = 3
    cache = dbg.LayerCache(shape.B, shape.H, shape.D, shape.Hg, shape.Wg, shape.d_t, shape.d_h,
                           shape.d_w, cap_frames=cap, max_pos_t=8, theta=shape.theta)
    ol = P.make_oracle(shape, cap)
    for f in range(6):
        q, k, v = W.gen_qkv(500 + f, shape)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        cache.rope_kv_append(qd, kd, vd, f, 1)
        out = cache.window_attn(qd, window)
        torch.cuda.synchronize()
        assert cache.device_error() == 0, f
        q_rot = ol.append(W.bits(q), W.bits(k), W.bits(v), f, 1)
        want = ol.attend(q_rot, window)
        want = want.reshape(shape.B, shape.H, shape.L, shape.D).transpose(0, 2, 1, 3)
        e = P.attn_errors(out.cpu().double().numpy(), want)
        assert e.ok(), (f, e)
