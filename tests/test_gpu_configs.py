"""The five workloads at full size on the GPU, checked against the oracle on sampled rows.

Every query row of a sample (tile and frame boundaries, the ragged last tile, random rows) is
compared element by element with the fp64 oracle; the oracle sees only the sampled heads
(heads are independent), so it stays fast.  Ring slots are compared bit-exactly after every
call, and the q = 0 closed form checks every output element of the full-size layer.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _sliced_oracle(wl, heads):
    s = wl.shape
    return oracle.OracleLayer(s.B, len(heads), s.Hg, s.Wg,
                              oracle.RopeSpec(s.d_t, s.d_h, s.d_w, s.theta), wl.cap)


def _check_rows(out_gpu, ol, q_rot, wl, heads, rows_per_head, rng, bs=None):
    s = wl.shape
    bs = list(range(s.B)) if bs is None else bs
    rows = P.sample_rows(s.L, s.Tf, rows_per_head, rng)
    sel = [(b, l, hi) for b in bs for hi in range(len(heads)) for l in rows]
    want = ol.attend(q_rot, wl.window, sel)
    got = np.stack([P.gpu_to_f64(out_gpu[b, l, heads[hi]]) for (b, l, hi) in sel])
    e = P.attn_errors(got, want)
    assert e.ok(), e
    assert e.rel_rms < 0.02, e
    return e


def test_wan_full_cache_last_chunk_all_heads():
    """Wan-shaped layer, full causal cache: the last chunk attends 32760 keys."""
    wl = W.WORKLOADS["wan_full"]
    s = wl.shape
    # the oracle needs the real keys of every frame in the window: keep all chunks for 3 heads
    heads = [0, 5, 11]
    rng = np.random.default_rng(1)
    cache = P.make_cache(s, wl.cap, max_pos_t=21)
    ol = _sliced_oracle(wl, heads)
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
    for c in range(wl.chunks):
        q, k, v = W.gen_qkv(W.qkv_seed(77, chunk=c), s)
        qd = q.cuda()
        cache.rope_kv_append(qd, k.cuda(), v.cuda(), wl.frame_idx(c), 3)
        cache.window_attn(qd, wl.window, out=out)
        sub = [np.ascontiguousarray(W.bits(t)[:, :, heads]) for t in (q, k, v)]
        q_rot = ol.append(*sub, wl.frame_idx(c), 3)
        assert cache.slot_frame.cpu().tolist() == ol.slot_frame
        if c in (0, 6):
            torch.cuda.synchronize()
            _check_rows(out, ol, q_rot, wl, heads, 160 if c == 6 else 32, rng)
    assert wl.keys_for_chunk(6) == 32760


@pytest.mark.parametrize("use_scratch", [True, False])
def test_wan_window_stream_every_chunk(use_scratch):
    """W = 9: 4680, 9360, then 14040 keys; the ring wraps from chunk 3 on."""
    wl = W.WORKLOADS["wan_window"]
    s = wl.shape
    heads = [3, 8]
    rng = np.random.default_rng(2)
    cache = P.make_cache(s, wl.cap, max_pos_t=21, use_scratch=use_scratch)
    ol = _sliced_oracle(wl, heads)
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
    for c in range(wl.chunks):
        q, k, v = W.gen_qkv(W.qkv_seed(88, chunk=c), s)
        qd = q.cuda()
        cache.rope_kv_append(qd, k.cuda(), v.cuda(), wl.frame_idx(c), 3)
        cache.window_attn(qd, wl.window, out=out)
        sub = [np.ascontiguousarray(W.bits(t)[:, :, heads]) for t in (q, k, v)]
        q_rot = ol.append(*sub, wl.frame_idx(c), 3)
        torch.cuda.synchronize()
        assert cache.slot_frame.cpu().tolist() == ol.slot_frame
        _check_rows(out, ol, q_rot, wl, heads, 48, rng)
    assert [wl.keys_for_chunk(c) for c in range(7)] == [4680, 9360] + [14040] * 5


def test_clip30_schedule_two_layers():
    """The 5-s clip through 30 stacked layers: 23 forwards per layer (Table 3); every forward
    writes its chunk and attends.  Layers 0 and 29 are checked against the oracle at every
    forward's last step of each chunk; all layers share one attention scratch."""
    wl = W.WORKLOADS["clip30"]
    s = wl.shape
    assert sum(wl.forwards(c) for c in range(wl.chunks)) == 23
    heads = [7]
    rng = np.random.default_rng(3)
    first = P.make_cache(s, wl.cap, max_pos_t=21)
    caches = [first] + [P.make_cache(s, wl.cap, max_pos_t=21, scratch=first.scratch)
                        for _ in range(wl.layers - 1)]
    checked = {0: _sliced_oracle(wl, heads), 29: _sliced_oracle(wl, heads)}
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
    calls = 0
    for c in range(wl.chunks):
        for f in range(wl.forwards(c)):
            for layer, cache in enumerate(caches):
                q, k, v = W.gen_qkv(W.qkv_seed(99, layer=layer, chunk=c, forward=f), s,
                                    device="cuda")
                q_host = q.cpu() if layer in checked else None
                cache.rope_kv_append(q, k, v, wl.frame_idx(c), 3)
                cache.window_attn(q, wl.window, out=out)
                calls += 1
                if layer in checked:
                    ol = checked[layer]
                    sub = [np.ascontiguousarray(W.bits(t)[:, :, heads])
                           for t in (q_host, k.cpu(), v.cpu())]
                    q_rot = ol.append(*sub, wl.frame_idx(c), 3)
                    torch.cuda.synchronize()
                    _check_rows(out, ol, q_rot, wl, heads, 24, rng)
    assert calls == 23 * 30
    for cache in caches:
        assert cache.device_error() == 0


def test_long_stream_batch4():
    """4 streams x 120 frames, W = 9: temporal positions up to 119, the ring wraps 13 times."""
    wl = W.WORKLOADS["long_b4"]
    s = wl.shape
    heads = [2]
    rng = np.random.default_rng(4)
    cache = P.make_cache(s, wl.cap, max_pos_t=120)
    ol = _sliced_oracle(wl, heads)
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
    check = {0, 1, 2, 3, 20, 38, 39}
    for c in range(wl.chunks):
        q, k, v = W.gen_qkv(W.qkv_seed(111, chunk=c), s, device="cuda")
        qh = q.cpu() if (c in check or c + 1 in check or c + 2 in check) else None
        cache.rope_kv_append(q, k, v, wl.frame_idx(c), 3)
        cache.window_attn(q, wl.window, out=out)
        if qh is not None:
            # chunks that end up in a checked chunk's window go through the oracle for real
            sub = [np.ascontiguousarray(W.bits(t)[:, :, heads]) for t in (qh, k.cpu(), v.cpu())]
            q_rot = ol.append(*sub, wl.frame_idx(c), 3)
        else:
            ol.fill_zero_frames(wl.frame_idx(c), 3)
        if c in check:
            torch.cuda.synchronize()
            assert cache.slot_frame.cpu().tolist() == ol.slot_frame
            _check_rows(out, ol, q_rot, wl, heads, 24, rng, bs=[0, 3])
    assert wl.frame_idx(39) + 2 == 119
    assert cache.device_error() == 0


@pytest.mark.parametrize("name", ["wan_full", "wan_window", "long_b4"])
def test_zero_query_closed_form_full_size(name):
    """q = 0 at full size: every output element equals the mean of V over the window."""
    wl = W.WORKLOADS[name]
    s = wl.shape
    cache = P.make_cache(s, wl.cap, max_pos_t=wl.frame_idx(wl.chunks))
    out = torch.empty(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
    l = torch.arange(s.L, device="cuda")
    for c in range(wl.chunks):
        f0 = wl.frame_idx(c)
        q = torch.zeros(s.B, s.L, s.H, s.D, dtype=torch.bfloat16, device="cuda")
        k = torch.randn(s.B, s.L, s.H, s.D, device="cuda").to(torch.bfloat16)
        v = torch.zeros(s.B, s.L, s.H, s.D, device="cuda")
        v[..., 0] = 1.0
        v[..., 1] = (f0 + l // s.Tf).float()[None, :, None]
        v[..., 2] = ((l % s.Tf) % 256).float()[None, :, None] / 256
        v[..., 3] = torch.arange(s.B, device="cuda").float()[:, None, None]
        cache.rope_kv_append(q, k, v.to(torch.bfloat16), f0, 3)
        cache.window_attn(q, wl.window, out=out)
    o = out.double()
    f_end = wl.frame_idx(wl.chunks - 1) + 2
    frames = np.arange(max(0, f_end - wl.window + 1), f_end + 1)
    for col, val in ((0, 1.0), (1, float(frames.mean())),
                     (2, float(np.mean(np.arange(s.Tf) % 256) / 256))):
        tol = float(P.bf16_ulp(np.array([val]))[0]) * 0.51 + 1e-7 * abs(val)
        assert torch.all((o[..., col] - val).abs() <= tol), (col, val)
    for b in range(s.B):
        assert torch.all(o[b, :, :, 3] == float(b))
    assert torch.all(o[..., 4:] == 0)
