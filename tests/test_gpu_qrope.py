"""Query RoPE inside the attention vs the two-call path, through the C ABI (needs a B200).

The fused form -- unstep_rope_kv_append_ex with UNSTEP_APPEND_DEFER_Q_ROPE, then
unstep_window_attn_ex with UNSTEP_ATTN_ROPE_Q on the un-rotated queries -- must give the same
bits as unstep_rope_kv_append (q rotated in place) followed by unstep_window_attn: the K/V cache,
slot_frame, the metadata and the attention output, after every call; and q must come back
untouched.  The streams cover ragged query tiles, a chunk shorter than one tile, ring wrap (two
key segments), re-forwards, B > 1, late positions, both head widths, both schedules (with and
without scratch) and the Wan-shaped layer; the tiny stream is also checked against the oracle.
"""
import numpy as np
import pytest
import torch

from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.int16)


def _meta(cache):
    c = cache.c
    return (c.frames_written, c.first_frame, c.last_chunk_start, c.last_chunk_frames)


def _pair_stream(shape, cap, window, schedule, seed, use_scratch=True, oracle_check=False):
    mp = max(f + n for f, n in schedule) + 1
    two = P.make_cache(shape, cap, max_pos_t=mp, use_scratch=use_scratch)
    fused = P.make_cache(shape, cap, max_pos_t=mp, use_scratch=use_scratch)
    ol = P.make_oracle(shape, cap) if oracle_check else None
    for n, (f0, frames) in enumerate(schedule):
        q, k, v = W.gen_qkv(seed + n, shape, device="cuda")
        q_two = q.clone()
        two.rope_kv_append(q_two, k, v, f0, frames)
        out_two = two.window_attn(q_two, window)
        q_raw = q.clone()
        fused.rope_kv_append(None, k, v, f0, frames, defer_q=True)
        out_fused = fused.window_attn(q_raw, window, rope_q=True)
        torch.cuda.synchronize()
        assert two.device_error() == 0 and fused.device_error() == 0
        assert torch.equal(_bits(q_raw), _bits(q)), "the fused path wrote q"
        assert torch.equal(_bits(two.k_cache), _bits(fused.k_cache)), n
        assert torch.equal(_bits(two.v_cache), _bits(fused.v_cache)), n
        assert torch.equal(two.slot_frame, fused.slot_frame), n
        assert _meta(two) == _meta(fused), n
        assert torch.equal(_bits(out_two), _bits(out_fused)), (n, f0)
        if ol is not None:
            q_rot = ol.append(W.bits(q.cpu()), W.bits(k.cpu()), W.bits(v.cpu()), f0, frames)
            want = ol.attend(q_rot, window)
            want = want.reshape(shape.B, shape.H, shape.L, shape.D).transpose(0, 2, 1, 3)
            e = P.attn_errors(P.gpu_to_f64(out_fused), want)
            assert e.ok(), (n, f0, e)


@pytest.mark.parametrize("use_scratch", [True, False])
def test_tiny_fused_matches_two_call_and_oracle(use_scratch):
    wl = W.WORKLOADS["tiny"]
    sched = [(wl.frame_idx(c), wl.shape.chunk_frames) for c in range(wl.chunks)]
    _pair_stream(wl.shape, wl.cap, wl.window, sched, seed=41, use_scratch=use_scratch,
                 oracle_check=True)


@pytest.mark.parametrize("D,split", [(64, (24, 20, 20)), (128, (44, 42, 42))])
@pytest.mark.parametrize("Hg,Wg,frames,cap,window,chunks,start,Bn,H", [
    (7, 9, 3, 5, 5, 4, 0, 1, 2),      # 189 queries (2 tiles, ragged), wrap of the ring
    (5, 13, 2, 7, 4, 6, 3, 2, 3),     # window < cap, B = 2, stream starting at frame 3
    (16, 16, 1, 4, 4, 6, 0, 1, 1),    # 256 queries = exactly two tiles, one-frame chunks
    (3, 5, 3, 3, 3, 3, 100, 1, 2),    # 45 queries (less than a tile), late positions
    (11, 23, 3, 9, 9, 3, 0, 1, 2),    # 759 queries: 6 tiles incl. a partial
    (3, 43, 1, 3, 3, 5, 0, 1, 2),     # 129 queries: the second query tile holds one row
])
@pytest.mark.parametrize("use_scratch", [True, False])
def test_fused_streams_match_two_call(D, split, Hg, Wg, frames, cap, window, chunks, start, Bn,
                                      H, use_scratch):
    shape = W.LayerShape(B=Bn, H=H, D=D, Hg=Hg, Wg=Wg, d_t=split[0], d_h=split[1],
                         d_w=split[2], chunk_frames=frames)
    sched = []
    for c in range(chunks):
        f = start + c * frames
        sched.append((f, frames))
        if c == 1:
            sched.append((f, frames))  # re-forward of the same chunk
    _pair_stream(shape, cap, window, sched, seed=3 * D + Hg, use_scratch=use_scratch,
                 oracle_check=(Bn * H * shape.L <= 1200))


@pytest.mark.parametrize("name", ["wan_window", "wan_full"])
def test_wan_layer_fused_matches_two_call(name):
    """The Wan-shaped layer (12 heads, 30 x 52 grid, 4680 queries with a 72-row last tile): the
    stream-K schedule splits units here, so merged pieces are covered too."""
    wl = W.WORKLOADS[name]
    sched = [(wl.frame_idx(c), wl.shape.chunk_frames) for c in range(wl.chunks)]
    _pair_stream(wl.shape, wl.cap, wl.window, sched, seed=77)


def test_four_streams_with_slot_wrap():
    wl = W.WORKLOADS["long_b4"]
    sched = [(wl.frame_idx(c), wl.shape.chunk_frames) for c in range(5)]  # wraps the 9-slot ring
    _pair_stream(wl.shape, wl.cap, wl.window, sched, seed=5)


def test_fused_q_is_rotated_like_the_append():
    """Zero K, V = one-hot rows would hide the rotation; instead check directly: the fused output
    with the RAW q equals the two-call output, and differs from attention on the raw q taken as
    if it were rotated (so the prologue really rotates)."""
    shape = W.LayerShape(B=1, H=2, D=128, Hg=6, Wg=8, d_t=44, d_h=42, d_w=42)
    cache = P.make_cache(shape, 4, max_pos_t=20)
    q, k, v = W.gen_qkv(9, shape, device="cuda")
    cache.rope_kv_append(None, k, v, 7, 3, defer_q=True)
    fused = cache.window_attn(q, 4, rope_q=True)
    plain = cache.window_attn(q, 4)          # raw q used as if rotated
    torch.cuda.synchronize()
    d = (fused.float() - plain.float()).abs().max().item()
    assert d > 1e-2, d
