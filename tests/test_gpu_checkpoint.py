"""Checkpoint and resume of a stream's layer state through the C ABI.

A stream saved after chunk k and restored into a fresh cache continues exactly as the
uninterrupted stream does: same output bits for every later chunk, same ring, same slot map and
metadata."""
import pytest
import torch

from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _inputs(wl, seed):
    return [W.gen_qkv(W.qkv_seed(seed, chunk=c), wl.shape, device="cuda")
            for c in range(wl.chunks)]


def _step(cache, wl, c, qkv):
    q, k, v = (t.clone() for t in qkv)
    cache.rope_kv_append(q, k, v, wl.frame_idx(c), wl.shape.chunk_frames)
    return cache.window_attn(q, wl.window)


@pytest.mark.parametrize("name,save_after", [("wan_window", 3), ("wan_window", 0),
                                              ("tiny", 1)])
def test_resume_continues_the_stream_bit_for_bit(name, save_after):
    wl = W.WORKLOADS[name]
    s = wl.shape
    data = _inputs(wl, seed=77)
    max_pos = wl.frame_idx(wl.chunks)

    ref = P.make_cache(s, wl.cap, max_pos_t=max_pos)
    want = [_step(ref, wl, c, data[c]) for c in range(wl.chunks)]

    first = P.make_cache(s, wl.cap, max_pos_t=max_pos)
    for c in range(save_after + 1):
        _step(first, wl, c, data[c])
    state = first.save_state()
    assert state.numel() == first.state_bytes()
    del first                                  # the original cache is gone

    resumed = P.make_cache(s, wl.cap, max_pos_t=max_pos)
    resumed.restore_state(state)
    assert resumed.c.frames_written == wl.frame_idx(save_after + 1)
    assert resumed.c.last_chunk_start == wl.frame_idx(save_after)
    for c in range(save_after + 1, wl.chunks):
        got = _step(resumed, wl, c, data[c])
        assert torch.equal(got, want[c]), c
    torch.cuda.synchronize()
    assert resumed.device_error() == 0
    assert torch.equal(resumed.slot_frame, ref.slot_frame)
    assert torch.equal(resumed.k_cache, ref.k_cache) and torch.equal(resumed.v_cache, ref.v_cache)
    for f in ("frames_written", "first_frame", "last_chunk_start", "last_chunk_frames"):
        assert getattr(resumed.c, f) == getattr(ref.c, f), f


def test_resume_allows_the_next_denoising_step_of_the_saved_chunk():
    """A re-forward of the chunk that was latest when the state was saved is accepted."""
    wl = W.WORKLOADS["tiny"]
    data = _inputs(wl, seed=78)
    a = P.make_cache(wl.shape, wl.cap, max_pos_t=12)
    _step(a, wl, 0, data[0])
    _step(a, wl, 1, data[1])
    state = a.save_state()
    want = _step(a, wl, 1, data[2])            # another forward of chunk 1, new inputs
    b = P.make_cache(wl.shape, wl.cap, max_pos_t=12)
    b.restore_state(state)
    assert torch.equal(_step(b, wl, 1, data[2]), want)


def test_restore_refuses_another_shape():
    wl = W.WORKLOADS["tiny"]
    a = P.make_cache(wl.shape, wl.cap, max_pos_t=12)
    _step(a, wl, 0, _inputs(wl, seed=79)[0])
    state = a.save_state()
    other = P.make_cache(wl.shape, wl.cap + 1, max_pos_t=12)
    buf = torch.zeros(other.state_bytes(), dtype=torch.uint8)   # large enough for `other`
    n = min(buf.numel(), state.numel())
    buf[:n] = state[:n]
    with pytest.raises(binding.UnstepError) as e:
        other.restore_state(buf)
    assert e.value.status == binding.UNSTEP_ERR_SHAPE
    assert other.c.last_chunk_frames == 0                      # nothing was restored
