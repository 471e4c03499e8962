"""The no-allocation attention entry point, through the C ABI (collected last on purpose).

unstep_window_attn_noalloc serves callers that cannot call cudaMalloc (code inside a framework or
allocator that owns every device allocation, or a process whose device footprint must stay fixed
after start-up): it keeps the attention's scratch in a fixed buffer that is part of the library
instead of one the caller provides.  This test streams a layer whose attention splits units
across CTAs (so the scratch is really used), then calls the no-allocation entry point twice in a
row on the same inputs and compares each output with the regular entry point's, within the
tolerance the parity tests use; a call too large for the buffer must be refused.
"""
import ctypes

import pytest
import torch

from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _noalloc(cache, q, window, out):
    L = binding.lib()
    return L.unstep_window_attn_noalloc(q.data_ptr(), ctypes.byref(cache.c), int(window),
                                        out.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("D,split,H", [(128, (44, 42, 42), 3), (64, (24, 20, 20), 5)])
def test_noalloc_matches_regular_entry_point_twice(D, split, H):
    shape = W.LayerShape(B=1, H=H, D=D, Hg=30, Wg=52, d_t=split[0], d_h=split[1],
                         d_w=split[2])
    cap = window = 9
    cache = P.make_cache(shape, cap, max_pos_t=12)
    q = None
    for c in range(4):
        q, k, v = W.gen_qkv(W.qkv_seed(31, chunk=c), shape, device="cuda")
        cache.rope_kv_append(q, k, v, 3 * c, 3)
    want = cache.window_attn(q, window)
    torch.cuda.synchronize()
    want64 = P.gpu_to_f64(want)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        assert _noalloc(cache, q, window, out) == binding.UNSTEP_OK
        torch.cuda.synchronize()
        assert cache.device_error() == 0
        e = P.attn_errors(P.gpu_to_f64(out), want64)
        assert e.max_abs <= P.MAX_ABS and e.mean_abs <= P.MEAN_ABS, (call, e)
        assert torch.equal(out, want), call      # same kernel and schedule: identical bits


def test_noalloc_refuses_calls_beyond_its_buffer():
    # the slots of one call always fit; a call with enough (head, query) units that its
    # counters alone exceed the buffer is refused before anything is launched
    shape = W.LayerShape(B=1, H=12, D=128, Hg=30, Wg=52, d_t=44, d_h=42, d_w=42)
    cache = P.make_cache(shape, 3, max_pos_t=3, use_scratch=False)
    q, k, v = W.gen_qkv(5, shape, device="cuda")
    cache.rope_kv_append(q, k, v, 0, 3)
    c = cache.c
    saved = (c.B, c.H)
    out = torch.empty_like(q)
    try:
        c.H = 1 << 20        # pretend a million heads: counters need > 48 MiB
        rc = _noalloc(cache, q, 3, out)
    finally:
        c.B, c.H = saved
    assert rc == binding.UNSTEP_ERR_SCRATCH_LIMIT
    assert binding.lib().unstep_status_string(rc) == (
        b"the call needs more scratch than the library's fixed device buffer holds")


@pytest.mark.parametrize("D,split", [(64, (24, 20, 20)), (128, (44, 42, 42))])
def test_noalloc_limit_is_exact(D, split):
    """The largest call the buffer holds is accepted and the next larger one is refused.

    The buffer (48 MiB) holds two slots per SM of 2 x (D x 128 + 256) floats and then the
    counters, 8 bytes per (head, 256-query) unit rounded up to 256 bytes.  With one 72-query
    chunk every head is one unit, so the head count sets the unit count.  Only the host-side
    checks run: the cache's K pointer is moved off its 16-byte alignment, so a call that passes
    the size check stops at the tensor map (UNSTEP_ERR_CUDA) and nothing is ever launched."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    slots = 2 * sms * 2 * (D * 128 + 256) * 4
    units_max = ((48 << 20) - slots) // 256 * 32
    shape = W.LayerShape(B=1, H=2, D=D, Hg=4, Wg=6, d_t=split[0], d_h=split[1], d_w=split[2])
    cache = P.make_cache(shape, 3, max_pos_t=3, use_scratch=False)
    q, k, v = W.gen_qkv(9, shape, device="cuda")
    cache.rope_kv_append(q, k, v, 0, 3)
    torch.cuda.synchronize()
    c = cache.c
    saved = (c.H, c.k_cache)
    out = torch.empty_like(q)
    try:
        c.k_cache = c.k_cache + 8
        c.H = units_max
        at_limit = _noalloc(cache, q, 3, out)
        c.H = units_max + 1
        beyond = _noalloc(cache, q, 3, out)
    finally:
        c.H, c.k_cache = saved
    assert at_limit == binding.UNSTEP_ERR_CUDA, at_limit
    assert beyond == binding.UNSTEP_ERR_SCRATCH_LIMIT, beyond
    # the cache is untouched and still works through the regular call
    want = cache.window_attn(q, 3)
    torch.cuda.synchronize()
    assert cache.device_error() == 0 and torch.isfinite(want.float()).all()
