"""The clip driver and the renoise kernel on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import clip
from causal_video_diffusion_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sigma", [0.0, 0.02, 0.625, 1.0])
@pytest.mark.parametrize("n", [299520, 8, 13, 1])
def test_renoise_matches_oracle(sigma, n):
    g = torch.Generator().manual_seed(n)
    x = torch.randn(n, generator=g).to(torch.bfloat16)
    e = torch.randn(n, generator=g).to(torch.bfloat16)
    got = binding.renoise(x.cuda(), e.cuda(), sigma).cpu()
    want = oracle.renoise(W.bits(x), W.bits(e), sigma)
    want_bf = oracle.bf16_to_f64(oracle.f64_to_bf16(want))
    g64 = got.double().numpy()
    if sigma in (0.0, 1.0):
        assert np.array_equal(g64, want_bf)            # exact: one operand is passed through
    # half a bf16 ulp of the result plus the fp32 evaluation error of (1-s) x0 + s eps, which
    # scales with the terms (they can cancel), not with the result
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
    terms = (1 - sigma) * np.abs(oracle.bf16_to_f64(W.bits(x))) + \
        sigma * np.abs(oracle.bf16_to_f64(W.bits(e)))
    assert np.all(np.abs(g64 - want) <= 0.5 * ulp * 1.01 + 2.0 ** -22 * terms + 1e-30)


def test_clip_graph_replays_the_eager_clip_exactly():
    """Three layers through the whole 23-forward schedule: the CUDA graph of the clip gives the
    same bits as launching every call eagerly, and every forward of Table 3 is issued."""
    wl = W.WORKLOADS["clip30"]
    drv = clip.ClipDriver(wl, layers=3, seed=4)
    assert drv.calls == 23 * 3
    pristine = [[t.clone() for t in (q,)] for row in drv.inputs for (q, k, v) in row]
    drv.run()
    torch.cuda.synchronize()
    eager = [o.clone() for o in drv.outs]
    lat_eager = drv.latent.clone()
    for c in drv.caches:
        assert c.device_error() == 0
    # restore the rotated-in-place queries, empty the caches, capture and replay
    i = 0
    for row in drv.inputs:
        for (q, k, v) in row:
            q.copy_(pristine[i][0])
            i += 1
    drv.reset()
    drv.capture()
    drv.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, drv.outs):
        assert torch.equal(a, b)
    assert torch.equal(lat_eager, drv.latent)
    # the clean-cache pass renoises to sigma* = 0.02 (the last forward of the clip)
    want = oracle.renoise(W.bits(drv.x_hat.cpu()), W.bits(drv.eps[-1].cpu()), 0.02)
    got = drv.latent.cpu().double().numpy()
    assert np.max(np.abs(got - want)) < 2e-2


def _oracle_clip_check(wl, layers, seed, heads, rows_per_forward=None):
    """Run the driver eagerly, keep every forward's output of every layer, and recompute each
    from the oracle with inputs regenerated from the documented seeds (layer, chunk, forward),
    streamed through one oracle cache per layer in the schedule's order.  This pins the driver's
    own sequencing: the frame index of every forward, which inputs go to which (forward, layer),
    and that every layer keeps its own ring."""
    from causal_video_diffusion_b200 import schedule as S
    from tests import parity as P
    s = wl.shape
    drv = clip.ClipDriver(wl, layers=layers, seed=seed)
    kept = []
    drv.run(on_forward=lambda n: kept.append([o.clone() for o in drv.outs]))
    torch.cuda.synchronize()
    for c in drv.caches:
        assert c.device_error() == 0
    sched = S.clip_schedule("unstep", wl.chunks)
    assert len(kept) == len(sched) == sum(wl.forwards(c) for c in range(wl.chunks))
    ols = [P.make_oracle(s, wl.cap, heads=heads) for _ in range(layers)]
    rng = np.random.default_rng(seed)
    worst = 0.0
    for n, f in enumerate(sched):
        f0 = wl.frame_idx(f.chunk)
        for layer in range(layers):
            # drawn again on the device (its generator is the driver's), independently of the
            # driver's own tensors
            q, k, v = (t.cpu() for t in W.gen_qkv(W.qkv_seed(seed, layer=layer, chunk=f.chunk,
                                                               forward=n), s, device="cuda"))
            q_rot = ols[layer].append(W.bits(q), W.bits(k), W.bits(v), f0, s.chunk_frames)
            if rows_per_forward is None:
                rows = [(b, l, h) for b in range(s.B) for h in heads for l in range(s.L)]
            else:
                ls = P.sample_rows(s.L, s.Tf, rows_per_forward, rng)
                rows = [(b, l, h) for b in range(s.B) for h in heads for l in ls]
            want = ols[layer].attend(q_rot, wl.window, rows)
            got = kept[n][layer].cpu().double().numpy()
            g = np.stack([got[b, l, h] for (b, l, h) in rows])
            e = P.attn_errors(g, want)
            assert e.max_abs <= P.MAX_ABS and e.mean_abs <= P.MEAN_ABS, (n, layer, e)
            worst = max(worst, e.max_abs)
    return worst


def test_clip_driver_forwards_match_the_oracle_small_layer():
    """Every one of the 23 forwards of every layer, all rows and heads, on a small layer that
    keeps the clip's schedule (seven chunks of three frames, W = 9, the Table 3 forward
    counts)."""
    small = W.LayerShape(B=1, H=2, D=64, Hg=6, Wg=8, d_t=24, d_h=20, d_w=20)
    wl = W.Workload("clip_small", small, cap=9, window=9, chunks=7, layers=2,
                    forwards_per_chunk=W.WORKLOADS["clip30"].forwards_per_chunk)
    _oracle_clip_check(wl, layers=2, seed=11, heads=[0, 1])


def test_clip_driver_forwards_match_the_oracle_wan_layer():
    """The Wan-shaped clip on two layers: head 5 of every forward of both layers, on sampled
    rows (tile and frame boundaries, the partial last tile, random rows)."""
    _oracle_clip_check(W.WORKLOADS["clip30"], layers=2, seed=12, heads=[5],
                       rows_per_forward=24)
