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
