"""The causal 3D convolution kernel against the fp64 oracle, through the C ABI (needs a B200).

Shapes span several position and channel tiles with ragged edges (frames not a multiple of the
8 x 16 tile, C_out not a multiple of 128, a frame smaller than one tile), several 64-channel
blocks, B > 1; the decoder-shaped layer (384 -> 384 channels on the 60 x 104 latent, a 3-frame
chunk with its 2 history frames) is checked on sampled rows, each from an exact slice.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, Wd, Ci, Co, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, T + 2, H, Wd, Ci), generator=g).to(torch.bfloat16)
    # weights at the scale that keeps outputs O(1): 1/sqrt(27 C_in)
    w = (torch.randn((Co, 3, 3, 3, Ci), generator=g) / np.sqrt(27 * Ci)).to(torch.bfloat16)
    bias = torch.randn((Co,), generator=g, dtype=torch.float32) * 0.1
    return x, w, bias


def _check(got, x_bits, w_bits, bias, want, row=None):
    # the bf16 output is within one ulp of the fp32 result (rounding, binade edges), and the
    # fp32 sum of K = 27 C_in products is within K 2^-24 sum |x w| of the exact one
    K = 27 * x_bits.shape[-1]
    absxw = oracle.conv3d_causal(oracle.f64_to_bf16(np.abs(oracle.bf16_to_f64(x_bits))),
                                 oracle.f64_to_bf16(np.abs(oracle.bf16_to_f64(w_bits))))
    if row is not None:
        absxw = absxw[:, :, row]
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
    bound = ulp + K * 2.0 ** -24 * (absxw + np.abs(bias)) + 1e-30
    d = np.abs(got - want)
    assert np.all(d <= bound), float(np.max(d / bound))
    rms = float(np.sqrt(np.mean(want ** 2)))
    assert d.max() / rms < 3e-2 and d.mean() / rms < 3e-3


@pytest.mark.parametrize("B,T,H,Wd,Ci,Co", [
    (1, 3, 13, 21, 64, 128),    # ragged position tiles (13 = 8 + 5 rows, 21 = 16 + 5 columns)
    (2, 2, 8, 16, 128, 200),    # exactly one position tile per frame, C_out = 128 + 72
    (1, 1, 5, 7, 192, 64),      # a frame smaller than one tile, 3 channel blocks, C_out < 128
    (1, 2, 17, 33, 64, 264),    # 3 x 3 tiles with 1-wide tails, 3 channel tiles (one of 8)
    (1, 9, 60, 104, 64, 256),   # 504 tiles: 3-4 per persistent CTA, both accumulator sets
                                # through both barrier phases
])
def test_conv_matches_oracle(B, T, H, Wd, Ci, Co):
    x, w, bias = _inputs(B, T, H, Wd, Ci, Co, seed=B * 1000 + H * 10 + Co)
    got = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda()).cpu().double().numpy()
    want = oracle.conv3d_causal(W.bits(x), W.bits(w), bias.double().numpy())
    _check(got, W.bits(x), W.bits(w), bias.double().numpy(), want)


def test_conv_without_bias_and_delta_kernel_is_exact():
    """A delta kernel (the output frame's own pixel, channel to channel) copies bf16 exactly."""
    B, T, H, Wd, C = 1, 3, 11, 19, 64
    x, _, _ = _inputs(B, T, H, Wd, C, C, seed=77)
    w = torch.zeros((C, 3, 3, 3, C), dtype=torch.bfloat16)
    w[torch.arange(C), 2, 1, 1, torch.arange(C)] = 1.0
    got = binding.conv3d_causal(x.cuda(), w.cuda()).cpu()
    assert torch.equal(got.view(torch.int16), x[:, 2:].contiguous().view(torch.int16))


def test_decoder_shaped_layer_on_sampled_rows():
    B, T, H, Wd, C = 1, 3, 60, 104, 384
    x, w, bias = _inputs(B, T, H, Wd, C, C, seed=5)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda(), dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = got.cpu().double().numpy()
    xb, wb, bb = W.bits(x), W.bits(w), bias.double().numpy()
    for h in (0, 7, 8, 31, 59):      # borders and tile edges
        lo, hi = max(0, h - 1), min(H, h + 2)
        # the rows h-1 .. h+1 of the input produce row h exactly (zero padding beyond the frame
        # is also the slice's padding at the true borders)
        want = oracle.conv3d_causal(xb[:, :, lo:hi], wb, bb)[:, :, h - lo]
        _check(got[:, :, h], xb[:, :, lo:hi], wb, bb, want, row=h - lo)
