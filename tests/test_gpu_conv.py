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


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _counters_zero(scratch):
    # every tail tile's count word is reset by the piece that merged it
    return int(scratch[:4 * _sms()].view(torch.int32).abs().sum().item()) == 0


@pytest.mark.parametrize("extra,Ci,Co", [
    (1, 256, 128),    # one 36-step tail tile cut into 2 pieces of 18 steps
    (37, 256, 128),   # 37 tail tiles over 83 CTAs: 16-step shares, 2-3 pieces per tile
    (130, 128, 128),  # most of a wave: 18-step tiles over 146 CTAs, 1-2 pieces per tile
    (30, 64, 128),    # 9-step tiles are too short to split: the scratch is left unused
])
def test_stream_k_tail_matches_oracle(extra, Ci, Co):
    """Frames of one 16 x 16 tile each, SMs + extra tiles: the first wave runs whole, the extra
    tiles are cut along K over the SMs (shares of at least 16 K steps of three 64-channel taps)
    and merged by the last piece to finish."""
    B, T, H, Wd = 1, _sms() + extra, 16, 16
    x, w, bias = _inputs(B, T, H, Wd, Ci, Co, seed=extra + Ci)
    scratch = binding.conv3d_scratch()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda(), dev_error=err, scratch=scratch)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert _counters_zero(scratch)
    xb, wb, bb = W.bits(x), W.bits(w), bias.double().numpy()
    # the whole first wave and the tail: frames 0..3 and the last 2 + extra frames
    for t0, t1 in ((0, 4), (T - extra - 2, T)):
        want = oracle.conv3d_causal(xb[:, t0:t1 + 2], wb, bb)
        _check(got[:, t0:t1].cpu().double().numpy(), xb[:, t0:t1 + 2], wb, bb, want)
    # the split tiles differ from whole ones only in the fp32 summation order
    whole = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda())
    d = (got.float() - whole.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * float(whole.float().abs().max())


@pytest.mark.parametrize("shape", [
    (1, 9, 60, 104, 128, 256),  # 504 tiles: 3 whole waves, 60 tail tiles over 67 CTAs
    (1, 3, 60, 104, 384, 384),  # the decoder layer: 1 whole wave, 104 tail tiles in 2-3 pieces
])
def test_stream_k_layers_on_sampled_rows_and_repeat_calls(shape):
    """Layer shapes with scratch: sampled rows against the oracle, the same bits on a second
    call with the same scratch (the counters' epochs keep launches apart)."""
    B, T, H, Wd, Ci, Co = shape
    x, w, bias = _inputs(B, T, H, Wd, Ci, Co, seed=Ci + Co)
    scratch = binding.conv3d_scratch()
    xc, wc, bc = x.cuda(), w.cuda(), bias.cuda()
    got = binding.conv3d_causal(xc, wc, bc, scratch=scratch)
    again = binding.conv3d_causal(xc, wc, bc, scratch=scratch)
    torch.cuda.synchronize()
    assert _counters_zero(scratch)
    assert torch.equal(got.view(torch.int16), again.view(torch.int16))
    got = got.cpu().double().numpy()
    xb, wb, bb = W.bits(x), W.bits(w), bias.double().numpy()
    for t in (0, T - 1):
        for h in (0, 15, 16, 59):
            lo, hi = max(0, h - 1), min(H, h + 2)
            want = oracle.conv3d_causal(xb[:, t:t + 3, lo:hi], wb, bb)[:, :, h - lo]
            _check(got[:, t:t + 1, h], xb[:, t:t + 3, lo:hi], wb, bb, want, row=h - lo)


def test_stream_k_scratch_too_small_is_rejected():
    x, w, bias = _inputs(1, _sms() + 3, 16, 16, 64, 128, seed=3)
    small = torch.zeros(binding.lib().unstep_conv3d_scratch_bytes() - 16, dtype=torch.uint8,
                        device="cuda")
    with pytest.raises(binding.UnstepError):
        binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda(), scratch=small)


def test_stream_k_with_ragged_tiles_and_two_streams():
    """Split tiles at the ragged edges: 13 x 21 frames (8 + 5 rows of a 16-row tile, 16 + 5
    columns), C_out = 200 (a 72-channel tile), B = 2; the tail is cut over the SMs."""
    B, H, Wd, Ci, Co = 2, 13, 21, 256, 200
    # 2 position tiles per frame x 2 channel tiles; frames per stream so that the tile count is
    # SMs + 40 (rounded up to whole frames of both streams)
    T = -(-(_sms() + 40) // (B * 2 * 2))
    x, w, bias = _inputs(B, T, H, Wd, Ci, Co, seed=13)
    scratch = binding.conv3d_scratch()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda(), dev_error=err, scratch=scratch)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert _counters_zero(scratch)
    xb, wb, bb = W.bits(x), W.bits(w), bias.double().numpy()
    want = oracle.conv3d_causal(xb, wb, bb)
    _check(got.cpu().double().numpy(), xb, wb, bb, want)


def test_pair_tiles_with_stream_k_at_ragged_edges():
    """Frames taller than one tile run on CTA pairs (32-row tiles, each CTA 16 rows and half of
    every weight slice).  H = 40: the second pair row has 8 live rows in its first CTA and none
    in its second; W = 21 (16 + 5 columns), C_out = 200 (a 72-channel tile, so the second CTA's
    weight half is partly and then wholly past C_out), B = 2, and tiles beyond the last whole wave
    of pairs cut along K, against the full oracle."""
    B, H, Wd, Ci, Co = 2, 40, 21, 128, 200
    pairs = _sms() // 2
    # 2 pair rows x 2 column tiles x 2 channel tiles per frame; about 30 tail tiles
    T = -(-(pairs + 30) // (B * 8))
    x, w, bias = _inputs(B, T, H, Wd, Ci, Co, seed=40)
    scratch = binding.conv3d_scratch()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda(), dev_error=err, scratch=scratch)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert _counters_zero(scratch)
    xb, wb, bb = W.bits(x), W.bits(w), bias.double().numpy()
    want = oracle.conv3d_causal(xb, wb, bb)
    _check(got.cpu().double().numpy(), xb, wb, bb, want)
    whole = binding.conv3d_causal(x.cuda(), w.cuda(), bias.cuda())
    d = (got.float() - whole.float()).abs()
    assert float(d.max()) <= 2.0 ** -6 * float(whole.float().abs().max())
