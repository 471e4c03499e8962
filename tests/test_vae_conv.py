"""Causal 3D convolution of the VAE decoder: the oracle's pins (CPU only).

The oracle (oracle.conv3d_causal) is pinned to things other than itself: nested loops that
spell the definition out element by element, torch's fp64 conv3d (a library routine the causal
convolution reduces to once the history frames are part of the input), a delta kernel, the
exact set of outputs one input frame can reach, and a constant-input closed form at interior
and border positions.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import workloads as W


def _rand_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return W.bits((torch.randn(shape, generator=g) * scale).to(torch.bfloat16))


def test_against_loops_on_a_tiny_case():
    B, T, H, Wd, Ci, Co = 2, 2, 3, 4, 3, 5
    x = _rand_bits((B, T + 2, H, Wd, Ci), 1)
    w = _rand_bits((Co, 3, 3, 3, Ci), 2)
    bias = np.random.default_rng(3).normal(size=Co)
    y = oracle.conv3d_causal(x, w, bias)
    xf, wf = oracle.bf16_to_f64(x), oracle.bf16_to_f64(w)
    ref = np.zeros((B, T, H, Wd, Co))
    for b, t, h, xx, o in itertools.product(range(B), range(T), range(H), range(Wd), range(Co)):
        acc = bias[o]
        for dt, dy, dx, c in itertools.product(range(3), range(3), range(3), range(Ci)):
            hh, ww = h + dy - 1, xx + dx - 1
            if 0 <= hh < H and 0 <= ww < Wd:
                acc += wf[o, dt, dy, dx, c] * xf[b, t + dt, hh, ww, c]
        ref[b, t, h, xx, o] = acc
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_against_torch_conv3d():
    B, T, H, Wd, Ci, Co = 1, 3, 7, 6, 8, 4
    x = _rand_bits((B, T + 2, H, Wd, Ci), 4)
    w = _rand_bits((Co, 3, 3, 3, Ci), 5)
    y = oracle.conv3d_causal(x, w)
    xt = torch.from_numpy(oracle.bf16_to_f64(x)).permute(0, 4, 1, 2, 3)      # [B][Ci][T+2][H][W]
    wt = torch.from_numpy(oracle.bf16_to_f64(w)).permute(0, 4, 1, 2, 3)      # [Co][Ci][3][3][3]
    ref = torch.nn.functional.conv3d(xt, wt, padding=(0, 1, 1)).permute(0, 2, 3, 4, 1).numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-10)


def test_delta_kernel_passes_the_current_frame():
    B, T, H, Wd, C = 1, 3, 5, 4, 6
    x = _rand_bits((B, T + 2, H, Wd, C), 6)
    w = np.zeros((C, 3, 3, 3, C))
    w[np.arange(C), 2, 1, 1, np.arange(C)] = 1.0        # dt = 2 is the output's own frame
    y = oracle.conv3d_causal(x, oracle.f64_to_bf16(w))
    np.testing.assert_array_equal(y, oracle.bf16_to_f64(x)[:, 2:])


def test_an_input_frame_reaches_only_its_own_and_the_next_two_outputs():
    B, T, H, Wd, C = 1, 5, 4, 4, 3
    x = _rand_bits((B, T + 2, H, Wd, C), 7)
    w = _rand_bits((2, 3, 3, 3, C), 8)
    y0 = oracle.conv3d_causal(x, w)
    for f in range(T + 2):
        xf = oracle.bf16_to_f64(x).copy()
        xf[:, f] += 1.0
        y1 = oracle.conv3d_causal(oracle.f64_to_bf16(xf), w)
        changed = [t for t in range(T) if not np.array_equal(y0[:, t], y1[:, t])]
        # input frame f is frame f - 2 of the chunk: it feeds outputs f - 2 .. f
        assert changed == [t for t in range(T) if f - 2 <= t <= f], (f, changed)


def test_constant_input_closed_form():
    B, T, H, Wd, Ci, Co = 1, 2, 4, 5, 3, 2
    x = oracle.f64_to_bf16(np.ones((B, T + 2, H, Wd, Ci)))
    w = _rand_bits((Co, 3, 3, 3, Ci), 9)
    wf = oracle.bf16_to_f64(w)
    y = oracle.conv3d_causal(x, w)
    # interior: every tap reads 1; top-left corner: only the taps with dy, dx >= 1 read inside
    np.testing.assert_allclose(y[0, :, 1:-1, 1:-1], np.broadcast_to(wf.sum(axis=(1, 2, 3, 4)),
                                                                    y[0, :, 1:-1, 1:-1].shape),
                               rtol=1e-12)
    np.testing.assert_allclose(y[0, :, 0, 0], np.broadcast_to(wf[:, :, 1:, 1:].sum(axis=(1, 2, 3, 4)),
                                                              y[0, :, 0, 0].shape), rtol=1e-12)
    np.testing.assert_allclose(y[0, :, -1, -1],
                               np.broadcast_to(wf[:, :, :2, :2].sum(axis=(1, 2, 3, 4)),
                                               y[0, :, -1, -1].shape), rtol=1e-12)


def test_conv_arguments_rejected_on_the_host():
    """Every failing call returns before any launch (no GPU needed)."""
    import ctypes
    from causal_video_diffusion_b200 import binding as B
    L = B.lib()
    p = ctypes.c_void_p(0x700000)
    odd = ctypes.c_void_p(0x700008)
    err = ctypes.c_void_p(0x710000)
    ok_args = (1, 3, 8, 16, 64, 128)
    f = L.unstep_conv3d_causal
    assert f(None, p, None, p, *ok_args, None, 0, err, None) == B.UNSTEP_ERR_ARG
    assert f(p, p, None, p, *ok_args, None, 0, None, None) == B.UNSTEP_ERR_ARG
    assert f(p, p, None, p, 1, 0, 8, 16, 64, 128, None, 0, err, None) == B.UNSTEP_ERR_ARG
    assert f(odd, p, None, p, *ok_args, None, 0, err, None) == B.UNSTEP_ERR_ALIGN
    assert f(p, p, ctypes.c_void_p(0x700002), p, *ok_args, None, 0, err, None) == B.UNSTEP_ERR_ALIGN
    assert f(p, p, None, p, *ok_args, odd, 1 << 30, err, None) == B.UNSTEP_ERR_ALIGN
    assert f(p, p, None, p, 1, 3, 8, 16, 48, 128, None, 0, err, None) == B.UNSTEP_ERR_UNSUPPORTED
    assert f(p, p, None, p, 1, 3, 8, 16, 64, 100, None, 0, err, None) == B.UNSTEP_ERR_UNSUPPORTED
