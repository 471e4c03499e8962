"""Truncated-SVD projections: the oracle's pins and the host-side checks (CPU only)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import binding as B
from causal_video_diffusion_b200 import lowrank
from causal_video_diffusion_b200 import workloads as W


def test_rank_reading_of_the_pages():
    # Figure 11 / Table 5: V/O rank retention fixed at 0.92 of the 1536-wide projections
    assert lowrank.retained_rank(1536) == 1413
    assert lowrank.padded(1413) == 1472    # zero factors up to 128-byte rows
    assert lowrank.padded(1413, 8) == 1416


def test_eckart_young_error_of_the_truncation():
    """||W - W_r||_F^2 equals the sum of the discarded squared singular values (closed form)."""
    Wm = np.random.default_rng(1).normal(size=(96, 80))
    for r in (1, 17, 73, 80):
        w1, w2, S = oracle.svd_truncate(Wm, r)
        err = np.sum((Wm - w2 @ w1) ** 2)
        assert err == pytest.approx(np.sum(S[r:] ** 2), rel=1e-9, abs=1e-18)
    w1, w2, _ = oracle.svd_truncate(Wm, 80)
    np.testing.assert_allclose(w2 @ w1, Wm, rtol=0, atol=1e-12)


def test_matmul_against_loops():
    rng = np.random.default_rng(2)
    a = oracle.f64_to_bf16(rng.normal(size=(5, 7)))
    b = oracle.f64_to_bf16(rng.normal(size=(3, 7)))
    got = oracle.matmul_bt(a, b)
    A, Bm = oracle.bf16_to_f64(a), oracle.bf16_to_f64(b)
    for i in range(5):
        for j in range(3):
            assert got[i, j] == pytest.approx(sum(A[i, k] * Bm[j, k] for k in range(7)), abs=1e-13)


def test_product_factors_match_the_oracle_truncation():
    """The product helper's bf16 factors reproduce the oracle's rank-r weight (up to bf16)."""
    Wt = W.gen_weight(3, 64, 48)
    w1, w2 = lowrank.svd_factors(Wt, 40, pad_to=8)
    assert w1.shape == (40, 48) and w2.shape == (64, 40)
    o1, o2, _ = oracle.svd_truncate(Wt.double().numpy(), 40)
    prod = w2.double().numpy() @ w1.double().numpy()
    ref = o2 @ o1
    assert np.max(np.abs(prod - ref)) < 2e-2 * np.max(np.abs(ref))
    # padding (to a multiple of 8 here, of 64 by default) adds zero factors only
    p1, p2 = lowrank.svd_factors(Wt, 37, pad_to=8)
    assert p1.shape == (40, 48) and torch.all(p1[37:] == 0) and torch.all(p2[:, 37:] == 0)
    d1, d2 = lowrank.svd_factors(Wt, 37)
    assert d1.shape == (64, 48) and d2.shape == (64, 64)
    assert torch.equal(d1[:40], p1) and torch.all(d1[40:] == 0) and torch.equal(d2[:, :40], p2)


def test_gemm_arguments_rejected_on_the_host():
    B_ = B.lib()
    fake = ctypes.c_void_p(0x700000)
    err = ctypes.c_void_p(0x800000)
    assert B_.unstep_gemm_bf16(None, 64, fake, 64, fake, 64, 8, 8, 64, err, None) == B.UNSTEP_ERR_ARG
    assert B_.unstep_gemm_bf16(fake, 64, fake, 64, fake, 12, 8, 12, 64, err, None) == B.UNSTEP_ERR_SHAPE
    assert B_.unstep_gemm_bf16(fake, 60, fake, 60, fake, 64, 8, 8, 60, err, None) == B.UNSTEP_ERR_SHAPE
    assert B_.unstep_gemm_bf16(fake, 64, fake, 64, fake, 64, 0, 8, 64, err, None) == B.UNSTEP_ERR_SHAPE
    assert B_.unstep_gemm_bf16(ctypes.c_void_p(0x700002), 64, fake, 64, fake, 64, 8, 8, 64, err,
                               None) == B.UNSTEP_ERR_ALIGN
    assert B_.unstep_lowrank_linear(fake, fake, fake, fake, fake, 8, 64, 1413, 64, err,
                                    None) == B.UNSTEP_ERR_SHAPE
