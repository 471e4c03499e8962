"""The tensor-core GEMM and the truncated-SVD projections against the fp64 oracle (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from causal_video_diffusion_b200 import binding
from causal_video_diffusion_b200 import lowrank
from causal_video_diffusion_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _rel_errors(got, want):
    d = np.abs(got - want)
    rms = float(np.sqrt(np.mean(want ** 2))) or 1.0
    return float(d.max()) / rms, float(d.mean()) / rms


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 8, 8), (300, 136, 1416), (4680, 1416, 1536),
                                   (257, 520, 72), (129, 264, 200),
                                   # 3-4 tiles per persistent pair / CTA: both accumulator sets
                                   # of each go through both barrier phases
                                   (4096, 4096, 128), (65536, 200, 64),
                                   # CTA pairs with K ending inside a 128- and a 192-deep step
                                   (512, 512, 200), (300, 264, 1416),
                                   # exactly one pair tile; K shorter than one 64-deep step
                                   (256, 256, 64), (256, 256, 8)])
def test_gemm_matches_oracle(M, N, K):
    a = W.gen_act(M * 7 + 1, M, K)
    b = W.gen_act(N * 11 + 2, N, K)
    got = binding.gemm_bf16(a.cuda(), b.cuda()).cpu().double().numpy()
    want = oracle.matmul_bt(W.bits(a), W.bits(b))
    # bound from the arithmetic: the bf16 output is within half an ulp of the fp32 sum, and the
    # fp32 sum of K products is within K * 2^-24 * sum_k |a_k b_k| of the exact one (generous:
    # the tensor core's accumulation order is unspecified)
    absab = np.abs(oracle.bf16_to_f64(W.bits(a))) @ np.abs(oracle.bf16_to_f64(W.bits(b))).T
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
    bound = 0.5 * ulp * 2 + K * 2.0 ** -24 * absab + 1e-30
    assert np.all(np.abs(got - want) <= bound), (M, N, K, float(np.max(np.abs(got - want) / bound)))
    mx, mean = _rel_errors(got, want)
    assert mx < 3e-2 and mean < 2e-3


def test_lowrank_projection_wan_shape():
    """V projection of the Wan layer through its rank-1413 (stored padded to 1472) factors, 4680
    tokens."""
    d, M = W.MODEL_DIM, 4680
    r = lowrank.retained_rank(d)
    Wt = W.gen_weight(21, d, d)
    w1, w2 = lowrank.svd_factors(Wt, r)
    x = W.gen_act(22, M, d)
    y = binding.lowrank_linear(x.cuda(), w1.cuda(), w2.cuda()).cpu().double().numpy()
    want_t = oracle.lowrank_linear(W.bits(x), W.bits(w1), W.bits(w2), round_t=True)
    mx, mean = _rel_errors(y, want_t)
    assert mx < 2e-2 and mean < 3e-3, (mx, mean)
    want = oracle.lowrank_linear(W.bits(x), W.bits(w1), W.bits(w2))
    mx, mean = _rel_errors(y, want)
    assert mx < 3e-2 and mean < 4e-3, (mx, mean)


def test_full_rank_factors_reproduce_the_linear_layer():
    d, M = 256, 300
    Wt = W.gen_weight(5, d, d)
    w1, w2 = lowrank.svd_factors(Wt, d)
    x = W.gen_act(6, M, d)
    y = binding.lowrank_linear(x.cuda(), w1.cuda(), w2.cuda()).cpu().double().numpy()
    full = x.double().numpy() @ Wt.double().numpy().T
    mx, mean = _rel_errors(y, full)
    assert mx < 5e-2 and mean < 1e-2, (mx, mean)   # bf16 factors and intermediate


def test_gemm_deterministic_and_no_device_error():
    a = W.gen_act(1, 1000, 512).cuda()
    b = W.gen_act(2, 768, 512).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    c1 = binding.gemm_bf16(a, b, dev_error=err)
    c2 = binding.gemm_bf16(a, b, dev_error=err)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    assert int(err.item()) == 0


def test_back_to_back_products_equal_serialised_ones():
    """Pair-GEMM launches overlap their set-up with the preceding launch (programmatic dependent
    launch): a chain in which every product reads the previous one's output (read after write)
    and overwrites a buffer the previous one read (write after read), issued back to back on one
    stream, must give the bits of the same chain with the device synchronised between calls."""
    M, d, r = 4680, 1536, 1472
    x = W.gen_act(31, M, d).cuda()
    w = [W.gen_act(32 + i, r if i % 2 == 0 else d, d if i % 2 == 0 else r).cuda()
         for i in range(4)]

    def chain(sync):
        t = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        z = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
        for _ in range(3):  # junk in every buffer, so that a read before the write shows
            t.fill_(7.0); y.fill_(-3.0); z.fill_(5.0)
            torch.cuda.synchronize()
        binding.gemm_bf16(x, w[0], t)          # t = x w0^T
        if sync: torch.cuda.synchronize()
        binding.gemm_bf16(t, w[1], y)          # y = t w1^T          (reads t)
        if sync: torch.cuda.synchronize()
        binding.gemm_bf16(y, w[2], t)          # t = y w2^T          (overwrites what the last read)
        if sync: torch.cuda.synchronize()
        binding.gemm_bf16(t, w[3], z)          # z = t w3^T
        if sync: torch.cuda.synchronize()
        binding.gemm_bf16(z, w[2], t)          # t = z w2^T
        torch.cuda.synchronize()
        return [W.bits(v.cpu()) for v in (t, y, z)]

    want = chain(True)
    for _ in range(3):
        got = chain(False)
        for g, e in zip(got, want):
            assert np.array_equal(g, e)
    # and the chain's first product is the oracle's
    t0 = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    binding.gemm_bf16(x, w[0], t0)
    rows = np.arange(0, M, 97)
    want0 = oracle.matmul_bt(W.bits(x.cpu())[rows], W.bits(w[0].cpu()))
    mx, mean = _rel_errors(t0.cpu()[rows].double().numpy(), want0)
    assert mx < 3e-2 and mean < 2e-3


@pytest.mark.parametrize("M,N,K,extra", [(300, 264, 200, 64), (4680, 1472, 1536, 8), (257, 520, 72, 24)])
def test_gemm_into_a_wider_output_leaves_the_rest_alone(M, N, K, extra):
    """unstep_gemm_bf16 with ldc > N (C a column block of a wider matrix): the N columns are the
    product, bit for bit what ldc = N gives, and the columns N .. ldc - 1 keep their values."""
    import ctypes
    a = W.gen_act(M + 41, M, K).cuda()
    b = W.gen_act(N + 43, N, K).cuda()
    want = binding.gemm_bf16(a, b)
    ldc = N + extra
    big = torch.full((M, ldc), 3.0, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = binding.lib().unstep_gemm_bf16(
        ctypes.c_void_p(a.data_ptr()), K, ctypes.c_void_p(b.data_ptr()), K,
        ctypes.c_void_p(big.data_ptr()), ldc, M, N, K, ctypes.c_void_p(err.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and int(err.item()) == 0
    assert torch.equal(big[:, :N], want)
    assert bool((big[:, N:] == 3.0).all())
