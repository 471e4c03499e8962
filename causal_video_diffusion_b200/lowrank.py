"""Weight preparation for the truncated-SVD projections (done once, on the host).

UnStep paper (arXiv 2609.32518), abstract and Figure 11 / Table 5: the DiT attention's value and
output projections are replaced by truncated SVDs keeping 92 % of their rank ("V/O rank
retention fixed at 0.92"; read here as a fraction of the singular values kept, so rank
floor(0.92 * 1536) = 1413 for the 1536-wide Wan projections).  A weight W [d_out][d_in] with
singular value decomposition W = U S V^T is kept as the two factors of its rank-r truncation,
  w1 = (V_r S_r)^T   [r][d_in]        w2 = U_r   [d_out][r],
so that x W_r^T = (x w1^T) w2^T, which ``binding.lowrank_linear`` evaluates on the tensor cores.
The rank is padded with zero factors to a multiple of 64 (128-byte rows of the rank-space
operands: the tensor-core GEMM reads them through 128-byte TMA rows, and a row pitch that is not a
multiple of 128 bytes makes every row straddle two L2 lines -- measured 22 % slower on the second
product); the product is unchanged, and at the Wan shape the padding adds no tile or K step.
"""
from __future__ import annotations

import math
from typing import Tuple

import torch

RANK_RETENTION = 0.92


def retained_rank(full_rank: int, retention: float = RANK_RETENTION) -> int:
    return int(math.floor(retention * full_rank))


def padded(rank: int, multiple: int = 64) -> int:
    return (rank + multiple - 1) // multiple * multiple


def svd_factors(W: torch.Tensor, rank: int, pad_to: int = 64) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 factors (w1 [r_pad][d_in], w2 [d_out][r_pad]) of the rank-`rank` truncation of W."""
    Wd = W.detach().to("cpu", torch.float64)
    U, S, Vh = torch.linalg.svd(Wd, full_matrices=False)
    r = int(rank)
    rp = padded(r, pad_to)
    d_out, d_in = Wd.shape
    w1 = torch.zeros((rp, d_in), dtype=torch.float64)
    w2 = torch.zeros((d_out, rp), dtype=torch.float64)
    w1[:r] = S[:r, None] * Vh[:r]
    w2[:, :r] = U[:, :r]
    return w1.to(torch.bfloat16), w2.to(torch.bfloat16)
