// gemm.h -- launch functions of the bf16 projection GEMMs, shared between the host API (api.cu)
// and the kernels (lowrank_gemm.cu, gemm2sm.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "limits.h"

namespace unstep {

// C[M][N] (ldc) = A[M][K] * B[N][K]^T, bf16, fp32 accumulation; tma: 2D (K, M) box (64, 128),
// tmb: 2D (K, N) box (64, 128), both 128B swizzle.
cudaError_t launch_gemm_bf16_tn(const CUtensorMap &ta, const CUtensorMap &tb, void *c, int M,
                                int N, int K, int ldc, int *dev_error, cudaStream_t stream);

// The same product on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 tiles); same A and B
// tensor maps, and C through tmc: 2D (N, M) box (64, 32), 128B swizzle (row stride ldc * 2).
cudaError_t launch_gemm2sm_bf16_tn(const CUtensorMap &ta, const CUtensorMap &tb,
                                   const CUtensorMap &tc, int M, int N, int K, int *dev_error,
                                   cudaStream_t stream);

}  // namespace unstep
