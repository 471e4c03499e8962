// renoise.cu -- x = (1 - sigma) * x0 + sigma * eps over a chunk's latent (bf16), one pass.
//
// UnStep paper (arXiv 2609.32518), abstract: the generated latent frames are renoised to a
// near-clean level before the existing clean-cache pass refines them (Table 4 / Table 5: the
// clean-cache level sigma* = 0.02 for UnStep, 0 for Self Forcing); a few-step student moves
// between its denoising steps the same way, re-noising its clean prediction to the next step's
// noise level.  Flow-matching interpolation between data and noise, elementwise, HBM-bound:
// each thread moves 16-byte vectors of x0 and eps, computes in fp32 (one fma) and rounds to bf16.
#include <cuda_bf16.h>

#include "internal.h"

namespace unstep {
namespace {

__global__ void __launch_bounds__(256) renoise_kernel(const __nv_bfloat16 *x0,
                                                      const __nv_bfloat16 *eps,
                                                      __nv_bfloat16 *out, long long n,
                                                      float sigma) {
  const float keep = 1.f - sigma;
  const long long n8 = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long v = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; v < n8;
       v += stride) {
    const uint4 a = reinterpret_cast<const uint4 *>(x0)[v];
    const uint4 e = reinterpret_cast<const uint4 *>(eps)[v];
    const uint32_t *pa = &a.x;
    const uint32_t *pe = &e.x;
    uint4 o;
    uint32_t *po = &o.x;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float a0 = __uint_as_float(pa[w] << 16), a1 = __uint_as_float(pa[w] & 0xFFFF0000u);
      const float e0 = __uint_as_float(pe[w] << 16), e1 = __uint_as_float(pe[w] & 0xFFFF0000u);
      __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(sigma, e0, keep * a0), fmaf(sigma, e1, keep * a1));
      po[w] = *reinterpret_cast<uint32_t *>(&r);
    }
    reinterpret_cast<uint4 *>(out)[v] = o;
  }
  // tail (n not a multiple of 8)
  const long long t = n8 * 8 + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blockIdx.x == 0 && t < n) {
    const float a = __bfloat162float(x0[t]), e = __bfloat162float(eps[t]);
    out[t] = __float2bfloat16_rn(fmaf(sigma, e, keep * a));
  }
}

}  // namespace

cudaError_t launch_renoise(const void *x0, const void *eps, void *out, long long n, float sigma,
                           cudaStream_t stream) {
  const long long n8 = n / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148 * 16) blocks = 148 * 16;
  renoise_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16 *>(x0), static_cast<const __nv_bfloat16 *>(eps),
      static_cast<__nv_bfloat16 *>(out), n, sigma);
  return cudaGetLastError();
}

}  // namespace unstep
