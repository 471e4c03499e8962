// conv3d.h -- launch parameters of the causal 3D convolution, shared between the host API
// (api.cu) and the kernel (conv3d.cu).
#pragma once

#include <cstddef>
#include <cuda.h>
#include <cuda_runtime.h>

#include "limits.h"

namespace unstep {

// Causal 3x3x3 convolution (channels-last implicit GEMM); see unstep_conv3d_causal.
struct ConvParams {
  void *y;            // bf16 [B][T][H][W][C_out]
  const float *bias;  // [C_out] or null
  int *dev_error;
  uint64_t wait_limit_ns;
  int B, T, H, W, C_in, C_out;
  int tiles_h, tiles_w;   // output tiles of kConvTileH rows x 16 columns per frame (the
                          // launcher recounts tiles_h and m_tiles in 32-row tiles for pairs)
  int m_tiles, n_tiles;   // B*T*tiles_h*tiles_w position tiles; ceil(C_out / 128) channel tiles
  // stream-K tail (g_sk = 0: none, every tile whole).  Tiles [0, tail0) are taken whole, tile
  // w*grid + c by CTA c; the K steps of tiles [tail0, m_tiles*n_tiles) are cut evenly over
  // g_sk CTAs, w_tail steps in all.
  int tail0, g_sk;
  long long w_tail;
  unsigned *counters;     // one word per tail tile: epoch << 8 | pieces counted
  float *slots;           // 2 g_sk slots of kConvSlotFloats fp32 partial sums
  unsigned epoch;         // 1 .. 2^24 - 1, different for each launch
};

// Rows of a convolution output tile (two 8 x 16 halves of 128 positions).
constexpr int kConvTileH = 16;
// Whether a frame of H rows runs on CTA pairs (tiles of 32 rows; with H <= 16 the second CTA
// would only read padding, and one CTA per tile runs instead).
constexpr bool conv_uses_pair(int H) { return H > kConvTileH; }
// Output channels of the weight TMA box: each CTA of a pair loads half of every slice.
constexpr int conv_weight_box_n(int H) { return conv_uses_pair(H) ? 64 : 128; }
// One partial output tile of the conv's stream-K tail: 2 x 128 positions x 128 channels, fp32.
constexpr long long kConvSlotFloats = 2 * 128ll * 128;
// Bytes of the conv's stream-K scratch for a device with `sms` SMs: one counter per tail tile
// (fewer tail tiles than SMs), 256-byte aligned, then 2 slots per SM.
constexpr size_t conv_counter_bytes(int sms) {
  return (static_cast<size_t>(sms) * 4 + 255) / 256 * 256;
}
constexpr size_t conv_scratch_bytes(int sms) {
  return conv_counter_bytes(sms) + static_cast<size_t>(2) * sms * kConvSlotFloats * 4;
}

// tmx: 4D (C_in, W, H, B*(T+2)) bf16, box (64, 16, kConvTileH + 2, 1); tmw: 3D (C_in, 27, C_out)
// bf16, box (64, 1, conv_weight_box_n(H)); both 128B swizzle.
cudaError_t launch_conv3d_causal(const CUtensorMap &tmx, const CUtensorMap &tmw,
                                 const ConvParams &p, cudaStream_t stream);

}  // namespace unstep
