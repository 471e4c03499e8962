// internal.h -- launch parameters shared between the host API (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace unstep {

// Default limit of every device-side wait: no legitimate wait of these kernels lasts this long.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct RopeAppendParams {
  const void *k;
  const void *v;
  void *q;
  void *k_cache;
  void *v_cache;
  int *slot_frame;
  const float2 *tab_t;  // [max_pos_t][d_t/2]
  const float2 *tab_h;  // [Hg][d_h/2]
  const float2 *tab_w;  // [Wg][d_w/2]
  int B, L, H, D;
  int Hg, Wg, Tf;
  int half_t, half_h, half_w;  // pairs per block
  int frame_idx, frames, cap;
  int rows;  // cap * Tf
};

cudaError_t launch_rope_kv_append(const RopeAppendParams &p, cudaStream_t stream);

struct AttnParams {
  void *out;         // bf16 [B][L][H][D]
  int *dev_error;
  int B, H, L;
  int n_pairs;       // CTAs per (b, h): two 128-row query tiles each
  int n_tiles;       // key tiles of 128 rows over both ring segments
  int seg_row[2];
  int seg_len[2];
  int seg_tiles[2];
  float scale_log2;  // log2(e) / sqrt(D)
  uint64_t wait_limit_ns;
};

// tmap_q: 4D (D, H, L, B) bf16, box (64, 1, 128, 1), 128B swizzle.
// tmap_k / tmap_v: 3D (D, cap*T_f, B*H) bf16, box (64, 128, 1), 128B swizzle.
cudaError_t launch_window_attn(int D, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                               const CUtensorMap &tmap_v, const AttnParams &p,
                               cudaStream_t stream);

cudaError_t launch_wait_timeout_selftest(int *dev_error, uint64_t limit_ns, cudaStream_t stream);

cudaError_t launch_exp2_selftest(const float *x, float *y_poly, float *y_mufu, int n,
                                 cudaStream_t stream);

}  // namespace unstep
