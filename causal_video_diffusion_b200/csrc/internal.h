// internal.h -- launch parameters of the RoPE/append, attention and renoise kernels, shared
// between the host API (api.cu) and those kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "limits.h"

namespace unstep {

// Division by a run-time invariant d by multiply-high (Granlund & Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, x / d = (umulhi(x, m) + x) >> l for 0 <= x < 2^31.
struct FastDiv {
  uint32_t d, m, l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  const uint64_t m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
  return FastDiv{d, static_cast<uint32_t>(m), l};
}

#ifdef __CUDACC__
// Index checks of the debug build (compiled with -DUNSTEP_DEBUG; empty otherwise): a failed
// check records UNSTEP_ERR_DEVICE_BOUNDS (-10) in the caller's error word, and the caller skips
// the access or winds the CTA down through its abort path.  Nothing ever traps.
#ifdef UNSTEP_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool debug_check(bool ok, int *dev_error) {
  if (kDebugChecks && !ok) {
    if (dev_error) atomicCAS(dev_error, 0, -10);
    return false;
  }
  return true;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t x, const FastDiv &f) {
  return (__umulhi(x, f.m) + x) >> f.l;
}

// One RoPE channel pair, two packed bf16 (a = low half, b = high half), rotated by (c, s):
// (a c - b s, a s + b c) in fp32, each rounded to bf16 (RNE).  The append kernel and the
// attention's query prologue both rotate through this function, so both give the same bits.
__device__ __forceinline__ uint32_t rope_rotate_pair(uint32_t w, float2 cs) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xFFFF0000u);
  const float ra = __fmaf_rn(a, cs.x, -__fmul_rn(b, cs.y));
  const float rb = __fmaf_rn(a, cs.y, __fmul_rn(b, cs.x));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(rb), "f"(ra));
  return r;
}
#endif

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
  // the shard's place in the activations [.][L][act_H][D]: stream b0 + b, head h0 + h
  int act_H, b0, h0;
  int sharded;    // 0: the activations are exactly [B][L][H][D]
  int Hg, Wg, Tf;
  int half_t, half_h, half_w;  // pairs per block
  int frame_idx, frames, cap;
  int rows;       // cap * Tf
  int act_B, max_pos_t;  // extents the debug build checks indices against
  int *dev_error;        // where the debug build records a failed check
  int slot0;      // frame_idx mod cap
  int rotate_q;   // 1: q rotated in place; 0: q neither read nor written
  FastDiv div_h;  // by H
  FastDiv div_l;  // by L
  FastDiv div_tf; // by Tf
  FastDiv div_wg; // by Wg
};

cudaError_t launch_rope_kv_append(const RopeAppendParams &p, cudaStream_t stream);

struct AttnParams {
  void *out;         // bf16 [act_B][L][act_H][D]; the shard's rows are written
  int *dev_error;
  int B, H, L;       // the shard: streams and heads of the cache
  int act_H, b0, h0; // its place in the activations: stream b0 + b, head h0 + h
  int act_B, rows;   // activation streams and cache rows per (stream, head): debug checks
  int n_pairs;       // units per (b, h): two 128-row query tiles each
  int n_units;       // B * H * n_pairs
  int n_tiles;       // key tiles of 128 rows over both ring segments
  int seg_row[2];
  int seg_len[2];
  int seg_tiles[2];
  float scale_log2;  // log2(e) / sqrt(D)
  uint64_t wait_limit_ns;
  // persistent schedule: dp_waves whole units per CTA, then the tail units
  // [u_tail0, n_units) cut into w_tail = (n_units - u_tail0) * n_tiles key tiles over g_sk CTAs
  int grid;
  int dp_waves;
  int u_tail0;
  int g_sk;
  long long w_tail;
  // scratch of split units: per-(unit, query tile) counts and two slots per CTA of
  // slot_floats floats each (per query tile: O[D][128], m[128], l[128])
  unsigned *counters;
  float *slots;
  int slot_floats;
  unsigned epoch;    // 1 .. 2^24-1, distinct for consecutive launches
  FastDiv div_pairs; // by n_pairs
  FastDiv div_heads; // by H
  // query RoPE in the prologue (rope_q != 0): q holds the chunk's un-rotated queries, chunk row
  // l being token (i, y, x) of frame frame0 + i, l = i*Tf + y*Wg + x
  int rope_q;
  const float2 *tab_t, *tab_h, *tab_w;  // as in RopeAppendParams
  int half_t, half_h, half_w;
  int Tf, Wg, frame0, frames;
  int tab_smem;      // 1: the chunk's rows fit in kQRopeTabBytes and are staged in shared memory
  FastDiv div_tf;    // by Tf
  FastDiv div_wg;    // by Wg
};

// Shared memory for the coefficient rows of the query rotation: frames*d_t/2 + Hg*d_h/2 +
// Wg*d_w/2 float2 (14.3 KB for a 3-frame 30x52 chunk at 44/42/42); larger chunks read the
// global tables instead.
constexpr int kQRopeTabBytes = 24 * 1024;

// Scratch layout shared by the host sizing and the kernel.
constexpr size_t attn_counter_bytes(long long max_units) {
  return ((static_cast<size_t>(max_units) * 2 * sizeof(unsigned) + 255) / 256) * 256;
}
constexpr size_t attn_slot_floats(int D) { return 2 * (static_cast<size_t>(D) * 128 + 256); }

// tmap_q: 4D (D, H, L, B) bf16, box (64, 1, 128, 1), 128B swizzle.
// tmap_k / tmap_v: 3D (D, cap*T_f, B*H) bf16, box (64, 128, 1), 128B swizzle.
cudaError_t launch_window_attn(int D, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                               const CUtensorMap &tmap_v, const AttnParams &p,
                               cudaStream_t stream);

cudaError_t launch_wait_timeout_selftest(int *dev_error, uint64_t limit_ns, cudaStream_t stream);

// out[i] = (1 - sigma) * x0[i] + sigma * eps[i], bf16, n elements.
cudaError_t launch_renoise(const void *x0, const void *eps, void *out, long long n, float sigma,
                           cudaStream_t stream);

// Size of the library's fixed device scratch buffer (see unstep_window_attn_noalloc).
constexpr size_t kStaticScratchBytes = 48ull << 20;

// Device address and size of that buffer on the current device; the first call on a device
// looks the address up (cudaGetSymbolAddress with the device current) and caches it.
cudaError_t static_attn_scratch(void **ptr, size_t *bytes);

cudaError_t launch_exp2_selftest(const float *x, float *y_poly, float *y_mufu, int n,
                                 cudaStream_t stream);

}  // namespace unstep
