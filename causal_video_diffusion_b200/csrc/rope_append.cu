// rope_append.cu -- fused 3D RoPE + ring-buffer KV-cache append (one launch per chunk).
//
// UnStep paper (arXiv 2609.32518), abstract: the DiT runtime stack applies RoPE from cached
// coefficients and indexes a KV cache that retains a limited temporal window.  This kernel does
// both in one pass over HBM: q, k, v are read once; rotated q goes back in place, rotated k and v
// go to ring slot f mod cap.  The work is pure streaming (6 bf16 tensors of B*L*H*D elements),
// so it is bound by HBM bandwidth: every thread moves 16-byte vectors, a warp covers 512
// contiguous bytes of each input, and the coefficient tables (< 20 KB) stay in L1/L2.  When the
// attention rotates the queries itself (its query prologue), the K/V-only instantiation leaves q
// alone and moves 4 of the 6 streams.
#include <cuda_bf16.h>

#include "internal.h"

namespace unstep {
namespace {

constexpr int kThreads = 256;
#ifndef UNSTEP_ROPE_ITEMS
#define UNSTEP_ROPE_ITEMS 1
#endif
// K/V-only form: two vectors of each of its two inputs per thread keep as many bytes in flight
#ifndef UNSTEP_ROPE_ITEMS_KV
#define UNSTEP_ROPE_ITEMS_KV 2
#endif
// independent 16-byte vectors (of each input) per thread
template <bool kQ>
constexpr int items_per_thread() { return kQ ? UNSTEP_ROPE_ITEMS : UNSTEP_ROPE_ITEMS_KV; }

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_plain(const void *p) {
  return *reinterpret_cast<const uint4 *>(p);
}

struct Item {
  long long e;       // element offset of the 8-channel vector in q/k/v (the activations)
  long long ce;      // element offset in the caches
  float2 cs[4];      // cos/sin of its 4 channel pairs
};

// Where item `it` (one 8-channel vector of one (stream, token, head)) lives, and its coefficients.
// All index arithmetic is 32-bit (items < 2^31, checked on the host) with multiply-high division.
// Returns false only in the debug build, when an index falls outside its tensor (the item is
// then skipped and the error word set).
template <int D>
__device__ __forceinline__ bool locate(const RopeAppendParams &p, uint32_t it, Item &m) {
  constexpr int kLogV = (D == 128) ? 4 : 3;  // 16-byte vectors per head row: D / 8
  const uint32_t c8 = it & ((1u << kLogV) - 1);
  const uint32_t r = it >> kLogV;             // (b*L + l)*H + h
  const uint32_t bl = fdiv(r, p.div_h);
  const uint32_t h = r - bl * static_cast<uint32_t>(p.H);
  const uint32_t b = fdiv(bl, p.div_l);
  const uint32_t l = bl - b * static_cast<uint32_t>(p.L);
  const uint32_t i = fdiv(l, p.div_tf);
  const uint32_t tok = l - i * static_cast<uint32_t>(p.Tf);
  const uint32_t y = fdiv(tok, p.div_wg);
  const uint32_t x = tok - y * static_cast<uint32_t>(p.Wg);
  const int f = p.frame_idx + static_cast<int>(i);
  int slot = p.slot0 + static_cast<int>(i);   // i < frames <= cap: one wrap at most
  if (slot >= p.cap) slot -= p.cap;
  // q, k, v: the shard's stream and head within the activations (it * 8 when unsharded)
  m.e = p.sharded ? ((static_cast<long long>(p.b0) + b) * p.L + l) * p.act_H * D +
                        (static_cast<long long>(p.h0) + h) * D + c8 * 8
                  : static_cast<long long>(it) * 8;
  m.ce = ((static_cast<long long>(b) * p.H + h) * p.rows + static_cast<long long>(slot) * p.Tf +
          tok) * D + c8 * 8;
  if (kDebugChecks) {
    const long long n_act = static_cast<long long>(p.act_B) * p.L * p.act_H * D;
    const long long n_cache = static_cast<long long>(p.B) * p.H * p.rows * D;
    const bool ok = b < static_cast<uint32_t>(p.B) && h < static_cast<uint32_t>(p.H) &&
                    i < static_cast<uint32_t>(p.frames) && y < static_cast<uint32_t>(p.Hg) &&
                    slot >= 0 && slot < p.cap && f >= 0 && f < p.max_pos_t && m.e >= 0 &&
                    m.e + 8 <= n_act && m.ce >= 0 && m.ce + 8 <= n_cache;
    if (!debug_check(ok, p.dev_error)) return false;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int pr = static_cast<int>(c8) * 4 + u;  // channel pair index
    const float2 *src;
    if (pr < p.half_t) {
      src = p.tab_t + f * p.half_t + pr;
    } else if (pr < p.half_t + p.half_h) {
      src = p.tab_h + static_cast<int>(y) * p.half_h + (pr - p.half_t);
    } else {
      src = p.tab_w + static_cast<int>(x) * p.half_w + (pr - p.half_t - p.half_h);
    }
    m.cs[u] = __ldg(src);
  }
  return true;
}

// kQ: q is rotated in place; without it q is neither read nor written.
template <int D, bool kQ>
__global__ void __launch_bounds__(kThreads) rope_kv_append_kernel(const RopeAppendParams p,
                                                                   uint32_t n_items) {
  constexpr int kItemsPerThread = items_per_thread<kQ>();
  const uint32_t base = blockIdx.x * (kThreads * kItemsPerThread) + threadIdx.x;
  if (blockIdx.x == 0 && threadIdx.x < p.frames) {
    const int f = p.frame_idx + threadIdx.x;
    if (debug_check(f >= 0 && p.cap > 0, p.dev_error)) p.slot_frame[f % p.cap] = f;
  }
  Item m[kItemsPerThread];
  uint4 qv[kItemsPerThread], kv[kItemsPerThread], vv[kItemsPerThread];
  bool live[kItemsPerThread];
#pragma unroll
  for (int u = 0; u < kItemsPerThread; ++u) {
    const uint32_t it = base + u * kThreads;
    live[u] = it < n_items && locate<D>(p, it, m[u]);
    if (live[u]) {
      if (kQ) qv[u] = ld_plain(static_cast<const __nv_bfloat16 *>(p.q) + m[u].e);
      kv[u] = ld_stream(static_cast<const __nv_bfloat16 *>(p.k) + m[u].e);
      vv[u] = ld_stream(static_cast<const __nv_bfloat16 *>(p.v) + m[u].e);
    }
  }
#pragma unroll
  for (int u = 0; u < kItemsPerThread; ++u) {
    if (!live[u]) continue;
    if (kQ) {
      uint4 qo;
      qo.x = rope_rotate_pair(qv[u].x, m[u].cs[0]);
      qo.y = rope_rotate_pair(qv[u].y, m[u].cs[1]);
      qo.z = rope_rotate_pair(qv[u].z, m[u].cs[2]);
      qo.w = rope_rotate_pair(qv[u].w, m[u].cs[3]);
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.q) + m[u].e) = qo;
    }
    uint4 ko;
    ko.x = rope_rotate_pair(kv[u].x, m[u].cs[0]);
    ko.y = rope_rotate_pair(kv[u].y, m[u].cs[1]);
    ko.z = rope_rotate_pair(kv[u].z, m[u].cs[2]);
    ko.w = rope_rotate_pair(kv[u].w, m[u].cs[3]);
    *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.k_cache) + m[u].ce) = ko;
    *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.v_cache) + m[u].ce) = vv[u];
  }
}

}  // namespace

cudaError_t launch_rope_kv_append(const RopeAppendParams &p, cudaStream_t stream) {
  const long long n_items = static_cast<long long>(p.B) * p.L * p.H * (p.D / 8);
  const int items = p.rotate_q ? items_per_thread<true>() : items_per_thread<false>();
  if (n_items >= (1ll << 31) - kThreads * items) return cudaErrorInvalidConfiguration;
  RopeAppendParams q = p;
  q.slot0 = p.frame_idx % p.cap;
  q.div_h = make_fastdiv(static_cast<uint32_t>(p.H));
  q.div_l = make_fastdiv(static_cast<uint32_t>(p.L));
  q.div_tf = make_fastdiv(static_cast<uint32_t>(p.Tf));
  q.div_wg = make_fastdiv(static_cast<uint32_t>(p.Wg));
  const long long per_block = kThreads * items;
  long long blocks = (n_items + per_block - 1) / per_block;
  if (blocks < 1) blocks = 1;
  const uint32_t n = static_cast<uint32_t>(n_items);
  const dim3 gb(static_cast<unsigned>(blocks));
  if (p.D == 128 && p.rotate_q) {
    rope_kv_append_kernel<128, true><<<gb, kThreads, 0, stream>>>(q, n);
  } else if (p.D == 128) {
    rope_kv_append_kernel<128, false><<<gb, kThreads, 0, stream>>>(q, n);
  } else if (p.D == 64 && p.rotate_q) {
    rope_kv_append_kernel<64, true><<<gb, kThreads, 0, stream>>>(q, n);
  } else if (p.D == 64) {
    rope_kv_append_kernel<64, false><<<gb, kThreads, 0, stream>>>(q, n);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace unstep
