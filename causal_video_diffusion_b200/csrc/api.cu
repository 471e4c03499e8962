// api.cu -- host side of the C ABI declared in include/unstep.h: argument validation, cache
// metadata, the RoPE coefficient tables, window resolution, TMA descriptors and launches.
//
// UnStep paper (arXiv 2609.32518), abstract: RoPE from precomputed coefficients, KV indexing and
// a limited temporal window of the attention KV cache; Table 3: chunks of three latent frames.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "../../include/unstep.h"
#include "conv3d.h"
#include "gemm.h"
#include "internal.h"

namespace {

constexpr int kInitMagic = 0x55535450;  // "USTP"

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Stream and head extents of the activation tensors the cache's shard lives in.
int act_B(const unstep_cache_t *c) { return c->act_B > 0 ? c->act_B : c->B; }
int act_H(const unstep_cache_t *c) { return c->act_H > 0 ? c->act_H : c->H; }

// Shape fields only (no pointers): 0 if valid, else a status code.
int check_shape(const unstep_cache_t *c) {
  if (!c) return UNSTEP_ERR_ARG;
  if (c->B < 1 || c->H < 1 || c->Hg < 1 || c->Wg < 1 || c->cap_frames < 1 || c->max_pos_t < 1)
    return UNSTEP_ERR_ARG;
  if (c->d_t < 0 || c->d_h < 0 || c->d_w < 0 || (c->d_t & 1) || (c->d_h & 1) || (c->d_w & 1))
    return UNSTEP_ERR_ARG;
  if (c->d_t + c->d_h + c->d_w != c->D) return UNSTEP_ERR_ARG;
  if (!(c->theta > 0.0) || !std::isfinite(c->theta)) return UNSTEP_ERR_ARG;
  if (c->D != 64 && c->D != 128) return UNSTEP_ERR_UNSUPPORTED;
  // row and element indices of the kernels: rows per (b, h) and TMA extents fit in int32,
  // every element offset in int64
  const long long tf = static_cast<long long>(c->Hg) * c->Wg;
  const long long rows = tf * c->cap_frames;
  if (tf > (1ll << 24) || rows > (1ll << 30) || static_cast<long long>(c->B) * c->H > (1ll << 30))
    return UNSTEP_ERR_UNSUPPORTED;
  if (c->max_pos_t > (1 << 24)) return UNSTEP_ERR_UNSUPPORTED;
  // the shard's place in the activations
  const long long act_b = act_B(c), act_h = act_H(c);
  if (c->act_B < 0 || c->act_H < 0 || c->b0 < 0 || c->h0 < 0) return UNSTEP_ERR_ARG;
  if (c->b0 + static_cast<long long>(c->B) > act_b || c->h0 + static_cast<long long>(c->H) > act_h)
    return UNSTEP_ERR_ARG;
  if (act_b * act_h > (1ll << 30)) return UNSTEP_ERR_UNSUPPORTED;
  return UNSTEP_OK;
}

size_t table_floats(const unstep_cache_t *c) {
  return 2ull * (static_cast<size_t>(c->max_pos_t) * (c->d_t / 2) +
                 static_cast<size_t>(c->Hg) * (c->d_h / 2) +
                 static_cast<size_t>(c->Wg) * (c->d_w / 2));
}

int check_ready(const unstep_cache_t *c) {
  int rc = check_shape(c);
  if (rc) return rc;
  if (c->initialized != kInitMagic) return UNSTEP_ERR_ARG;
  if (!c->k_cache || !c->v_cache || !c->slot_frame || !c->cos_sin || !c->dev_error)
    return UNSTEP_ERR_ARG;
  return UNSTEP_OK;
}

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle: dims[0] is the contiguous channel axis (boxed 64 wide).
bool encode_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                 const cuuint64_t *strides_bytes, const cuuint32_t *box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                  const_cast<void *>(base), dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Multiprocessor count of the current device (cached per device).
int device_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) {
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

long long max_units(const unstep_cache_t *c) {
  const long long rows = static_cast<long long>(c->cap_frames) * c->Hg * c->Wg;
  return static_cast<long long>(c->B) * c->H * ((rows + 255) / 256);
}

size_t scratch_bytes_for(const unstep_cache_t *c, int sms) {
  return unstep::attn_counter_bytes(max_units(c)) +
         2ull * static_cast<size_t>(sms) * unstep::attn_slot_floats(c->D) * sizeof(float);
}

// ---- checkpoint buffer header (layout documented with unstep_cache_save) ----
constexpr int kStateMagic = 0x43545355;  // "USTC"
constexpr int kStateVersion = 1;
constexpr size_t kStateSlotOffset = 128;

size_t state_header_bytes(const unstep_cache_t *c) {
  return kStateSlotOffset + ((sizeof(int) * static_cast<size_t>(c->cap_frames) + 15) / 16) * 16;
}

void put_i32(unsigned char *p, size_t off, int v) { std::memcpy(p + off, &v, sizeof(int)); }
int get_i32(const unsigned char *p, size_t off) {
  int v;
  std::memcpy(&v, p + off, sizeof(int));
  return v;
}

void write_state_header(const unstep_cache_t *c, unsigned char *p) {
  const int f[14] = {c->B,  c->H,          c->D,         c->Hg,  c->Wg,  c->d_t, c->d_h,
                     c->d_w, c->cap_frames, c->max_pos_t, act_B(c), act_H(c), c->b0, c->h0};
  put_i32(p, 0, kStateMagic);
  put_i32(p, 4, kStateVersion);
  for (int i = 0; i < 14; ++i) put_i32(p, 8 + 4 * i, f[i]);
  std::memcpy(p + 64, &c->theta, sizeof(double));
  put_i32(p, 72, c->frames_written);
  put_i32(p, 76, c->first_frame);
  put_i32(p, 80, c->last_chunk_start);
  put_i32(p, 84, c->last_chunk_frames);
}

int read_state_header(const unsigned char *p, unstep_cache_t *c) {
  if (get_i32(p, 0) != kStateMagic || get_i32(p, 4) != kStateVersion) return UNSTEP_ERR_ARG;
  int *f[14] = {&c->B,  &c->H,          &c->D,         &c->Hg,    &c->Wg,    &c->d_t, &c->d_h,
                &c->d_w, &c->cap_frames, &c->max_pos_t, &c->act_B, &c->act_H, &c->b0,  &c->h0};
  for (int i = 0; i < 14; ++i) *f[i] = get_i32(p, 8 + 4 * i);
  std::memcpy(&c->theta, p + 64, sizeof(double));
  c->frames_written = get_i32(p, 72);
  c->first_frame = get_i32(p, 76);
  c->last_chunk_start = get_i32(p, 80);
  c->last_chunk_frames = get_i32(p, 84);
  return UNSTEP_OK;
}

// Shape and shard identical (the metadata may differ).
bool same_state_shape(const unstep_cache_t *a, const unstep_cache_t *b) {
  return a->B == b->B && a->H == b->H && a->D == b->D && a->Hg == b->Hg && a->Wg == b->Wg &&
         a->d_t == b->d_t && a->d_h == b->d_h && a->d_w == b->d_w &&
         a->cap_frames == b->cap_frames && a->max_pos_t == b->max_pos_t &&
         act_B(a) == act_B(b) && act_H(a) == act_H(b) && a->b0 == b->b0 && a->h0 == b->h0 &&
         std::memcmp(&a->theta, &b->theta, sizeof(double)) == 0;
}

unsigned next_epoch() {
  static std::atomic<unsigned> counter{0};
  return counter.fetch_add(1, std::memory_order_relaxed) % 0xFFFFFFu + 1u;
}

}  // namespace

extern "C" {

int unstep_version(void) { return 101; }

const char *unstep_status_string(int status) {
  switch (status) {
    case UNSTEP_OK: return "ok";
    case UNSTEP_ERR_ARG: return "invalid argument";
    case UNSTEP_ERR_SHAPE: return "shape mismatch";
    case UNSTEP_ERR_ALIGN: return "pointer not 16-byte aligned";
    case UNSTEP_ERR_FRAME_ORDER: return "frame_idx is neither the next chunk nor the latest chunk";
    case UNSTEP_ERR_WINDOW: return "window outside [chunk frames, cache capacity] or empty cache";
    case UNSTEP_ERR_UNSUPPORTED: return "unsupported head width or size";
    case UNSTEP_ERR_CUDA: return "CUDA runtime error";
    case UNSTEP_ERR_DEVICE_TIMEOUT: return "a device-side wait timed out";
    case UNSTEP_ERR_SCRATCH_LIMIT:
      return "the call needs more scratch than the library's fixed device buffer holds";
    case UNSTEP_ERR_DEVICE_BOUNDS:
      return "a device-side index check failed (debug build)";
    default: return "unknown status";
  }
}

size_t unstep_cache_table_bytes(const unstep_cache_t *cache) {
  if (check_shape(cache)) return 0;
  return table_floats(cache) * sizeof(float);
}

size_t unstep_cache_kv_bytes(const unstep_cache_t *cache) {
  if (check_shape(cache)) return 0;
  return static_cast<size_t>(cache->B) * cache->H * cache->cap_frames * cache->Hg * cache->Wg *
         cache->D * 2;
}

size_t unstep_attn_scratch_bytes(const unstep_cache_t *cache) {
  if (check_shape(cache)) return 0;
  const int sms = device_sms();
  if (sms <= 0) return 0;
  return scratch_bytes_for(cache, sms);
}

int unstep_cache_init(unstep_cache_t *cache, unstep_stream_t stream) {
  int rc = check_shape(cache);
  if (rc) return rc;
  if (!cache->k_cache || !cache->v_cache || !cache->slot_frame || !cache->cos_sin ||
      !cache->dev_error)
    return UNSTEP_ERR_ARG;
  if (!aligned16(cache->k_cache) || !aligned16(cache->v_cache) || !aligned16(cache->cos_sin) ||
      !aligned16(cache->attn_scratch))
    return UNSTEP_ERR_ALIGN;
  if (cache->attn_scratch) {
    const int sms = device_sms();
    if (sms <= 0) return UNSTEP_ERR_CUDA;
    if (cache->attn_scratch_bytes < scratch_bytes_for(cache, sms)) return UNSTEP_ERR_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // cached coefficients: cos/sin of pos * theta^(-2j/d_a), computed in fp64, stored fp32
  std::vector<float> tab(table_floats(cache));
  size_t o = 0;
  const int dims[3] = {cache->d_t, cache->d_h, cache->d_w};
  const int npos[3] = {cache->max_pos_t, cache->Hg, cache->Wg};
  for (int a = 0; a < 3; ++a) {
    const int half = dims[a] / 2;
    for (int pos = 0; pos < npos[a]; ++pos) {
      for (int j = 0; j < half; ++j) {
        const double inv = std::pow(cache->theta, -2.0 * j / static_cast<double>(dims[a]));
        const double ang = static_cast<double>(pos) * inv;
        tab[o++] = static_cast<float>(std::cos(ang));
        tab[o++] = static_cast<float>(std::sin(ang));
      }
    }
  }
  const size_t kvb = unstep_cache_kv_bytes(cache);
  if (cudaMemcpyAsync(cache->cos_sin, tab.data(), tab.size() * sizeof(float),
                      cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemsetAsync(cache->k_cache, 0, kvb, s) != cudaSuccess ||
      cudaMemsetAsync(cache->v_cache, 0, kvb, s) != cudaSuccess ||
      cudaMemsetAsync(cache->slot_frame, 0xFF, sizeof(int) * cache->cap_frames, s) !=
          cudaSuccess ||
      cudaMemsetAsync(cache->dev_error, 0, sizeof(int), s) != cudaSuccess ||
      (cache->attn_scratch &&
       cudaMemsetAsync(cache->attn_scratch, 0, unstep::attn_counter_bytes(max_units(cache)), s) !=
           cudaSuccess)) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  cache->frames_written = 0;
  cache->first_frame = 0;
  cache->last_chunk_start = -1;
  cache->last_chunk_frames = 0;
  cache->initialized = kInitMagic;
  return UNSTEP_OK;
}

int unstep_append_plan(const unstep_cache_t *cache, int frame_idx, unstep_grid_t grid,
                       int *slots_out) {
  int rc = check_shape(cache);
  if (rc) return rc;
  if (cache->initialized != kInitMagic) return UNSTEP_ERR_ARG;
  if (grid.Hg != cache->Hg || grid.Wg != cache->Wg || grid.frames < 1) return UNSTEP_ERR_SHAPE;
  if (grid.frames > cache->cap_frames) return UNSTEP_ERR_WINDOW;
  if (frame_idx < 0 || static_cast<long long>(frame_idx) + grid.frames > cache->max_pos_t)
    return UNSTEP_ERR_ARG;
  int is_new;
  if (cache->last_chunk_frames == 0) {
    is_new = 1;  // the stream's first chunk may start at any temporal position
  } else if (frame_idx == cache->frames_written) {
    is_new = 1;
  } else if (frame_idx == cache->last_chunk_start && grid.frames == cache->last_chunk_frames) {
    is_new = 0;
  } else {
    return UNSTEP_ERR_FRAME_ORDER;
  }
  if (slots_out)
    for (int i = 0; i < grid.frames; ++i) slots_out[i] = (frame_idx + i) % cache->cap_frames;
  return is_new;
}

int unstep_rope_kv_append_ex(void *q, const void *k, const void *v, unstep_cache_t *cache,
                             int frame_idx, unstep_grid_t grid, unsigned flags,
                             unstep_stream_t stream) {
  int rc = check_ready(cache);
  if (rc) return rc;
  if (flags & ~static_cast<unsigned>(UNSTEP_APPEND_DEFER_Q_ROPE)) return UNSTEP_ERR_ARG;
  const bool rotate_q = !(flags & UNSTEP_APPEND_DEFER_Q_ROPE);
  if ((rotate_q && !q) || !k || !v) return UNSTEP_ERR_ARG;
  if ((rotate_q && !aligned16(q)) || !aligned16(k) || !aligned16(v)) return UNSTEP_ERR_ALIGN;
  const int is_new = unstep_append_plan(cache, frame_idx, grid, nullptr);
  if (is_new < 0) return is_new;
  unstep::RopeAppendParams p{};
  p.q = rotate_q ? q : nullptr;
  p.rotate_q = rotate_q ? 1 : 0;
  p.k = k;
  p.v = v;
  p.k_cache = cache->k_cache;
  p.v_cache = cache->v_cache;
  p.slot_frame = cache->slot_frame;
  const float2 *tab = reinterpret_cast<const float2 *>(cache->cos_sin);
  p.tab_t = tab;
  p.tab_h = p.tab_t + static_cast<size_t>(cache->max_pos_t) * (cache->d_t / 2);
  p.tab_w = p.tab_h + static_cast<size_t>(cache->Hg) * (cache->d_h / 2);
  p.B = cache->B;
  p.H = cache->H;
  p.act_H = act_H(cache);
  p.b0 = cache->b0;
  p.h0 = cache->h0;
  p.sharded = (p.act_H != p.H || p.b0 != 0 || p.h0 != 0) ? 1 : 0;
  p.D = cache->D;
  p.Hg = cache->Hg;
  p.Wg = cache->Wg;
  p.Tf = cache->Hg * cache->Wg;
  p.L = grid.frames * p.Tf;
  p.half_t = cache->d_t / 2;
  p.half_h = cache->d_h / 2;
  p.half_w = cache->d_w / 2;
  p.frame_idx = frame_idx;
  p.frames = grid.frames;
  p.cap = cache->cap_frames;
  p.rows = cache->cap_frames * p.Tf;
  p.act_B = act_B(cache);
  p.max_pos_t = cache->max_pos_t;
  p.dev_error = cache->dev_error;
  if (unstep::launch_rope_kv_append(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  if (is_new) {
    if (cache->last_chunk_frames == 0) cache->first_frame = frame_idx;
    cache->frames_written = frame_idx + grid.frames;
  }
  cache->last_chunk_start = frame_idx;
  cache->last_chunk_frames = grid.frames;
  return UNSTEP_OK;
}

int unstep_rope_kv_append(void *q, const void *k, const void *v, unstep_cache_t *cache,
                          int frame_idx, unstep_grid_t grid, unstep_stream_t stream) {
  return unstep_rope_kv_append_ex(q, k, v, cache, frame_idx, grid, 0u, stream);
}

int unstep_window_plan(const unstep_cache_t *cache, int window, unstep_window_plan_t *plan) {
  int rc = check_shape(cache);
  if (rc) return rc;
  if (!plan || cache->initialized != kInitMagic) return UNSTEP_ERR_ARG;
  if (cache->last_chunk_frames < 1) return UNSTEP_ERR_WINDOW;
  if (window < cache->last_chunk_frames || window > cache->cap_frames) return UNSTEP_ERR_WINDOW;
  const int tf = cache->Hg * cache->Wg;
  const int cap = cache->cap_frames;
  const int f_end = cache->last_chunk_start + cache->last_chunk_frames - 1;
  int f0 = f_end - window + 1;
  if (f0 < cache->first_frame) f0 = cache->first_frame;
  const int nf = f_end - f0 + 1;
  const int s0 = f0 % cap;
  plan->first_frame = f0;
  plan->last_frame = f_end;
  plan->keys = nf * tf;
  plan->seg_row[0] = s0 * tf;
  if (s0 + nf <= cap) {
    plan->seg_len[0] = nf * tf;
    plan->seg_row[1] = 0;
    plan->seg_len[1] = 0;
  } else {
    plan->seg_len[0] = (cap - s0) * tf;
    plan->seg_row[1] = 0;
    plan->seg_len[1] = (s0 + nf - cap) * tf;
  }
  return UNSTEP_OK;
}

}  // extern "C"

namespace {

// What unstep_window_attn_ex and unstep_window_attn_noalloc share: validation, the window plan,
// the tensor maps, the persistent schedule and the launch.  `fixed_buffer` selects the scratch:
// false, the cache's own (cache->attn_scratch, sized at unstep_cache_init; none: one CTA per
// unit); true, the library's fixed device buffer, whose counters are zeroed on `st` first.
int window_attn_launch(const void *q, const unstep_cache_t *cache, int window, void *out,
                       unsigned flags, bool fixed_buffer, cudaStream_t st) {
  int rc = check_ready(cache);
  if (rc) return rc;
  if (flags & ~static_cast<unsigned>(UNSTEP_ATTN_ROPE_Q)) return UNSTEP_ERR_ARG;
  if (!q || !out) return UNSTEP_ERR_ARG;
  if (!aligned16(q) || !aligned16(out)) return UNSTEP_ERR_ALIGN;
  unstep_window_plan_t plan;
  rc = unstep_window_plan(cache, window, &plan);
  if (rc) return rc;
  const int D = cache->D, H = cache->H, B = cache->B;
  const int tf = cache->Hg * cache->Wg;
  const int L = cache->last_chunk_frames * tf;
  const long long R = static_cast<long long>(cache->cap_frames) * tf;
  const int n_pairs = (L + 255) / 256;
  // (head, 256-query) units are numbered in int32 by the kernel
  const long long units = static_cast<long long>(B) * H * n_pairs;
  if (units > INT_MAX) return fixed_buffer ? UNSTEP_ERR_SCRATCH_LIMIT : UNSTEP_ERR_UNSUPPORTED;
  const int U = static_cast<int>(units);

  void *scratch = nullptr;
  size_t counter_bytes = 0;
  int sms = 0;
  if (fixed_buffer) {
    size_t capacity = 0;
    if (unstep::static_attn_scratch(&scratch, &capacity) != cudaSuccess) {
      cudaGetLastError();
      return UNSTEP_ERR_CUDA;
    }
    sms = device_sms();
    if (sms <= 0) return UNSTEP_ERR_CUDA;
    counter_bytes = unstep::attn_counter_bytes(U);
    const size_t need = counter_bytes + 2ull * static_cast<size_t>(sms) *
                                            unstep::attn_slot_floats(D) * sizeof(float);
    if (need > capacity) return UNSTEP_ERR_SCRATCH_LIMIT;
  } else if (cache->attn_scratch) {
    scratch = cache->attn_scratch;
    counter_bytes = unstep::attn_counter_bytes(max_units(cache));
    sms = device_sms();
  }

  CUtensorMap tq, tk, tv;
  {
    // the whole activation tensor; the shard's streams and heads are TMA coordinates
    const cuuint64_t aB = static_cast<cuuint64_t>(act_B(cache));
    const cuuint64_t aH = static_cast<cuuint64_t>(act_H(cache));
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), aH, static_cast<cuuint64_t>(L), aB};
    const cuuint64_t str[3] = {static_cast<cuuint64_t>(D) * 2, aH * D * 2,
                               static_cast<cuuint64_t>(L) * aH * D * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    if (!encode_bf16(&tq, q, 4, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(R),
                                static_cast<cuuint64_t>(B) * H};
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(D) * 2,
                               static_cast<cuuint64_t>(R) * D * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if (!encode_bf16(&tk, cache->k_cache, 3, dims, str, box)) return UNSTEP_ERR_CUDA;
    if (!encode_bf16(&tv, cache->v_cache, 3, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  unstep::AttnParams p{};
  p.out = out;
  p.dev_error = cache->dev_error;
  p.B = B;
  p.H = H;
  p.act_H = act_H(cache);
  p.act_B = act_B(cache);
  p.b0 = cache->b0;
  p.h0 = cache->h0;
  p.L = L;
  p.rows = static_cast<int>(R);
  p.n_pairs = n_pairs;
  p.n_units = U;
  for (int s = 0; s < 2; ++s) {
    p.seg_row[s] = plan.seg_row[s];
    p.seg_len[s] = plan.seg_len[s];
    p.seg_tiles[s] = (plan.seg_len[s] + 127) / 128;
  }
  p.n_tiles = p.seg_tiles[0] + p.seg_tiles[1];
  p.div_pairs = unstep::make_fastdiv(static_cast<uint32_t>(p.n_pairs));
  p.div_heads = unstep::make_fastdiv(static_cast<uint32_t>(H));
  if (scratch && sms > 0) {
    // persistent schedule: whole units in waves of `sms` CTAs, the remainder split along keys
    p.dp_waves = U / sms;
    const int tail = U - p.dp_waves * sms;
    p.u_tail0 = p.dp_waves * sms;
    p.w_tail = static_cast<long long>(tail) * p.n_tiles;
    long long gsk = tail > 0 ? static_cast<long long>(tail) * 8 : 0;  // at most ~8 pieces/unit
    if (gsk > sms) gsk = sms;
    if (gsk > p.w_tail) gsk = p.w_tail;
    p.g_sk = static_cast<int>(gsk);
    p.grid = p.dp_waves > 0 ? sms : p.g_sk;
    p.counters = static_cast<unsigned *>(scratch);
    p.slots = reinterpret_cast<float *>(static_cast<char *>(scratch) + counter_bytes);
    p.slot_floats = static_cast<int>(unstep::attn_slot_floats(D));
    p.epoch = next_epoch();
  } else {
    // no scratch: one CTA per unit, nothing is split
    p.dp_waves = 1;
    p.grid = p.n_units;
    p.u_tail0 = p.n_units;
    p.g_sk = 0;
    p.w_tail = 0;
  }
  p.scale_log2 = static_cast<float>(1.4426950408889634073599 / std::sqrt(static_cast<double>(D)));
  p.wait_limit_ns = unstep::kWaitLimitNs;
  if (flags & UNSTEP_ATTN_ROPE_Q) {
    // q is the latest chunk's un-rotated queries: row l is token (i, y, x) of frame
    // last_chunk_start + i, rotated with the append's tables in the kernel's prologue
    const float2 *tab = reinterpret_cast<const float2 *>(cache->cos_sin);
    p.rope_q = 1;
    p.tab_t = tab;
    p.tab_h = p.tab_t + static_cast<size_t>(cache->max_pos_t) * (cache->d_t / 2);
    p.tab_w = p.tab_h + static_cast<size_t>(cache->Hg) * (cache->d_h / 2);
    p.half_t = cache->d_t / 2;
    p.half_h = cache->d_h / 2;
    p.half_w = cache->d_w / 2;
    p.Tf = tf;
    p.Wg = cache->Wg;
    p.frame0 = cache->last_chunk_start;
    p.frames = cache->last_chunk_frames;
    const size_t tab_bytes = sizeof(float2) * (static_cast<size_t>(p.frames) * p.half_t +
                                               static_cast<size_t>(cache->Hg) * p.half_h +
                                               static_cast<size_t>(cache->Wg) * p.half_w);
    p.tab_smem = tab_bytes <= static_cast<size_t>(unstep::kQRopeTabBytes) ? 1 : 0;
    p.div_tf = unstep::make_fastdiv(static_cast<uint32_t>(tf));
    p.div_wg = unstep::make_fastdiv(static_cast<uint32_t>(cache->Wg));
  }
  // the fixed buffer keeps whatever the previous call left in it: the counts must start at zero
  if (fixed_buffer && cudaMemsetAsync(scratch, 0, counter_bytes, st) != cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  if (unstep::launch_window_attn(D, tq, tk, tv, p, st) != cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

}  // namespace

extern "C" {

int unstep_window_attn_ex(const void *q, const unstep_cache_t *cache, int window, void *out,
                          unsigned flags, unstep_stream_t stream) {
  return window_attn_launch(q, cache, window, out, flags, false,
                            reinterpret_cast<cudaStream_t>(stream));
}

int unstep_window_attn(const void *q, const unstep_cache_t *cache, int window, void *out,
                       unstep_stream_t stream) {
  return unstep_window_attn_ex(q, cache, window, out, 0u, stream);
}

int unstep_window_attn_noalloc(const void *q, const unstep_cache_t *cache, int window,
                               void *out, unstep_stream_t stream) {
  return window_attn_launch(q, cache, window, out, 0u, true,
                            reinterpret_cast<cudaStream_t>(stream));
}

int unstep_gemm_bf16(const void *a, int lda, const void *b, int ldb, void *c, int ldc, int M,
                     int N, int K, int *dev_error, unstep_stream_t stream) {
  if (!a || !b || !c || !dev_error) return UNSTEP_ERR_ARG;
  if (M < 1 || N < 1 || K < 1) return UNSTEP_ERR_SHAPE;
  if ((N & 7) || (K & 7) || (lda & 7) || (ldb & 7) || (ldc & 7) || lda < K || ldb < K || ldc < N)
    return UNSTEP_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return UNSTEP_ERR_ALIGN;
  CUtensorMap ta, tb;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(lda) * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode_bf16(&ta, a, 2, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(ldb) * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode_bf16(&tb, b, 2, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  // CTA pairs (256 x 256 tiles) when the product is at least one pair tile; else single CTAs
#ifndef UNSTEP_GEMM_2SM
#define UNSTEP_GEMM_2SM 1
#endif
  const bool pair = UNSTEP_GEMM_2SM && M >= 256 && N >= 256;
  CUtensorMap tc;
  if (pair) {
    // the pair kernel stores C through TMA, one 64-column x 32-row box per epilogue warp
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    const cuuint64_t str[1] = {static_cast<cuuint64_t>(ldc) * 2};
    const cuuint32_t box[2] = {64, 32};
    if (!encode_bf16(&tc, c, 2, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  const cudaError_t e =
      pair ? unstep::launch_gemm2sm_bf16_tn(ta, tb, tc, M, N, K, dev_error,
                                            reinterpret_cast<cudaStream_t>(stream))
           : unstep::launch_gemm_bf16_tn(ta, tb, c, M, N, K, ldc, dev_error,
                                         reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

int unstep_lowrank_linear(const void *x, const void *w1, const void *w2, void *t, void *y, int M,
                          int d_in, int rank, int d_out, int *dev_error, unstep_stream_t stream) {
  int rc = unstep_gemm_bf16(x, d_in, w1, d_in, t, rank, M, rank, d_in, dev_error, stream);
  if (rc) return rc;
  return unstep_gemm_bf16(t, rank, w2, rank, y, d_out, M, d_out, rank, dev_error, stream);
}

int unstep_renoise(const void *x0, const void *eps, void *out, long long n, float sigma,
                   unstep_stream_t stream) {
  if (!x0 || !eps || !out || n < 0) return UNSTEP_ERR_ARG;
  if (!(sigma >= 0.f && sigma <= 1.f)) return UNSTEP_ERR_ARG;
  if (!aligned16(x0) || !aligned16(eps) || !aligned16(out)) return UNSTEP_ERR_ALIGN;
  if (n == 0) return UNSTEP_OK;
  if (unstep::launch_renoise(x0, eps, out, n, sigma, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

size_t unstep_conv3d_scratch_bytes(void) {
  const int sms = device_sms();
  if (sms <= 0) return 0;
  return unstep::conv_scratch_bytes(sms);
}

int unstep_conv3d_causal(const void *x, const void *w, const float *bias, void *y, int B, int T,
                         int H, int W, int C_in, int C_out, void *scratch, size_t scratch_bytes,
                         int *dev_error, unstep_stream_t stream) {
  if (!x || !w || !y || !dev_error) return UNSTEP_ERR_ARG;
  if (B < 1 || T < 1 || H < 1 || W < 1 || C_in < 1 || C_out < 1) return UNSTEP_ERR_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || !aligned16(scratch) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return UNSTEP_ERR_ALIGN;
  int sms = 0;
  if (scratch) {
    sms = device_sms();
    if (sms <= 0) return UNSTEP_ERR_CUDA;
    if (scratch_bytes < unstep::conv_scratch_bytes(sms)) return UNSTEP_ERR_ARG;
  }
  if (C_in % 64 != 0 || C_out % 8 != 0) return UNSTEP_ERR_UNSUPPORTED;
  const long long frames = static_cast<long long>(B) * (T + 2);
  const long long tiles_h = (H + unstep::kConvTileH - 1) / unstep::kConvTileH;
  const long long tiles_w = (W + 15) / 16;
  const long long m_tiles = static_cast<long long>(B) * T * tiles_h * tiles_w;
  const long long n_tiles = (C_out + 127) / 128;
  if (frames > 0x7FFFFFFFll || m_tiles * n_tiles > 0x7FFFFFFFll || W > (1 << 24) ||
      H > (1 << 24) || C_in > (1 << 16) || C_out > (1 << 24))
    return UNSTEP_ERR_UNSUPPORTED;
  CUtensorMap tmx, tmw;
  {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C_in), static_cast<cuuint64_t>(W),
                                static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(frames)};
    const cuuint64_t str[3] = {static_cast<cuuint64_t>(C_in) * 2,
                               static_cast<cuuint64_t>(W) * C_in * 2,
                               static_cast<cuuint64_t>(H) * W * C_in * 2};
    // the output tile's rows and a halo row on each side, for the three dy taps at once
    const cuuint32_t box[4] = {64, 16, static_cast<cuuint32_t>(unstep::kConvTileH + 2), 1};
    if (!encode_bf16(&tmx, x, 4, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C_in), 27,
                                static_cast<cuuint64_t>(C_out)};
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(C_in) * 2,
                               static_cast<cuuint64_t>(C_in) * 27 * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(unstep::conv_weight_box_n(H))};
    if (!encode_bf16(&tmw, w, 3, dims, str, box)) return UNSTEP_ERR_CUDA;
  }
  unstep::ConvParams p{};
  p.y = y;
  p.bias = bias;
  p.dev_error = dev_error;
  p.wait_limit_ns = unstep::kWaitLimitNs;
  p.B = B;
  p.T = T;
  p.H = H;
  p.W = W;
  p.C_in = C_in;
  p.C_out = C_out;
  p.tiles_h = static_cast<int>(tiles_h);
  p.tiles_w = static_cast<int>(tiles_w);
  p.m_tiles = static_cast<int>(m_tiles);
  p.n_tiles = static_cast<int>(n_tiles);
  if (scratch) {
    p.counters = static_cast<unsigned *>(scratch);
    p.slots = reinterpret_cast<float *>(static_cast<char *>(scratch) +
                                        unstep::conv_counter_bytes(sms));
    p.epoch = next_epoch();
  }
  if (unstep::launch_conv3d_causal(tmx, tmw, p, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

size_t unstep_cache_state_bytes(const unstep_cache_t *cache) {
  if (check_shape(cache)) return 0;
  return state_header_bytes(cache) + 2 * unstep_cache_kv_bytes(cache);
}

int unstep_cache_save(const unstep_cache_t *cache, void *host_dst, size_t bytes,
                      unstep_stream_t stream) {
  int rc = check_ready(cache);
  if (rc) return rc;
  if (!host_dst || bytes < unstep_cache_state_bytes(cache)) return UNSTEP_ERR_ARG;
  unsigned char *dst = static_cast<unsigned char *>(host_dst);
  const size_t hb = state_header_bytes(cache), kvb = unstep_cache_kv_bytes(cache);
  std::memset(dst, 0, hb);
  write_state_header(cache, dst);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(dst + kStateSlotOffset, cache->slot_frame,
                      sizeof(int) * cache->cap_frames, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(dst + hb, cache->k_cache, kvb, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(dst + hb + kvb, cache->v_cache, kvb, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

int unstep_cache_restore(unstep_cache_t *cache, const void *host_src, size_t bytes,
                         unstep_stream_t stream) {
  int rc = check_ready(cache);
  if (rc) return rc;
  if (!host_src || bytes < kStateSlotOffset) return UNSTEP_ERR_ARG;
  const unsigned char *src = static_cast<const unsigned char *>(host_src);
  unstep_cache_t saved{};
  rc = read_state_header(src, &saved);
  if (rc) return rc;
  if (!same_state_shape(cache, &saved)) return UNSTEP_ERR_SHAPE;
  if (bytes < unstep_cache_state_bytes(cache)) return UNSTEP_ERR_ARG;
  // the saved metadata must describe a ring this cache can hold
  if (saved.last_chunk_frames < 0 || saved.last_chunk_frames > cache->cap_frames ||
      saved.frames_written < 0 || saved.frames_written > cache->max_pos_t)
    return UNSTEP_ERR_ARG;
  const size_t hb = state_header_bytes(cache), kvb = unstep_cache_kv_bytes(cache);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(cache->slot_frame, src + kStateSlotOffset,
                      sizeof(int) * cache->cap_frames, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(cache->k_cache, src + hb, kvb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(cache->v_cache, src + hb + kvb, kvb, cudaMemcpyHostToDevice, s) !=
          cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  cache->frames_written = saved.frames_written;
  cache->first_frame = saved.first_frame;
  cache->last_chunk_start = saved.last_chunk_start;
  cache->last_chunk_frames = saved.last_chunk_frames;
  return UNSTEP_OK;
}

int unstep_get_device_error(const unstep_cache_t *cache, unstep_stream_t stream) {
  if (!cache || !cache->dev_error) return UNSTEP_ERR_ARG;
  int v = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, cache->dev_error, sizeof(int), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return v;
}

int unstep_selftest_wait_timeout(int *dev_error, uint64_t limit_ns, unstep_stream_t stream) {
  if (!dev_error) return UNSTEP_ERR_ARG;
  if (unstep::launch_wait_timeout_selftest(dev_error, limit_ns,
                                           reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

int unstep_selftest_exp2(const float *x, float *y_poly, float *y_mufu, int n,
                         unstep_stream_t stream) {
  if (!x || !y_poly || !y_mufu || n < 0) return UNSTEP_ERR_ARG;
  if (n == 0) return UNSTEP_OK;
  if (unstep::launch_exp2_selftest(x, y_poly, y_mufu, n, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return UNSTEP_ERR_CUDA;
  }
  return UNSTEP_OK;
}

}  // extern "C"
