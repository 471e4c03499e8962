// window_attn.cu -- windowed chunk-causal attention on the Blackwell tensor cores.
//
// UnStep paper (arXiv 2609.32518): the chunk's queries attend to the keys of the limited
// temporal window kept in the KV cache (abstract; Table 1 row C4), all queries of a chunk seeing
// the same key set.  out = softmax(q K^T / sqrt(D)) V, computed as a streaming (online) softmax
// over 128-key tiles:
//
//   S_j  = Q K_j^T                      tcgen05.mma, A = Q (smem), B = K_j (smem), fp32 in TMEM
//   m    = running max (raised lazily), P_j = exp2(S_j * log2(e)/sqrt(D) - m)   (fp32 -> bf16)
//   O   += P_j V_j                      tcgen05.mma, A = P_j (TMEM), B = V_j (smem)
//   l   += rowsum(P_j);   out = O / l  (bf16)
//
// Work split of one CTA (one (stream, head) and two 128-row query tiles, 384 threads):
//   warps 0-3  softmax + epilogue of query tile 0 (thread t owns TMEM lane / query row t)
//   warps 4-7  softmax + epilogue of query tile 1
//   warp  8    TMA producer: Q once, then K_0, V_0, K_1, V_1, ... through an NS-stage ring
//   warp  9    MMA issuer (one thread): QK^T and PV for both tiles, ping-ponging so that the
//              tensor core works on one tile while the other tile's softmax runs
//   warps 10-11 idle (they complete the third warpgroup, whose registers the softmax takes)
// When q arrives un-rotated, each softmax warpgroup first applies the 3D RoPE to its loaded Q
// tile in shared memory (once per segment, from coefficient rows staged in shared memory),
// before the MMA issuer may use it.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D); P0 and P1
// alias S0 and S1 for D = 128 and sit at [384,448) and [448,512) for D = 64.
//
// The ring cache holds the window as at most two contiguous row ranges; each range is tiled on
// its own (its last tile masked), so a tile never straddles the wrap and the ring slot offset is
// simply the TMA row coordinate.  The running max is only raised when a tile's max exceeds it
// by more than 8 (log2 units): below that, P <= 2^8 is exact enough in bf16/fp32 and O needs no
// rescale; above it, the owning warp rescales its O rows in TMEM after the previous PV retired.
//
// Every wait is bounded (WaitGuard): on a timeout the CTA records UNSTEP_ERR_DEVICE_TIMEOUT,
// lets in-flight TMA copies and MMAs land, frees TMEM and exits.
#include <cuda_bf16.h>

#include <mutex>

#include "../../include/unstep.h"
#include "internal.h"
#include "sm100.cuh"

namespace unstep {
namespace {

constexpr int kThreads = 384;
// Register split: launched at 168 per thread (384 x 168 = 64512), the producer/MMA warpgroup
// drops to kRegsIo and the two softmax warpgroups rise to kRegsSoftmax; the static_assert keeps
// 2 x 128 x kRegsSoftmax + 128 x kRegsIo within the launch total (184/128: 63488), so the claim
// can always be satisfied.  With the polynomial share below, 184/128 measured 1-2 % faster than
// 200/96 on full-cache and windowed layers.
#ifndef UNSTEP_REGS_SOFTMAX
#define UNSTEP_REGS_SOFTMAX 184
#endif
#ifndef UNSTEP_REGS_IO
#define UNSTEP_REGS_IO 128
#endif
constexpr int kRegsSoftmax = UNSTEP_REGS_SOFTMAX;
constexpr int kRegsIo = UNSTEP_REGS_IO;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsIo <= kThreads * 168, "register split");
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

#ifndef UNSTEP_KV_STAGES
#define UNSTEP_KV_STAGES 2
#endif

template <int D, bool kRopeQ = false>
struct Cfg {
  static constexpr int kBoxes = D / 64;                // 128-byte swizzle boxes per row
  static constexpr int kTileBytes = 128 * D * 2;       // 128 rows x D bf16
  static constexpr int kStages = UNSTEP_KV_STAGES;     // ring stages, one key tile's K and V each
  static constexpr int kStageBytes = 2 * kTileBytes;   // K tile, then V tile
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemKV = 2 * kTileBytes;
  static constexpr int kSmemBar = kSmemKV + kStages * kStageBytes;
  static constexpr int kSmemTab = kSmemBar + 256;      // RoPE rows of the chunk (kRopeQ)
  static constexpr int kSmemUsed = kSmemTab + (kRopeQ ? kQRopeTabBytes : 0);
  // at least ~116 KB so that a second CTA (which would block on TMEM) never shares the SM
  static constexpr int kSmemAlloc = (kSmemUsed + 1024 > 118 * 1024) ? kSmemUsed + 1024
                                                                    : 118 * 1024;
  // e.g. three K/V stages of 64 KB beside the 64 KB of Q do not fit (D = 128)
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA: fewer K/V stages");
  static constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO0 = 256, kTmO1 = 256 + D;
  // P (bf16, 64 columns per tile).  tcgen05.mma operations are only guaranteed to execute in
  // issue order when they have the same shape; QK^T (N = 128) may overwrite the S columns
  // while the previous PV (N = D) still reads them unless N = D.  So P aliases S only for
  // D = 128; for D = 64 it has columns of its own (the commit that announces the next S also
  // covers the previous PV, so P is never rewritten while a PV reads it).
  static constexpr uint32_t kTmP0 = D == 128 ? kTmS0 : 384, kTmP1 = D == 128 ? kTmS1 : 448;
  static_assert(D == 128 || 256 + 2 * D <= 384, "TMEM columns");
  static constexpr uint32_t kTmCols = 512;
};

__device__ __forceinline__ void key_tile(const AttnParams &p, int t, int &row, int &valid) {
  if (t < p.seg_tiles[0]) {
    row = p.seg_row[0] + t * 128;
    valid = min(128, p.seg_len[0] - t * 128);
  } else {
    const int u = t - p.seg_tiles[0];
    row = p.seg_row[1] + u * 128;
    valid = min(128, p.seg_len[1] - u * 128);
  }
}

// A wait used only while tearing down after an abort: ignores the abort flag.
__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Share of the exponentials computed on the FMA pipe (exp2_poly2) instead of MUFU: in every 8
// column pairs of a 128-key tile, the last kEmuPairsPer8 pairs.  MUFU alone (16 per clock per SM)
// needs as long for one tile's 16384 exponentials as the tensor core needs for the other tile's
// two 128x128x128 products, so moving part of them to the FMA pipe shortens the softmax phase.
// The polynomial costs more issue slots than one MUFU op, and the softmax warps share the SM's
// issue slots with the MMA issuer: 2 of 8 measured fastest (3 of 8: +6 %, 4 of 8: +15 %, 1 of 8
// and 0 of 8: +2-3 %).
#ifndef UNSTEP_EMU_PAIRS_PER8
#define UNSTEP_EMU_PAIRS_PER8 2
#endif
constexpr int kEmuPairsPer8 = UNSTEP_EMU_PAIRS_PER8;

// Max of a row's 128 scores: eight independent chains of 3-input max, then a short tree.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[4][32]) {
  float m8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = k >> 1, e0 = (k & 1) * 16;
    float m = fmax3(__uint_as_float(s[c][e0]), __uint_as_float(s[c][e0 + 1]),
                    __uint_as_float(s[c][e0 + 2]));
#pragma unroll
    for (int e = 3; e < 15; e += 2)
      m = fmax3(m, __uint_as_float(s[c][e0 + e]), __uint_as_float(s[c][e0 + e + 1]));
    m8[k] = fmaxf(m, __uint_as_float(s[c][e0 + 15]));
  }
  return fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

// P for one 32-column chunk of a row: p = 2^(s * scale - m), summed into acc (four packed
// accumulators), rounded to bf16 pairs and stored to the 16 TMEM columns at `taddr` (for
// D = 128 the P columns alias the S columns already read).  kMasked: columns >= valid are zero (a segment's
// last, partial tile), all exponentials on MUFU so that masked ones are exactly 0.
template <bool kMasked>
__device__ __forceinline__ void exp_chunk(const uint32_t (&s)[32], int col0, int valid,
                                          uint64_t sc2, uint64_t nm2, uint64_t (&acc)[4],
                                          uint32_t taddr) {
  uint32_t w[16];

#pragma unroll
  for (int pi = 0; pi < 16; ++pi) {
    const uint64_t x2 = ffma2(f2_make(__uint_as_float(s[2 * pi]), __uint_as_float(s[2 * pi + 1])),
                              sc2, nm2);
    uint64_t p2;
    if (!kMasked && (pi & 7) >= 8 - kEmuPairsPer8) {
      p2 = exp2_poly2(x2);
    } else {
      float x0, x1;
      f2_split(x2, x0, x1);
      float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      if (kMasked) {
        p0 = (col0 + 2 * pi < valid) ? p0 : 0.f;
        p1 = (col0 + 2 * pi + 1 < valid) ? p1 : 0.f;
      }
      p2 = f2_make(p0, p1);
    }
    acc[pi & 3] = fadd2(acc[pi & 3], p2);
    float p0, p1;
    f2_split(p2, p0, p1);
    w[pi] = pack_bf16x2(p0, p1);
  }
  tmem_st16(taddr, w);
}

// ---------------------------------------------------------------------------------------------
// Work decomposition.  A unit is one (stream, head) with two 128-row query tiles over all of the
// window's key tiles; units are numbered head-major, u = (b*H + h)*n_pairs + pair.  The grid is
// persistent: CTA c first takes whole units in dp_waves data-parallel waves (unit w*grid + c, so
// that concurrent CTAs share a head's K/V in L2), then its share of the remaining tail units'
// key tiles, cut evenly over g_sk CTAs (stream-K).  A tail unit split between CTAs leaves each
// piece's unnormalised O, running max and row sum in a scratch slot; the last CTA to finish a
// piece of it (an atomic count per unit and query tile) merges them.  No CTA waits for another.
// ---------------------------------------------------------------------------------------------
struct Seg {
  int u;        // unit
  int k0, k1;   // key tiles [k0, k1) of the unit
  int slot;     // scratch slot of a partial segment (2c or 2c+1), -1 when the unit is whole
};

__device__ __forceinline__ long long sk_lo(const AttnParams &p, int c) {
  return static_cast<long long>(c) * p.w_tail / p.g_sk;
}

// This CTA's share [lo, hi) of the tail's key tiles, computed once.
struct SkRange {
  long long lo, hi;
  long long u_rel0;  // tail unit holding tile lo
};

__device__ __forceinline__ SkRange sk_range(const AttnParams &p, int c) {
  SkRange r{0, 0, 0};
  if (c < p.g_sk) {
    r.lo = sk_lo(p, c);
    r.hi = sk_lo(p, c + 1);
    r.u_rel0 = r.lo / p.n_tiles;
  }
  return r;
}

// The q-th segment of CTA c; false when the CTA has no more.
__device__ __forceinline__ bool get_seg(const AttnParams &p, int c, const SkRange &sk, int q,
                                        Seg &s) {
  if (q < p.dp_waves) {
    s.u = q * p.grid + c;
    s.k0 = 0;
    s.k1 = p.n_tiles;
    s.slot = -1;
    return true;
  }
  const int r = q - p.dp_waves;
  if (c >= p.g_sk || r > 1) return false;
  const long long u_rel = sk.u_rel0 + r;
  const long long us = u_rel * p.n_tiles;
  if (us >= sk.hi) return false;
  s.u = p.u_tail0 + static_cast<int>(u_rel);
  s.k0 = static_cast<int>((sk.lo > us ? sk.lo : us) - us);
  s.k1 = static_cast<int>((sk.hi < us + p.n_tiles ? sk.hi : us + p.n_tiles) - us);
  s.slot = (s.k0 == 0 && s.k1 == p.n_tiles) ? -1 : 2 * c + r;
  return true;
}

struct UnitPos {
  int b, h, bh, q0;
  bool has1;
};

__device__ __forceinline__ UnitPos unit_pos(const AttnParams &p, int u) {
  UnitPos x;
  x.bh = static_cast<int>(fdiv(static_cast<uint32_t>(u), p.div_pairs));
  const int pair = u - x.bh * p.n_pairs;
  x.b = static_cast<int>(fdiv(static_cast<uint32_t>(x.bh), p.div_heads));
  x.h = x.bh - x.b * p.H;
  x.q0 = pair * 256;
  x.has1 = x.q0 + 128 < p.L;
  return x;
}

// Coefficient rows the query rotation reads: the chunk's temporal rows (frames frame0 ..) and
// the h and w tables, either staged in shared memory (t row i = frame frame0 + i) or in global
// memory (t row = absolute frame).
struct QTabs {
  const float2 *t, *h, *w;
  int t_base;  // added to the chunk-relative frame i
};

// Rotation of one query tile in shared memory (kRopeQ): the warpgroup's warp wq takes rows
// wq, wq + 4, ...; a row is D channels in D/64 boxes of 128 bytes (128-byte swizzle: 16-byte
// chunk c of row r sits at chunk c ^ (r mod 8)), and lane ln takes channels
// [ln*D/32, (ln+1)*D/32), i.e. D/64 channel pairs, so that a warp's coefficient reads are one
// contiguous run per axis block and its shared-memory accesses are conflict-free.  Rows past the
// chunk end (TMA zero fill) are left as loaded.  The arithmetic is the append kernel's, so the
// tile holds exactly what unstep_rope_kv_append would have written to q.
template <int D>
__device__ __forceinline__ void rope_q_tile(const AttnParams &p, const QTabs &tabs,
                                            uint8_t *tile, int l0, int wq, int lane) {
  constexpr int kPairs = D / 64;              // channel pairs per lane
  const int ch0 = lane * (D / 32);            // first channel of the lane
  const int box = ch0 >> 6;
  const int byte_in_box = (ch0 & 63) * 2;
  const int chunk = byte_in_box >> 4, sub = byte_in_box & 15;
  const float2 *tb[kPairs];
  int stride[kPairs], axis[kPairs];
#pragma unroll
  for (int u = 0; u < kPairs; ++u) {
    const int pr = ch0 / 2 + u;
    if (pr < p.half_t) {
      axis[u] = 0;
      tb[u] = tabs.t + pr;
      stride[u] = p.half_t;
    } else if (pr < p.half_t + p.half_h) {
      axis[u] = 1;
      tb[u] = tabs.h + (pr - p.half_t);
      stride[u] = p.half_h;
    } else {
      axis[u] = 2;
      tb[u] = tabs.w + (pr - p.half_t - p.half_h);
      stride[u] = p.half_w;
    }
  }
  // 32 rows per warp in batches of kBatch: every load of a batch is issued before its first
  // use; rows past the chunk end decode a clamped position and skip only their store
  constexpr int kBatch = 8;
  const int n_live = min(128, p.L - l0);
#pragma unroll 1
  for (int r0 = 0; r0 < 128; r0 += 4 * kBatch) {
    float2 cs[kBatch][kPairs];
    uint32_t v[kBatch][kPairs];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int r = r0 + 4 * b + wq;
      const uint32_t l = static_cast<uint32_t>(l0 + min(r, n_live - 1));
      const uint32_t i = fdiv(l, p.div_tf);
      const uint32_t tok = l - i * static_cast<uint32_t>(p.Tf);
      const uint32_t y = fdiv(tok, p.div_wg);
      const uint32_t x = tok - y * static_cast<uint32_t>(p.Wg);
#pragma unroll
      for (int u = 0; u < kPairs; ++u) {
        const int pos = axis[u] == 0 ? static_cast<int>(i) + tabs.t_base
                                     : (axis[u] == 1 ? static_cast<int>(y) : static_cast<int>(x));
        cs[b][u] = tb[u][pos * stride[u]];
      }
      const uint8_t *a = tile + box * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4) + sub;
      if constexpr (kPairs == 2) {
        const uint2 w2 = *reinterpret_cast<const uint2 *>(a);
        v[b][0] = w2.x;
        v[b][kPairs - 1] = w2.y;
      } else {
        v[b][0] = *reinterpret_cast<const uint32_t *>(a);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int r = r0 + 4 * b + wq;
      if (r >= n_live) continue;
      uint8_t *a = tile + box * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4) + sub;
      if constexpr (kPairs == 2) {
        *reinterpret_cast<uint2 *>(a) = make_uint2(rope_rotate_pair(v[b][0], cs[b][0]),
                                                   rope_rotate_pair(v[b][1], cs[b][1]));
      } else {
        *reinterpret_cast<uint32_t *>(a) = rope_rotate_pair(v[b][0], cs[b][0]);
      }
    }
  }
}

// Named barrier of one softmax warpgroup (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void wg_sync(int i) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + i) : "memory");
}

// Cold per-segment work of a softmax thread (one query row).  Inlined by default (measured
// faster on B200 than out-of-line calls, whose register saves cost more than they free);
// UNSTEP_COLD_NOINLINE moves them out of line.
#ifdef UNSTEP_COLD_NOINLINE
#define UNSTEP_COLD_FN __device__ __noinline__
#else
#define UNSTEP_COLD_FN __device__ __forceinline__
#endif

// O row / l -> bf16, stored to dst (the row's D channels) when `live` (row < L).
template <int D>
UNSTEP_COLD_FN void store_row(uint32_t tO, float inv, __nv_bfloat16 *dst, bool live) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + c * 32, o);
    tmem_wait_ld();
    if (live) {
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
  }
}

// A piece of a split unit: the row's unnormalised O, running max and row sum, column-major in
// the slot (consecutive rows -> consecutive addresses), through L2.
template <int D>
UNSTEP_COLD_FN void write_piece(uint32_t tO, float *mine, int row, float m_run,
                                         float l_run) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) __stcg(mine + (c * 32 + e) * 128 + row, __uint_as_float(o[e]));
  }
  __stcg(mine + D * 128 + row, m_run);
  __stcg(mine + D * 128 + 128 + row, l_run);
  __threadfence();
}

// Scratch slot holding CTA c's piece of the tail unit whose first tile is t0 (tail-relative):
// its first piece if its range starts inside the unit, else its second.
__device__ __forceinline__ int piece_slot(const AttnParams &p, int c, long long t0) {
  return 2 * c + (sk_lo(p, c) >= t0 ? 0 : 1);
}

// Merge the pieces of CTAs c_first..c_last for one row: rescale each to the common max,
// sum, normalise, store.  The merge only reads L2 and is bound by its latency: each step takes
// one piece's max and kMergeCB of its channels in one round trip, so the number of round trips
// is (D / kMergeCB) x pieces.  Piece c > c_first is the first piece of its CTA (slot 2c): its
// range starts inside the unit; only c_first's slot needs the range test.
#ifndef UNSTEP_MERGE_CB
#define UNSTEP_MERGE_CB 32
#endif
template <int D>
UNSTEP_COLD_FN void merge_row(const AttnParams &p, int i, int row, long long t0,
                              int c_first, int c_last, __nv_bfloat16 *dst, bool live) {
  constexpr int kTileFloats = D * 128 + 256;
  constexpr int kCB = UNSTEP_MERGE_CB;
  __threadfence();
  const int first_slot = piece_slot(p, c_first, t0);
  auto piece = [&](int c) {
    return p.slots + static_cast<long long>(c == c_first ? first_slot : 2 * c) * p.slot_floats +
           i * kTileFloats + row;
  };
  float M = -INFINITY;
#pragma unroll 1
  for (int c = c_first; c <= c_last; ++c) M = fmaxf(M, __ldcg(piece(c) + D * 128));
  float Lsum = 0.f;
#pragma unroll 1
  for (int c = c_first; c <= c_last; ++c) {
    const float *src = piece(c);
    Lsum += __ldcg(src + D * 128 + 128) * ex2_approx(__ldcg(src + D * 128) - M);
  }
  const float inv = 1.f / Lsum;
#pragma unroll 1
  for (int cb = 0; cb < D / kCB; ++cb) {
    float a[kCB];
#pragma unroll
    for (int e = 0; e < kCB; ++e) a[e] = 0.f;
#pragma unroll 1
    for (int c = c_first; c <= c_last; ++c) {
      const float *src = piece(c);
      const float w = ex2_approx(__ldcg(src + D * 128) - M);
#pragma unroll
      for (int e = 0; e < kCB; ++e) a[e] = fmaf(w, __ldcg(src + (cb * kCB + e) * 128), a[e]);
    }
    if (live) {
      uint4 *d4 = reinterpret_cast<uint4 *>(dst + cb * kCB);
#pragma unroll
      for (int q = 0; q < kCB / 8; ++q)
        d4[q] = make_uint4(pack_bf16x2(a[8 * q] * inv, a[8 * q + 1] * inv),
                           pack_bf16x2(a[8 * q + 2] * inv, a[8 * q + 3] * inv),
                           pack_bf16x2(a[8 * q + 4] * inv, a[8 * q + 5] * inv),
                           pack_bf16x2(a[8 * q + 6] * inv, a[8 * q + 7] * inv));
    }
  }
}

// kRopeQ: q is un-rotated; both softmax warpgroups rotate their query tiles in shared memory.
template <int D, bool kRopeQ>
__global__ void __launch_bounds__(kThreads, 1)
    window_attn_kernel(const __grid_constant__ CUtensorMap tmq,
                       const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const AttnParams p) {
  using C = Cfg<D, kRopeQ>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kSmemBar);
  uint64_t *q_full = bars;
  uint64_t *q_empty = bars + 1;
  uint64_t *full = bars + 2;
  uint64_t *empty = full + NS;
  uint64_t *s_full = empty + NS;
  uint64_t *p_ready = s_full + 2;
  uint64_t *o_done = p_ready + 2;
  uint64_t *drain = o_done + 2;
  uint64_t *q_rot = drain + 1;    // query tiles rotated by both warpgroups (kRopeQ)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(q_rot + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *merge_word = reinterpret_cast<volatile int *>(tmem_slot + 2);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(q_rot, 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, C::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, p.dev_error, p.wait_limit_ns};
  constexpr int E = UNSTEP_ERR_DEVICE_TIMEOUT;
  const SkRange sk = sk_range(p, cta);

  if (warp >= 8) {
    regs_release<kRegsIo>();
    if (warp == 8) {
      // -------------------------------------------------------------- TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        int n = 0;   // key tiles (K/V stages) issued
        int nq = 0;  // Q loads issued
        bool ok = true;
        Seg sg;
        for (int q = 0; ok && get_seg(p, cta, sk, q, sg); ++q) {
          const UnitPos up = unit_pos(p, sg.u);
          if (q > 0 && !(ok = wait_bounded(q_empty, static_cast<uint32_t>(q - 1) & 1u, g, E)))
            break;
          const int ntq = up.has1 ? 2 : 1;
          if (kDebugChecks &&
              !debug_check(up.bh < p.B * p.H && p.b0 + up.b < p.act_B && p.h0 + up.h < p.act_H &&
                               up.q0 + (ntq - 1) * 128 < p.L && sg.k0 >= 0 && sg.k0 < sg.k1 &&
                               sg.k1 <= p.n_tiles,
                           p.dev_error)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(q_full, ntq * C::kTileBytes);
          for (int t = 0; t < ntq; ++t)
            for (int c = 0; c < C::kBoxes; ++c)
              tma_load_4d(smem + C::kSmemQ + t * C::kTileBytes + c * 16384, &tmq, q_full,
                          c * 64, p.h0 + up.h, up.q0 + t * 128, p.b0 + up.b);
          nq = q + 1;
          for (int kt = sg.k0; ok && kt < sg.k1; ++kt) {
            int row, valid;
            key_tile(p, kt, row, valid);
            if (kDebugChecks &&
                !debug_check(row >= 0 && row < p.rows && valid >= 1 && valid <= 128,
                             p.dev_error)) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            // one stage per key tile: its K tile and its V tile under one barrier
            const int s = n % NS;
            const uint32_t r = static_cast<uint32_t>(n / NS);
            if (!(ok = wait_bounded(&empty[s], (r & 1u) ^ 1u, g, E))) break;
            mbar_arrive_expect_tx(&full[s], C::kStageBytes);
            uint8_t *st = smem + C::kSmemKV + s * C::kStageBytes;
            for (int c = 0; c < C::kBoxes; ++c)
              tma_load_3d(st + c * 16384, &tmk, &full[s], c * 64, row, up.bh);
            for (int c = 0; c < C::kBoxes; ++c)
              tma_load_3d(st + C::kTileBytes + c * 16384, &tmv, &full[s], c * 64, row, up.bh);
            ++n;
          }
        }
        if (*abort_flag) {
          // let every copy still in flight land before the CTA's shared memory is released
          for (int k = max(0, n - NS); k < n; ++k)
            wait_drain(&full[k % NS], static_cast<uint32_t>(k / NS) & 1u);
          if (nq > 0) wait_drain(q_full, static_cast<uint32_t>(nq - 1) & 1u);
        }
      }
      __syncwarp();
    } else if (warp == 9) {
      // -------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);
        const uint32_t sQ = smem_u32(smem + C::kSmemQ);
        const uint32_t sKV = smem_u32(smem + C::kSmemKV);
        // descriptors as 32-bit halves: the high half (stride offset, version, swizzle) is the
        // same for every operand of a kind; only the start address in the low half moves
        const uint32_t kHiK = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
        const uint32_t kHiV = static_cast<uint32_t>(sdesc_sw128(0, 16384, 1024) >> 32);
        const uint32_t loQ = static_cast<uint32_t>(sdesc_sw128(sQ, 16, 1024));
        const uint32_t loK = static_cast<uint32_t>(sdesc_sw128(sKV, 16, 1024));
        const uint32_t loV =
            static_cast<uint32_t>(sdesc_sw128(sKV + C::kTileBytes, 16384, 1024));
        auto qk = [&](int t, int s) {
          const uint32_t dS = tmem + (t ? C::kTmS1 : C::kTmS0);
          const uint32_t qa = loQ + static_cast<uint32_t>(t * (C::kTileBytes >> 4));
          const uint32_t kb = loK + static_cast<uint32_t>(s * (C::kStageBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = static_cast<uint32_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            umma_ss(dS, f2u64(qa + off, kHiK), f2u64(kb + off, kHiK), kIdQK, kk > 0 ? 1u : 0u);
          }
        };
        auto pv = [&](int t, int s, bool acc) {
          const uint32_t dO = tmem + (t ? C::kTmO1 : C::kTmO0);
          const uint32_t aP = tmem + (t ? C::kTmP1 : C::kTmP0);
          const uint32_t vb = loV + static_cast<uint32_t>(s * (C::kStageBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(dO, aP + kk * 8, f2u64(vb + static_cast<uint32_t>(kk * (2048 >> 4)), kHiV),
                    kIdPV, (acc || kk > 0) ? 1u : 0u);
        };
        auto wait_full = [&](int k) {
          return wait_bounded(&full[k % NS], static_cast<uint32_t>(k / NS) & 1u, g, E);
        };
        // Per key tile the issuer waits three times (the next stage, P0, P1) and commits three
        // times (S0, S1, the stage); o_done is committed only after a segment's last PV, since
        // the commit that announces S(j) already covers PV(j-1) for a softmax that rescales O.
        int n = 0;                      // key tiles (stages) consumed
        uint32_t done0 = 0, done1 = 0;  // PVs issued per query tile (barrier phases)
        bool ok = true;
        Seg sg;
        for (int q = 0; ok && get_seg(p, cta, sk, q, sg); ++q) {
          const bool has1 = unit_pos(p, sg.u).has1;
          const int ntl = sg.k1 - sg.k0;
          if (!(ok = wait_bounded(kRopeQ ? q_rot : q_full, static_cast<uint32_t>(q) & 1u, g, E)))
            break;
          if (!(ok = wait_full(n))) break;
          tc_fence_after();
          qk(0, n % NS);
          umma_commit(&s_full[0]);
          if (has1) {
            qk(1, n % NS);
            umma_commit(&s_full[1]);
          }
          if (ntl == 1) umma_commit(q_empty);
          for (int j = 0; j < ntl; ++j) {
            const int st = (n + j) % NS, nst = (n + j + 1) % NS;
            const bool more = j + 1 < ntl;
            if (!(ok = wait_bounded(&p_ready[0], done0 & 1u, g, E))) break;
            tc_fence_after();
            pv(0, st, j > 0);
            if (!more) umma_commit(&o_done[0]);
            ++done0;
            if (more) {
              if (!(ok = wait_full(n + j + 1))) break;
              tc_fence_after();
              qk(0, nst);
              umma_commit(&s_full[0]);
            }
            if (has1) {
              if (!(ok = wait_bounded(&p_ready[1], done1 & 1u, g, E))) break;
              tc_fence_after();
              pv(1, st, j > 0);
              if (!more) umma_commit(&o_done[1]);
              ++done1;
            }
            umma_commit(&empty[st]);  // key tile j's K and V are read for the last time
            if (more) {
              if (has1) {
                qk(1, nst);
                umma_commit(&s_full[1]);
              }
              if (j + 2 == ntl) umma_commit(q_empty);  // the segment's last QK^T is issued
            }
          }
          n += ntl;
        }
        // every MMA issued above has completed once `drain` flips
        umma_commit(drain);
        wait_drain(drain, 0);
      }
      __syncwarp();
    }
  } else {
    regs_claim<kRegsSoftmax>();
    // ---------------------------------------------------------------- softmax + epilogue
    const int i = warp >> 2;          // query tile of this warpgroup
    const int wq = warp & 3;          // TMEM lane quarter
    const int row = threadIdx.x & 127;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + (i ? C::kTmS1 : C::kTmS0);
    const uint32_t tP = tmem + lane_base + (i ? C::kTmP1 : C::kTmP0);
    const uint32_t tO = tmem + lane_base + (i ? C::kTmO1 : C::kTmO0);
    const float scale = p.scale_log2;
    constexpr int kTileFloats = D * 128 + 256;  // one query tile of a scratch slot
    uint32_t cnt = 0;                           // key tiles this warpgroup has processed
    uint32_t n_seg = 0;                         // segments of this query tile completed
    bool ok = true;
    QTabs qt{p.tab_t, p.tab_h, p.tab_w, p.frame0};
    if constexpr (kRopeQ) {
      if (p.tab_smem) {
        // the chunk's coefficient rows into shared memory, once per CTA, by both warpgroups
        float2 *st = reinterpret_cast<float2 *>(smem + C::kSmemTab);
        const int nt = p.frames * p.half_t, nh = (p.Tf / p.Wg) * p.half_h, nw = p.Wg * p.half_w;
        const float2 *gt = p.tab_t + static_cast<long long>(p.frame0) * p.half_t;
        // all of a thread's loads are issued before its stores (first touch: HBM latency once)
        constexpr int kPer = kQRopeTabBytes / 8 / 256;
        float2 tv[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
          const int e = threadIdx.x + 256 * k;
          if (e < nt + nh + nw)
            tv[k] = e < nt ? gt[e] : (e < nt + nh ? p.tab_h[e - nt] : p.tab_w[e - nt - nh]);
        }
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
          const int e = threadIdx.x + 256 * k;
          if (e < nt + nh + nw) st[e] = tv[k];
        }
        qt = QTabs{st, st + nt, st + nt + nh, 0};
        asm volatile("bar.sync 3, 256;" ::: "memory");
      }
    }
    Seg sg;
    // Every segment is walked even after an abort (the work is skipped), so that the named
    // barriers of the warpgroup are always reached by all of its threads.
    for (int q = 0; get_seg(p, cta, sk, q, sg); ++q) {
      const UnitPos up = unit_pos(p, sg.u);
      if constexpr (kRopeQ) {
        // every segment's query tiles pass through both warpgroups before the MMA issuer may
        // read them; warpgroup 1 takes part even when the segment has no second tile, so that
        // every waiter on q_full observes its phases one by one
        if (ok) ok = __all_sync(kFull, wait_bounded(q_full, static_cast<uint32_t>(q) & 1u, g, E));
        if (ok && (i == 0 || up.has1))
          rope_q_tile<D>(p, qt, smem + C::kSmemQ + i * C::kTileBytes, up.q0 + i * 128, wq, lane);
        fence_proxy_async_smem();
        mbar_arrive(q_rot);
      }
      if (i == 1 && !up.has1) continue;
      const int ntl = sg.k1 - sg.k0;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; ok && j < ntl; ++j) {
        int krow, valid;
        key_tile(p, sg.k0 + j, krow, valid);
        ok = __all_sync(kFull, wait_bounded(&s_full[i], cnt & 1u, g, E));
        if (!ok) break;
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, s[c]);
        tmem_wait_ld();
        const bool masked = valid < 128;
        if (masked) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e >= valid) s[c][e] = __float_as_uint(-INFINITY);
        }
        const float mt = row_max128(s) * scale;
        if (j == 0) {
          m_run = mt;
        } else if (__any_sync(kFull, mt > m_run + 8.f)) {
          const float m_new = fmaxf(m_run, mt);
          const float f = ex2_approx(m_run - m_new);
          l_run *= f;
          m_run = m_new;
          // PV(j-1) has completed: the commit that announced S(j) was issued after it
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tO + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st16(tO + c * 16, o);
          }
          tmem_wait_st();
        }
        const uint64_t sc2 = f2_make(scale, scale);
        const uint64_t nm2 = f2_make(-m_run, -m_run);
        uint64_t acc[4] = {0, 0, 0, 0};
        if (!masked) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            exp_chunk<false>(s[c], c * 32, 128, sc2, nm2, acc, tP + c * 16);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            exp_chunk<true>(s[c], c * 32, valid, sc2, nm2, acc, tP + c * 16);
        }
        float a0, a1;
        f2_split(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
        l_run += a0 + a1;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[i]);
        ++cnt;
      }
      // o_done[i] completes once per segment of this query tile, after its last PV
      if (ok) ok = __all_sync(kFull, wait_bounded(&o_done[i], n_seg & 1u, g, E));
      if (ok) tc_fence_after();
      ++n_seg;
      const int l = up.q0 + i * 128 + row;
      if (kDebugChecks &&
          !debug_check(p.b0 + up.b < p.act_B && p.h0 + up.h < p.act_H &&
                           (sg.slot < 0 || (sg.slot < 2 * p.grid && 2 * sg.u + i < 2 * p.n_units)),
                       p.dev_error)) {
        *abort_flag = 1;
        ok = false;
      }
      __nv_bfloat16 *dst =
          static_cast<__nv_bfloat16 *>(p.out) +
          ((static_cast<long long>(p.b0 + up.b) * p.L + l) * p.act_H + p.h0 + up.h) * D;
      if (sg.slot < 0) {
        if (ok) store_row<D>(tO, 1.f / l_run, dst, l < p.L);  // whole unit: normalise, store
        continue;
      }
      // piece of a split unit: leave it in the CTA's slot, count it, and merge if it was last
      if (ok)
        write_piece<D>(tO, p.slots + static_cast<long long>(sg.slot) * p.slot_floats +
                               i * kTileFloats, row, m_run, l_run);
      wg_sync(i);
      const long long t0 = static_cast<long long>(sg.u - p.u_tail0) * p.n_tiles;
      const int c_first = static_cast<int>(((t0 + 1) * p.g_sk - 1) / p.w_tail);
      const int c_last = static_cast<int>(((t0 + p.n_tiles) * p.g_sk - 1) / p.w_tail);
      if (threadIdx.x == 128 * i) {
        int last = 0;
        if (!*abort_flag) {
          // count this piece; the count word carries the launch's epoch in its high bits, so a
          // word left behind by an aborted launch is never mistaken for a current count
          unsigned *ctr = p.counters + 2 * sg.u + i;
          const unsigned ep = p.epoch << 8;
          unsigned old = *reinterpret_cast<volatile unsigned *>(ctr), nw;
          while (true) {
            nw = ((old & 0xFFFFFF00u) == ep) ? old + 1 : (ep | 1u);
            const unsigned seen = atomicCAS(ctr, old, nw);
            if (seen == old) break;
            old = seen;
          }
          last = static_cast<int>(nw & 0xFFu) == c_last - c_first + 1;
          if (last) atomicExch(ctr, 0u);
        }
        merge_word[i] = last;
      }
      wg_sync(i);
      bool merge = ok && merge_word[i] != 0;
      if (kDebugChecks && merge &&
          !debug_check(c_first >= 0 && c_first <= c_last && c_last < p.g_sk, p.dev_error)) {
        *abort_flag = 1;
        merge = false;
      }
      wg_sync(i);  // merge_word is rewritten by the next piece
      if (merge) merge_row<D>(p, i, row, t0, c_first, c_last, dst, l < p.L);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

__global__ void wait_timeout_selftest_kernel(int *dev_error, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives on it
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitGuard g{&abort_flag, dev_error, limit_ns};
  const bool ok = __all_sync(kFull, wait_bounded(&bar, 0, g, UNSTEP_ERR_DEVICE_TIMEOUT));
  if (ok && threadIdx.x == 0) atomicCAS(dev_error, 0, 1);  // impossible: flags a broken wait
}

__global__ void exp2_selftest_kernel(const float *x, float *y_poly, float *y_mufu, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = 2 * i;
  if (j >= n) return;
  const float x0 = x[j], x1 = (j + 1 < n) ? x[j + 1] : 0.f;
  float p0, p1;
  f2_split(exp2_poly2(f2_make(x0, x1)), p0, p1);
  y_poly[j] = p0;
  y_mufu[j] = ex2_approx(x0);
  if (j + 1 < n) {
    y_poly[j + 1] = p1;
    y_mufu[j + 1] = ex2_approx(x1);
  }
}

template <int D, bool kRopeQ>
cudaError_t launch_d(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     const AttnParams &p, cudaStream_t stream) {
  using C = Cfg<D, kRopeQ>;
  // the shared-memory opt-in is per device; remember which devices have it
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(__atomic_load_n(&attr_set, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(window_attn_kernel<D, kRopeQ>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
    if (e != cudaSuccess) return e;
    if (dev < 64) __atomic_fetch_or(&attr_set, bit, __ATOMIC_RELEASE);
  }
  if (p.grid < 1) return cudaErrorInvalidConfiguration;
  window_attn_kernel<D, kRopeQ>
      <<<static_cast<unsigned>(p.grid), kThreads, C::kSmemAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn(int D, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                               const CUtensorMap &tmap_v, const AttnParams &p,
                               cudaStream_t stream) {
  if (D == 128)
    return p.rope_q ? launch_d<128, true>(tmap_q, tmap_k, tmap_v, p, stream)
                    : launch_d<128, false>(tmap_q, tmap_k, tmap_v, p, stream);
  if (D == 64)
    return p.rope_q ? launch_d<64, true>(tmap_q, tmap_k, tmap_v, p, stream)
                    : launch_d<64, false>(tmap_q, tmap_k, tmap_v, p, stream);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------------------------
// Fixed device scratch for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc: code that runs inside a framework or allocator
// that owns every device allocation, or a process that must not grow its device footprint once
// it has started.  For them the attention's split-unit scratch (per-unit counts and the pieces'
// partial results) lives in this buffer, which is part of the library image: every device that
// loads the library holds kStaticScratchBytes of it until the process exits.  Host code cannot
// use the symbol's name as a device address (it names a host-side stand-in), so the address is
// looked up once per device, with that device current, and passed to the kernel.
// ---------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_attn_static_scratch[kStaticScratchBytes];

cudaError_t static_attn_scratch(void **ptr, size_t *bytes) {
  static std::mutex mu;
  static void *addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *a = nullptr;
    e = cudaGetSymbolAddress(&a, g_attn_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = a;
  }
  *ptr = addr[dev];
  *bytes = kStaticScratchBytes;
  return cudaSuccess;
}

cudaError_t launch_exp2_selftest(const float *x, float *y_poly, float *y_mufu, int n,
                                 cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y_poly, y_mufu, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(int *dev_error, uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(dev_error, limit_ns);
  return cudaGetLastError();
}

}  // namespace unstep
