// conv3d.cu -- the VAE decoder's causal 3D convolution on the Blackwell tensor cores.
//
// UnStep paper (arXiv 2609.32518), abstract and Table 1 row C2: the decoder runs with an
// optimised memory layout, precision and convolution kernels.  The layer here is the causal
// 3x3x3 convolution of a video decoder, channels-last, bf16 in and out, fp32 accumulation:
//
//   y[b, t, h, x, o] = bias[o] + sum over (dt, dy, dx, c) of
//                      w[o, dt, dy, dx, c] * in[b, t + dt, h + dy - 1, x + dx - 1, c]
//
// where each stream's input carries two history frames in front (output frame t sees input
// frames t .. t + 2) and positions outside the frame read zero.  It is computed as an implicit
// GEMM: M = output positions, N = output channels, K = 27 taps x C_in.  An output tile is 16
// rows x 16 columns of one frame (two halves of 128 positions) by 128 channels; a K step is one
// (dt, dx) tap column and 64 input channels, all three dy taps: its A operand is one TMA box {64
// channels, 16 x, 18 y, 1 frame} of the input (the tile's rows and one halo row on each side) at
// the column's offset -- it lands in shared memory as 288 rows of 128 bytes with the 128-byte
// swizzle, the K-major operand layout, and each (half, dy) operand is 128 consecutive rows of it
// starting at a whole row of 16 positions; the box's out-of-range part (the frame's border, the
// padding) is zero-filled by the TMA unit.  B is each tap's {64 channels x 128 output channels}
// slice of the weights, shared by both halves.  A persistent grid, a TMA ring of whole K steps
// (a step's A box and weight slices under one barrier), tcgen05.mma K=16 per half into one of
// two TMEM accumulator sets, a 4-warp epilogue (thread = TMEM lane = output position of a half)
// adding the bias and storing bf16.  Frames taller than one tile run on CTA pairs (2-CTA
// clusters, cta_group::2, M=256): a pair tile is 32 rows, each CTA loads its own A box and half
// of every weight slice, 60 KB per step and SM instead of 84 KB.  With caller scratch, the tiles
// of the last, partial wave are cut along K over all SMs (stream-K, below).
#include <cuda_bf16.h>

#include "../../include/unstep.h"
#include "conv3d.h"
#include "sm100.cuh"

namespace unstep {
namespace {

// Two 128-position halves per output tile (rows 16 x 16 columns), each its own M=128 product
// against the same weight slice, so that one B load serves 256 positions.  A K step is one
// (dt, dx) tap column and 64 input channels: its A operand is ONE TMA box of the tile's 16 rows
// plus a halo row above and below (18 rows x 16 columns x 64 channels), and the three dy taps
// read it at row offsets dy, dy + 8 -- whole rows of 16 positions, i.e. multiples of 2048 bytes
// in shared memory, so each tap's operand is the same box under a shifted descriptor.  Per K
// step: 36 KB of A and three 16 KB weight slices for six 128x128x64 products.
constexpr int kMT = kConvTileH / 8;
constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kTileH = kConvTileH, kTileW = 16;      // an output tile: 16 rows x 16 columns
constexpr int kBoxH = kTileH + 2;                    // rows of an A box: the tile and its halo
constexpr int kRowBytes = kTileW * kBK * 2;          // one row of 16 positions x 64 channels
constexpr int kABytes = kBoxH * kRowBytes;           // 36 KB
// One stage = one K step: the A box and the step's three weight slices under ONE barrier, so
// that the MMA thread waits once and commits once per 24 products.  A barrier per weight slice
// was 12-15 % slower and separate A and weight rings 2-4 % slower, with deeper rings no faster:
// the synchronisation points per step, not the lookahead, limited the MMA issue.
// One CTA: the step's three weight slices of 128 outputs (16 KB each), 84 KB stages, two in the
// ring.  A CTA pair: each CTA holds 64 outputs of each slice (8 KB), 60 KB stages, three.
template <bool kPair>
struct ConvForm {
  static constexpr int kCta = kPair ? 2 : 1;
  static constexpr int kBBytes = (kBN / kCta) * kBK * 2;
  static constexpr int kStageBytes = kABytes + 3 * kBBytes;
  static constexpr int kStages = kPair ? 3 : 2;
  static constexpr int kSmemBar = kStages * kStageBytes;
  static constexpr int kSmemAlloc = kSmemBar + 256 + 1024;
  static_assert(kStageBytes % 1024 == 0 && kSmemAlloc <= 232448, "stage layout");
};
constexpr int kThreads = 256;                        // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr int kAccCols = kMT * kBN;                  // TMEM columns of one accumulator set
static_assert(kMT == 2 && kABytes % 1024 == 0 && kRowBytes % 1024 == 0, "A box layout");
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Output tile t -> (n block, frame index b*T + t, first row, first column).
struct ConvTile {
  int n0, bt, h0, w0;
};

// With CTA pairs a tile has kCta * 16 rows (p.tiles_h counts such rows) and CTA `rank` of the
// pair takes rows 16 rank .. 16 rank + 15 of it.
template <int kCta>
__device__ __forceinline__ ConvTile conv_tile(const ConvParams &p, int t, uint32_t rank) {
  ConvTile c;
  const int m = t % p.m_tiles;
  c.n0 = (t / p.m_tiles) * kBN;
  c.bt = m / (p.tiles_h * p.tiles_w);
  const int r = m - c.bt * (p.tiles_h * p.tiles_w);
  c.h0 = (r / p.tiles_w) * (kCta * kTileH) + kTileH * static_cast<int>(rank);
  c.w0 = (r % p.tiles_w) * kTileW;
  return c;
}

// ---------------------------------------------------------------------------------------------
// Work list of unit c (a CTA, or a CTA pair walking one list); the grid is persistent.  Without
// a stream-K tail (g_sk = 0) unit c takes tiles c, c + units, ... whole.  With one, it first takes
// its share [lo, hi) of the tail tiles' K steps (at most two pieces, as a share is never longer
// than one tile), then whole tiles w*units + c below tail0.  The tail comes first so that the
// merges of split tiles overlap the whole tiles' main loops instead of ending the launch.  A
// piece that is not a whole tile leaves its fp32 sums in the CTA's slot 2 (kCta c + rank) +
// (piece index); the last of a tile's pieces to finish (an atomic count per tile and rank) sums
// all the pieces' slots in piece order (so that the result does not depend on which piece
// finished last) and stores the tile.  No CTA waits for another.
// ---------------------------------------------------------------------------------------------
struct ConvItem {
  int t;        // output tile
  int k0, k1;   // K steps [k0, k1) of the tile
  int slot;     // scratch slot of a partial piece, -1 when the tile is whole
  long long s0; // first K step of the tile in the tail's numbering (partial pieces only)
};

__device__ __forceinline__ long long conv_sk_lo(const ConvParams &p, int c) {
  return static_cast<long long>(c) * p.w_tail / p.g_sk;
}

struct ConvList {
  long long lo, hi;
  int n_sk;    // tail pieces of this CTA
  int dp_end;  // whole tiles are those below dp_end
};

__device__ __forceinline__ ConvList conv_list(const ConvParams &p, int c, int k_steps) {
  ConvList l{0, 0, 0, p.m_tiles * p.n_tiles};
  if (p.g_sk > 0) {
    l.dp_end = p.tail0;
    if (c < p.g_sk) {
      l.lo = conv_sk_lo(p, c);
      l.hi = conv_sk_lo(p, c + 1);
      if (l.hi > l.lo) l.n_sk = static_cast<int>((l.hi - 1) / k_steps - l.lo / k_steps) + 1;
    }
  }
  return l;
}

// The q-th item of CTA c; false past the last one.
__device__ __forceinline__ bool conv_item(const ConvParams &p, const ConvList &l, int c, int units,
                                          int slot0, int q, int k_steps, ConvItem &it) {
  if (q < l.n_sk) {
    const long long ut = l.lo / k_steps + q;
    const long long s0 = ut * k_steps;
    it.t = p.tail0 + static_cast<int>(ut);
    it.k0 = static_cast<int>(l.lo > s0 ? l.lo - s0 : 0);
    it.k1 = static_cast<int>(l.hi - s0 < k_steps ? l.hi - s0 : k_steps);
    it.slot = (it.k0 == 0 && it.k1 == k_steps) ? -1 : slot0 + q;
    it.s0 = s0;
    return true;
  }
  const long long t = static_cast<long long>(q - l.n_sk) * units + c;
  if (t >= l.dp_end) return false;
  it.t = static_cast<int>(t);
  it.k0 = 0;
  it.k1 = k_steps;
  it.slot = -1;
  it.s0 = 0;
  return true;
}

// Slot of unit c's piece (CTA `rank` of it) of the tail tile whose first step is s0: its first
// piece if its share starts inside the tile, else its second.
template <int kCta>
__device__ __forceinline__ int conv_piece_slot(const ConvParams &p, int c, uint32_t rank,
                                               long long s0) {
  return 2 * (kCta * c + static_cast<int>(rank)) + (conv_sk_lo(p, c) >= s0 ? 0 : 1);
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// A slot holds a piece as [mt][32-channel chunk][8 float4 groups][128 rows][4]: for each chunk
// and group the 128 rows of a half are consecutive, so a warp's 32 rows move 512 contiguous bytes.
__device__ __forceinline__ float4 *slot_group(float *slot, int mt, int cc, int v, int row) {
  return reinterpret_cast<float4 *>(slot) + ((mt * (kBN / 32) + cc) * 8 + v) * kBM + row;
}

// ---------------------------------------------------------------------------------------------
// CTA-pair form (cta_group::2).  A 2-CTA cluster computes a pair tile of 32 rows x 16 columns x
// 128 output channels: CTA r holds rows 16 r .. 16 r + 15 (its own halo A box, as above) and
// loads only output channels 64 r .. 64 r + 63 of each weight slice; one M=256 N=128 K=16 MMA,
// issued by CTA 0, multiplies both CTAs' A rows by the pair's two weight halves, each CTA's TMEM
// receiving its own 128 rows.  Per SM and K step this moves 60 KB (36 KB of A, 24 KB of weights)
// instead of 84 KB for the same six 128x128x64 products.
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(const void *ptr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(ptr)), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// TMA loads into this CTA's shared memory that complete on the barrier at cluster address mbar
// (CTA 0's); no multicast.
__device__ __forceinline__ void tma_load_4d_pair(void *dst, const CUtensorMap *map, uint32_t mbar,
                                                 int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t mbar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive once on the barrier at this shared offset in both CTAs when the pair's earlier MMAs
// have completed
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"(mask)
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair_local(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

template <bool kPair>
__device__ __forceinline__ void conv_body(const CUtensorMap &tmx, const CUtensorMap &tmw,
                                          const ConvParams &p) {
  using F = ConvForm<kPair>;
  constexpr int kCta = F::kCta, kStages = F::kStages, kStageBytes = F::kStageBytes;
  constexpr int kBBytes = F::kBBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + F::kSmemBar);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;   // [2]
  uint64_t *acc_empty = acc_full + 2;     // [2]
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *merge_word = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_rank() : 0u;
  const int unit = static_cast<int>(blockIdx.x) / kCta;    // CTA, or pair, index
  const int units = static_cast<int>(gridDim.x) / kCta;
  const int slot0 = 2 * (kCta * unit + static_cast<int>(rank));  // this CTA's two slots
  const int ncb = p.C_in / kBK;            // 64-channel blocks per tap
  const int k_steps = 9 * ncb;             // (dt, dx) tap columns x channel blocks
  const ConvList list = conv_list(p, unit, k_steps);

  if (threadIdx.x == 0) {
    // pairs: CTA 0's full barriers take its producer's arrival and both CTAs' bytes, its
    // acc_empty barriers both CTAs' epilogue threads; the empty and acc_full barriers of both
    // CTAs take one multicast commit per use
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128 * kCta);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(2 * kAccCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      tmem_alloc(tmem_slot, 2 * kAccCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // both CTAs' barriers and TMEM ready before remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, p.dev_error, p.wait_limit_ns};
  constexpr int E = UNSTEP_ERR_DEVICE_TIMEOUT;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmx);
      tma_prefetch_desc(&tmw);
      int n = 0;  // stages filled
      bool ok = true;
      ConvItem it;
      for (int q = 0; ok && conv_item(p, list, unit, units, slot0, q, k_steps, it); ++q) {
        const ConvTile c = conv_tile<kCta>(p, it.t, rank);
        const int b = c.bt / p.T;
        const int f0 = c.bt + 2 * b;       // input frame of tap dt = 0 (streams hold T + 2)
        for (int k = it.k0; k < it.k1; ++k, ++n) {
          const int col = k / ncb, c0 = (k - col * ncb) * kBK;
          const int dt = col / 3, dx = col % 3;
          const int s = n % kStages;
          if (!(ok = wait_bounded(&empty[s], (static_cast<uint32_t>(n / kStages) & 1u) ^ 1u, g, E)))
            break;
          uint8_t *st = smem + s * kStageBytes;
          // rows h0 - 1 .. h0 + 16 at the tap column's offset: x and y may start at -1 and run
          // past the frame (zero fill outside)
          if constexpr (kPair) {
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kStageBytes);
            const uint32_t fb = peer_addr(&full[s], 0);
            tma_load_4d_pair(st, &tmx, fb, c0, c.w0 + dx - 1, c.h0 - 1, f0 + dt);
            for (int dy = 0; dy < 3; ++dy)
              tma_load_3d_pair(st + kABytes + dy * kBBytes, &tmw, fb, c0, dt * 9 + dy * 3 + dx,
                               c.n0 + (kBN / 2) * static_cast<int>(rank));
          } else {
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_4d(st, &tmx, &full[s], c0, c.w0 + dx - 1, c.h0 - 1, f0 + dt);
            for (int dy = 0; dy < 3; ++dy)
              tma_load_3d(st + kABytes + dy * kBBytes, &tmw, &full[s], c0, dt * 9 + dy * 3 + dx,
                          c.n0);
          }
        }
      }
      // after an abort, let every copy still in flight land before shared memory is released
      // (with pairs CTA 0's barriers count both CTAs' bytes)
      if (*abort_flag && rank == 0)
        for (int k = max(0, n - kStages); k < n; ++k)
          drain_wait(&full[k % kStages], static_cast<uint32_t>(k / kStages) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(kCta * kBM, kBN, false, false);
      const uint32_t hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
      const uint32_t lo0 = static_cast<uint32_t>(sdesc_sw128(smem_u32(smem), 16, 1024));
      bool ok = true;
      int n = 0, i = 0;
      ConvItem it;
      for (; ok && conv_item(p, list, unit, units, slot0, i, k_steps, it); ++i) {
        const int acc = i & 1;
        if (!(ok = wait_bounded(&acc_empty[acc], (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g, E)))
          break;
        tc_fence_after();
        const uint32_t d = tmem + acc * kAccCols;
        for (int k = it.k0; k < it.k1; ++k, ++n) {
          const int s = n % kStages;
          if (!(ok = wait_bounded(&full[s], static_cast<uint32_t>(n / kStages) & 1u, g, E))) break;
          tc_fence_after();
          const uint32_t la = lo0 + static_cast<uint32_t>((s * kStageBytes) >> 4);
#pragma unroll
          for (int dy = 0; dy < 3; ++dy) {
            const uint32_t lb = la + static_cast<uint32_t>((kABytes + dy * kBBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt)
              {
                // half mt (of both CTAs of a pair), tap dy: output row 8 mt + r reads box row
                // 8 mt + r + dy
                const uint64_t ad = f2u64(la + (((8 * mt + dy) * kRowBytes) >> 4) + kk * 2, hi);
                const uint64_t bd = f2u64(lb + kk * 2, hi);
                const uint32_t accum = (k > it.k0 || dy > 0 || kk > 0) ? 1u : 0u;
                if constexpr (kPair)
                  umma_ss_pair(d + mt * kBN, ad, bd, kId, accum);
                else
                  umma_ss(d + mt * kBN, ad, bd, kId, accum);
              }
          }
          if constexpr (kPair) umma_commit_pair(&empty[s]); else umma_commit(&empty[s]);
        }
        if (ok) {
          if constexpr (kPair) umma_commit_pair(&acc_full[acc]); else umma_commit(&acc_full[acc]);
        }
      }
      if constexpr (kPair) umma_commit_pair_local(drain); else umma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int row = threadIdx.x - 128;  // TMEM lane = output position of a 128-position half
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const int hh = row / 16, ww = row % 16;
    // with pairs the accumulator set is handed back on CTA 0's barrier
    const uint32_t peer_empty0 = kPair ? peer_addr(&acc_empty[0], 0) : 0u;
    const uint32_t peer_empty1 = kPair ? peer_addr(&acc_empty[1], 0) : 0u;
    auto release_acc = [&](int a) {
      tc_fence_before();
      if constexpr (kPair)
        mbar_arrive_remote(a ? peer_empty1 : peer_empty0);
      else
        mbar_arrive(&acc_empty[a]);
    };
    bool ok = true;
    int i = 0;
    ConvItem it;
    // After a timeout the four warps keep walking the same list without waiting, so that all
    // of them reach every epi_sync (a warp that left would stall the others there).
    for (; conv_item(p, list, unit, units, slot0, i, k_steps, it); ++i) {
      const int acc = i & 1;
      if (ok)
        ok = __all_sync(kFull, wait_bounded(&acc_full[acc], static_cast<uint32_t>(i >> 1) & 1u, g, E));
      if (ok) tc_fence_after();
      const uint32_t src0 = tmem + lane_base + acc * kAccCols;
      // the first and last unit holding a piece of this tile (partial pieces only)
      int c_first = 0, c_last = 0;
      bool merge = false;
      if (it.slot >= 0) {
        // a piece of a split tile: leave it in this CTA's slot, count it, merge if it was last
        float *mine = p.slots + static_cast<long long>(it.slot) * kConvSlotFloats;
#pragma unroll 1
        for (int mt = 0; ok && mt < kMT; ++mt)
#pragma unroll 1
          for (int cc = 0; cc < kBN / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(src0 + mt * kBN + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int v = 0; v < 8; ++v)
              __stcg(slot_group(mine, mt, cc, v, row),
                     make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3])));
          }
        __threadfence();
        // a warp with ok false has set abort_flag before it arrives here, so row 0 counts only
        // when all four warps hold their sums: a merge implies ok in every warp
        epi_sync();
        c_first = static_cast<int>(((it.s0 + 1) * p.g_sk - 1) / p.w_tail);
        c_last = static_cast<int>(((it.s0 + k_steps) * p.g_sk - 1) / p.w_tail);
        if (row == 0) {
          int last = 0;
          if (!*abort_flag) {
            // the count word carries the launch's epoch in its high bits, so a word left by an
            // aborted launch is never taken for a count of this one
            unsigned *ctr = p.counters + (it.t - p.tail0) * kCta + rank;
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
          *merge_word = last;
        }
        epi_sync();
        merge = *merge_word != 0;
        epi_sync();  // merge_word is written again by the next piece
        if (!merge) {
          if (ok) release_acc(acc);
          continue;
        }
        __threadfence();
      }
      if (!ok) continue;
      const ConvTile c = conv_tile<kCta>(p, it.t, rank);
#pragma unroll 1
      for (int mt = 0; mt < kMT; ++mt) {
      const int h = c.h0 + 8 * mt + hh, x = c.w0 + ww;
      const bool live = h < p.H && x < p.W;
      __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) +
                           ((static_cast<long long>(c.bt) * p.H + h) * p.W + x) * p.C_out;
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t o[32];
        const int nb = c.n0 + cc * 32;
        if (!merge) {
          tmem_ld32(src0 + mt * kBN + cc * 32, o);
          tmem_wait_ld();
        } else {
          // the pieces of this tile (this CTA's rank), its own included, summed in piece order
          // from the slots: the result does not depend on which piece finished last
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
#pragma unroll 1
          for (int cp = c_first; cp <= c_last; ++cp) {
            const float *other =
                p.slots +
                static_cast<long long>(conv_piece_slot<kCta>(p, cp, rank, it.s0)) * kConvSlotFloats;
            float4 r[8];
#pragma unroll
            for (int v = 0; v < 8; ++v)
              r[v] = __ldcg(slot_group(const_cast<float *>(other), mt, cc, v, row));
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              o[4 * v] = __float_as_uint(__uint_as_float(o[4 * v]) + r[v].x);
              o[4 * v + 1] = __float_as_uint(__uint_as_float(o[4 * v + 1]) + r[v].y);
              o[4 * v + 2] = __float_as_uint(__uint_as_float(o[4 * v + 2]) + r[v].z);
              o[4 * v + 3] = __float_as_uint(__uint_as_float(o[4 * v + 3]) + r[v].w);
            }
          }
        }
        if (live && nb < p.C_out) {
          float bv[32];
#pragma unroll
          for (int e = 0; e < 32; ++e)
            bv[e] = (p.bias != nullptr && nb + e < p.C_out) ? __ldg(p.bias + nb + e) : 0.f;
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) + bv[2 * e],
                                __uint_as_float(o[2 * e + 1]) + bv[2 * e + 1]);
          const int nv = (p.C_out - nb) >= 32 ? 4 : (p.C_out - nb) / 8;  // 16-byte groups
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (v < nv)
              reinterpret_cast<uint4 *>(dst + nb)[v] =
                  make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
        }
      }
      }
      release_acc(acc);
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // the pair's MMAs and both epilogues are done with TMEM
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(2 * kAccCols)
                   : "memory");
    else
      tmem_dealloc(tmem, 2 * kAccCols);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    conv3d_causal_kernel(const __grid_constant__ CUtensorMap tmx,
                         const __grid_constant__ CUtensorMap tmw, const ConvParams p) {
  conv_body<false>(tmx, tmw, p);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    conv3d_causal_pair_kernel(const __grid_constant__ CUtensorMap tmx,
                              const __grid_constant__ CUtensorMap tmw, const ConvParams p) {
  conv_body<true>(tmx, tmw, p);
}

}  // namespace

// Sets the kernel's dynamic shared memory once per device.
static cudaError_t conv_set_smem(const void *kernel, int bytes, unsigned long long *done, int dev) {
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev < 64 && (__atomic_load_n(done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) __atomic_fetch_or(done, bit, __ATOMIC_RELEASE);
  return e;
}

cudaError_t launch_conv3d_causal(const CUtensorMap &tmx, const CUtensorMap &tmw,
                                 const ConvParams &p, cudaStream_t stream) {
  static unsigned long long attr_single = 0, attr_pair = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool pair = conv_uses_pair(p.H);
  e = pair ? conv_set_smem(reinterpret_cast<const void *>(conv3d_causal_pair_kernel),
                           ConvForm<true>::kSmemAlloc, &attr_pair, dev)
           : conv_set_smem(reinterpret_cast<const void *>(conv3d_causal_kernel),
                           ConvForm<false>::kSmemAlloc, &attr_single, dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int cta = pair ? 2 : 1;
  ConvParams q = p;
  q.tail0 = 0;
  q.g_sk = 0;
  q.w_tail = 0;
  if (pair) {
    // tiles of 32 rows, CTA r of the pair taking rows 16 r .. 16 r + 15
    q.tiles_h = (p.H + 2 * kTileH - 1) / (2 * kTileH);
    q.m_tiles = p.B * p.T * q.tiles_h * p.tiles_w;
  }
  const long long tiles = static_cast<long long>(q.m_tiles) * q.n_tiles;
  if (tiles < 1 || tiles > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  const int units_max = sms / cta;
  if (units_max < 1) return cudaErrorInvalidConfiguration;
  const int units = static_cast<int>(tiles < units_max ? tiles : units_max);
  // stream-K over the tiles that do not fill a last whole wave, when the caller gave scratch:
  // each tail tile is cut into at most kMaxSplit pieces (the merge reads the other pieces from
  // L2) of at least kMinShare K steps (a piece's fp32 write-back and merge cost about as much as
  // a few dozen 64-channel taps: tiles of 27 taps measured slower split than whole).  The split
  // needs more units (CTAs or pairs) than tail tiles, and a share is then never longer than one
  // tile.  Slots: 2 per CTA; count words: one per tail tile and CTA of a unit (< SMs).
  constexpr int kMaxSplit = 4;
  constexpr long long kMinShare = 16;  // K steps of three taps each
  const int tail = static_cast<int>(tiles % units);
  if (p.counters != nullptr && p.slots != nullptr && tiles > units && tail > 0) {
    const int k_steps = 9 * (p.C_in / kBK);
    const long long w_tail = static_cast<long long>(tail) * k_steps;
    long long g = w_tail / kMinShare;
    if (g > static_cast<long long>(tail) * kMaxSplit) g = static_cast<long long>(tail) * kMaxSplit;
    if (g > units) g = units;
    if (g > tail) {
      q.tail0 = static_cast<int>(tiles - tail);
      q.g_sk = static_cast<int>(g);
      q.w_tail = w_tail;
    }
  }
  if (pair)
    conv3d_causal_pair_kernel<<<2 * units, kThreads, ConvForm<true>::kSmemAlloc, stream>>>(tmx, tmw,
                                                                                        q);
  else
    conv3d_causal_kernel<<<units, kThreads, ConvForm<false>::kSmemAlloc, stream>>>(tmx, tmw, q);
  return cudaGetLastError();
}

}  // namespace unstep
