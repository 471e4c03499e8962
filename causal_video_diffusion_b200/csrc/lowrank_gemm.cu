// lowrank_gemm.cu -- the truncated-SVD projections on the Blackwell tensor cores.
//
// UnStep paper (arXiv 2609.32518), abstract and Figure 11 / Table 5: truncated SVD applied to
// the DiT attention's value and output projections (V/O rank retention 0.92).  A projection
// y = x W^T with W ~ U_r S_r V_r^T becomes two products through the rank-r space:
//   t = x w1^T   (w1 = (V_r S_r)^T, [r][in])       y = t w2^T   (w2 = U_r, [out][r])
// Each is C[M][N] = A[M][K] * B[N][K]^T, bf16 operands, fp32 accumulation, bf16 output: a
// persistent grid of one CTA per SM over 128 x 128 output tiles, K in steps of 64 through a
// 6-stage TMA ring (128-byte swizzle), tcgen05.mma M=128 N=128 K=16 into one of two 128-column
// TMEM accumulators, a 4-warp epilogue (thread = TMEM lane = output row) draining one
// accumulator while the products of the next tile fill the other.  Ragged M, N and K tails come
// from TMA zero fill and are not stored.
#include <cuda_bf16.h>

#include "../../include/unstep.h"
#include "gemm.h"
#include "sm100.cuh"

namespace unstep {
namespace {

// kMT 128-row halves per output tile, each its own M=128 product against the same B tile
#ifndef UNSTEP_GEMM_MT
#define UNSTEP_GEMM_MT 2
#endif
constexpr int kMT = UNSTEP_GEMM_MT;
constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = kMT == 1 ? 6 : 4;
constexpr int kThreads = 256;                       // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr int kABytes = kMT * kBM * kBK * 2;        // 16 KB per 128 rows
constexpr int kAccCols = kMT * kBN;                 // TMEM columns of one accumulator set
constexpr int kBBytes = kBN * kBK * 2;              // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kSmemBar = kStages * kStageBytes;
constexpr int kSmemAlloc = kSmemBar + 256 + 1024;
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Persistent: CTA c takes output tiles c, c + grid, ...; tiles are m-major within an n column
// (tile t -> n block t / m_tiles, m block t % m_tiles), two TMEM accumulators alternate so the
// epilogue of one tile overlaps the products of the next.
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tma,
                        const __grid_constant__ CUtensorMap tmb, __nv_bfloat16 *out, int M,
                        int N, int K, int ldc, int *dev_error, uint64_t wait_limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kSmemBar);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;   // [2]
  uint64_t *acc_empty = acc_full + 2;     // [2]
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + kMT * kBM - 1) / (kMT * kBM);
  const int n_tiles = (N + kBN - 1) / kBN;
  const int tiles = m_tiles * n_tiles;
  const int k_steps = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, dev_error, wait_limit_ns};
  constexpr int E = UNSTEP_ERR_DEVICE_TIMEOUT;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tma);
      tma_prefetch_desc(&tmb);
      int n = 0;  // stage fills issued
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t % m_tiles) * (kMT * kBM), n0 = (t / m_tiles) * kBN;
        for (int k = 0; k < k_steps; ++k, ++n) {
          const int s = n % kStages;
          const uint32_t r = static_cast<uint32_t>(n / kStages);
          if (!(ok = wait_bounded(&empty[s], (r & 1u) ^ 1u, g, E))) break;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          uint8_t *st = smem + s * kStageBytes;
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt)
            tma_load_2d(st + mt * (kBM * kBK * 2), &tma, &full[s], k * kBK, m0 + mt * kBM);
          tma_load_2d(st + kABytes, &tmb, &full[s], k * kBK, n0);
        }
      }
      if (*abort_flag)
        for (int k = max(0, n - kStages); k < n; ++k)
          drain_wait(&full[k % kStages], static_cast<uint32_t>(k / kStages) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(kBM, kBN, false, false);
      const uint32_t hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
      const uint32_t lo0 = static_cast<uint32_t>(sdesc_sw128(smem_u32(smem), 16, 1024));
      bool ok = true;
      int n = 0, i = 0;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
        const int acc = i & 1;
        if (!(ok = wait_bounded(&acc_empty[acc], (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g, E)))
          break;
        tc_fence_after();
        const uint32_t d = tmem + acc * kAccCols;
        for (int k = 0; k < k_steps; ++k, ++n) {
          const int s = n % kStages;
          if (!(ok = wait_bounded(&full[s], static_cast<uint32_t>(n / kStages) & 1u, g, E))) break;
          tc_fence_after();
          const uint32_t la = lo0 + static_cast<uint32_t>((s * kStageBytes) >> 4);
          const uint32_t lb = la + static_cast<uint32_t>(kABytes >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
              umma_ss(d + mt * kBN, f2u64(la + mt * ((kBM * kBK * 2) >> 4) + kk * 2, hi),
                      f2u64(lb + kk * 2, hi), kId, (k > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[acc]);
      }
      umma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int row = threadIdx.x - 128;  // TMEM lane = output row
    const uint32_t lane_base = static_cast<uint32_t>((warp - 4) * 32) << 16;
    bool ok = true;
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int acc = i & 1;
      if (ok) ok = __all_sync(kFull, wait_bounded(&acc_full[acc], static_cast<uint32_t>(i >> 1) & 1u, g, E));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int mt = 0; mt < kMT; ++mt) {
      const int m = (t % m_tiles) * (kMT * kBM) + mt * kBM + row, n0 = (t / m_tiles) * kBN;
      const uint32_t src = tmem + lane_base + acc * kAccCols + mt * kBN;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(src + c * 32, o);
        tmem_wait_ld();
        const int n = n0 + c * 32;
        if (m < M && n < N) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1]));
          __nv_bfloat16 *dst = out + static_cast<long long>(m) * ldc + n;
          const int nv = (N - n) >= 32 ? 4 : (N - n) / 8;  // 16-byte groups (N is a multiple of 8)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (v < nv)
              reinterpret_cast<uint4 *>(dst)[v] =
                  make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kAccCols);
  }
}

}  // namespace

cudaError_t launch_gemm_bf16_tn(const CUtensorMap &ta, const CUtensorMap &tb, void *c, int M,
                                int N, int K, int ldc, int *dev_error, cudaStream_t stream) {
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(__atomic_load_n(&attr_set, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(gemm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemAlloc);
    if (e != cudaSuccess) return e;
    if (dev < 64) __atomic_fetch_or(&attr_set, bit, __ATOMIC_RELEASE);
  }
  const long long tiles =
      static_cast<long long>((M + kMT * kBM - 1) / (kMT * kBM)) * ((N + kBN - 1) / kBN);
  if (tiles < 1 || tiles > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  gemm_bf16_tn_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(
      ta, tb, static_cast<__nv_bfloat16 *>(c), M, N, K, ldc, dev_error, kWaitLimitNs);
  return cudaGetLastError();
}

}  // namespace unstep
