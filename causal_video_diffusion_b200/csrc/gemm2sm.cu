// gemm2sm.cu -- C = A B^T on CTA pairs (tcgen05.mma.cta_group::2): the projections' GEMM.
//
// Same product as lowrank_gemm.cu (bf16 in, fp32 accumulation, bf16 out; the truncated-SVD V/O
// projections of the UnStep paper, abstract and Figure 11 / Table 5), on 2-CTA clusters: a pair
// computes a 256 x 256 output tile with one tcgen05.mma M=256 N=256 K=16 per 16-deep step,
// issued by CTA 0 of the pair.  Each CTA of the pair holds its own 128 rows of A and 128 rows of
// B for every 64-deep K step (16 KB + 16 KB), so an SM moves 32 KB per K step for 128 x 256 x 64
// products, two thirds of what one SM alone needs for the same work.  D lives in each CTA's TMEM
// (its 128 rows x 256 columns, two accumulator sets alternating).
//
// Handshake of the pair:
//   * both CTAs' TMA loads complete on CTA 0's stage barrier, which CTA 0's producer arms for the
//     bytes of both;
//   * CTA 0's MMA thread commits to the stage's "empty" barrier and to "acc_full" in both CTAs
//     (multicast commit), so each producer refills its own stage and each epilogue drains its
//     own rows;
//   * each epilogue thread arrives on CTA 0's "acc_empty" (128 local + 128 remote arrivals) once
//     it has read its row of the accumulator out of TMEM;
//   * TMEM is allocated and freed by warp 1 of both CTAs together; the pair meets at cluster
//     barriers after set-up and before TMEM is freed.
// Epilogue: each of the four epilogue warps owns 32 rows; per 64-column chunk it rounds its rows
// to bf16 into a 4 KB staging buffer in shared memory (the 128-byte-swizzled layout of a 64 x 32
// TMA box) and one lane stores the box with a bulk tensor copy.  Two buffers per warp alternate,
// so the rounding of one chunk overlaps the store of the previous one.
// Launch overlap: the kernel is launched with programmatic stream serialization and lets its
// dependents launch as soon as it starts, so that the next product's CTAs set up (barriers, TMEM,
// cluster sync) on the SMs this grid's finished pairs release; the producer alone waits for the
// preceding grid (griddepcontrol.wait) before its first load, and everything this grid writes
// follows that wait.
// No TMA load uses multicast.  Every wait is bounded (WaitGuard).
#include <cuda_bf16.h>

#include "../../include/unstep.h"
#include "gemm.h"
#include "sm100.cuh"

namespace unstep {
namespace {

constexpr int kTM = 256, kTN = 256, kBK = 64;    // output tile of a pair, K step
#ifndef UNSTEP_GEMM_PDL
#define UNSTEP_GEMM_PDL 1
#endif
#ifndef UNSTEP_GEMM2SM_STAGES
#define UNSTEP_GEMM2SM_STAGES 6
#endif
constexpr int kStages = UNSTEP_GEMM2SM_STAGES;
constexpr int kThreads = 256;                    // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr int kABytes = 128 * kBK * 2;           // this CTA's 128 rows of A: 16 KB
constexpr int kBBytes = 128 * kBK * 2;           // this CTA's 128 rows of B: 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kOutCols = 64;                     // columns per staged output box
constexpr int kStgBytes = 32 * kOutCols * 2;     // one warp's 32 rows x 64 columns: 4 KB
constexpr int kSmemStg = kStages * kStageBytes;  // 2 staging buffers per epilogue warp
constexpr int kSmemBar = kSmemStg + 4 * 2 * kStgBytes;
constexpr int kSmemAlloc = kSmemBar + 256 + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
constexpr int kAccCols = kTN;                    // 256 TMEM columns per accumulator set
constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// TMA 2D load into this CTA's shared memory, completing on the barrier at cluster address mbar
// (CTA 0's); no multicast.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t mbar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(mbar)
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

// Arrive (once) on the barrier at this shared offset in both CTAs of the pair when the pair's
// earlier MMAs have completed.
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

// TMA 2D store of a box from this CTA's shared memory (bulk async-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(smem_u32(src))
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Until at most one bulk group of this thread still reads shared memory.
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Until every bulk group of this thread has completed (its writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Persistent over pairs: pair q takes tiles q, q + pairs, ...; tiles are m-major within an n
// column (tile t -> n block t / m_tiles, m block t % m_tiles).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm2sm_bf16_tn_kernel(const __grid_constant__ CUtensorMap tma,
                           const __grid_constant__ CUtensorMap tmb,
                           const __grid_constant__ CUtensorMap tmc, int M, int N, int K,
                           int *dev_error, uint64_t wait_limit_ns) {
  if (UNSTEP_GEMM_PDL && threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");
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
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  const int m_tiles = (M + kTM - 1) / kTM;
  const int n_tiles = (N + kTN - 1) / kTN;
  const int tiles = m_tiles * n_tiles;
  const int k_steps = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);     // CTA 0's: its producer's arrival plus both CTAs' bytes
      mbar_init(&empty[s], 1);    // one multicast commit per use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 256);   // CTA 0's: both CTAs' epilogue threads
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(2 * kAccCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers initialised and TMEM allocated before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitGuard g{abort_flag, dev_error, wait_limit_ns};
  constexpr int E = UNSTEP_ERR_DEVICE_TIMEOUT;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tma);
      tma_prefetch_desc(&tmb);
      // A and B may be the preceding grid's output: wait for it to complete before any load
      if (UNSTEP_GEMM_PDL) asm volatile("griddepcontrol.wait;" ::: "memory");
      int n = 0;  // stage fills issued
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += pairs) {
        const int m0 = (t % m_tiles) * kTM + 128 * static_cast<int>(rank);
        const int n0 = (t / m_tiles) * kTN + 128 * static_cast<int>(rank);
        for (int k = 0; k < k_steps; ++k, ++n) {
          const int s = n % kStages;
          const uint32_t r = static_cast<uint32_t>(n / kStages);
          if (!(ok = wait_bounded(&empty[s], (r & 1u) ^ 1u, g, E))) break;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kStageBytes);
          const uint32_t fb = peer_addr(&full[s], 0);
          uint8_t *st = smem + s * kStageBytes;
          tma_load_2d_pair(st, &tma, fb, k * kBK, m0);
          tma_load_2d_pair(st + kABytes, &tmb, fb, k * kBK, n0);
        }
      }
      // after an abort, CTA 0 lets every copy of the pair still in flight land (its stage
      // barriers count both CTAs' bytes) before the pair's shared memory is released
      if (*abort_flag && rank == 0)
        for (int k = max(0, n - kStages); k < n; ++k)
          drain_wait(&full[k % kStages], static_cast<uint32_t>(k / kStages) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(kTM, kTN, false, false);
      const uint32_t hi = static_cast<uint32_t>(sdesc_sw128(0, 16, 1024) >> 32);
      const uint32_t lo0 = static_cast<uint32_t>(sdesc_sw128(smem_u32(smem), 16, 1024));
      bool ok = true;
      int n = 0, i = 0;
      for (int t = pair; ok && t < tiles; t += pairs, ++i) {
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
            umma_ss_pair(d, f2u64(la + kk * 2, hi), f2u64(lb + kk * 2, hi), kId,
                         (k > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(&empty[s]);
        }
        if (ok) umma_commit_pair(&acc_full[acc]);
      }
      umma_commit_pair_local(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int wq = warp - 4;            // this warp's 32 TMEM lanes = output rows 32 wq ..
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t acc_empty0 = peer_addr(&acc_empty[0], 0);
    const uint32_t acc_empty1 = peer_addr(&acc_empty[1], 0);
    uint8_t *stg = smem + kSmemStg + wq * 2 * kStgBytes;
    if (lane == 0) tma_prefetch_desc(&tmc);
    bool ok = true;
    int i = 0, nst = 0;
    for (int t = pair; t < tiles; t += pairs, ++i) {
      const int acc = i & 1;
      if (ok)
        ok = __all_sync(kFull, wait_bounded(&acc_full[acc], static_cast<uint32_t>(i >> 1) & 1u, g, E));
      if (!ok) break;
      tc_fence_after();
      const int m0 = (t % m_tiles) * kTM + 128 * static_cast<int>(rank) + wq * 32;
      const int n0 = (t / m_tiles) * kTN;
      const uint32_t src = tmem + lane_base + acc * kAccCols;
#pragma unroll 1
      for (int c = 0; c < kTN / kOutCols; ++c, ++nst) {
        uint32_t o[2][32];
        tmem_ld32(src + c * kOutCols, o[0]);
        tmem_ld32(src + c * kOutCols + 32, o[1]);
        tmem_wait_ld();
        uint8_t *buf = stg + (nst & 1) * kStgBytes;
        if (lane == 0) bulk_wait_read1();  // the store issued from this buffer two chunks ago
        __syncwarp();
        // row `lane` of the box: 16-byte chunk j (columns 8j .. 8j+7) at position j ^ (lane & 7)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int h = j >> 2, e = (j & 3) * 8;
          const uint4 v = make_uint4(
              pack_bf16x2(__uint_as_float(o[h][e]), __uint_as_float(o[h][e + 1])),
              pack_bf16x2(__uint_as_float(o[h][e + 2]), __uint_as_float(o[h][e + 3])),
              pack_bf16x2(__uint_as_float(o[h][e + 4]), __uint_as_float(o[h][e + 5])),
              pack_bf16x2(__uint_as_float(o[h][e + 6]), __uint_as_float(o[h][e + 7])));
          *reinterpret_cast<uint4 *>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // rows past M and columns past N are clipped by the tensor map; a box that starts
          // past either edge holds nothing of the output and is not stored
          if (m0 < M && n0 + c * kOutCols < N) tma_store_2d(&tmc, buf, n0 + c * kOutCols, m0);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive_remote(acc ? acc_empty1 : acc_empty0);
    }
    if (lane == 0) bulk_wait_all();  // the stores have read the buffers and written C
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the pair's MMAs and both epilogues are done with the TMEM of both CTAs
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * kAccCols)
                 : "memory");
  }
}

}  // namespace

cudaError_t launch_gemm2sm_bf16_tn(const CUtensorMap &ta, const CUtensorMap &tb,
                                   const CUtensorMap &tc, int M, int N, int K, int *dev_error,
                                   cudaStream_t stream) {
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(__atomic_load_n(&attr_set, __ATOMIC_ACQUIRE) & bit)) {
    e = cudaFuncSetAttribute(gemm2sm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemAlloc);
    if (e != cudaSuccess) return e;
    if (dev < 64) __atomic_fetch_or(&attr_set, bit, __ATOMIC_RELEASE);
  }
  const long long tiles = static_cast<long long>((M + kTM - 1) / kTM) * ((N + kTN - 1) / kTN);
  if (tiles < 1 || tiles > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int pairs_max = sms / 2;
  const int pairs = static_cast<int>(tiles < pairs_max ? tiles : pairs_max);
  if (pairs < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = UNSTEP_GEMM_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm2sm_bf16_tn_kernel, ta, tb, tc, M, N, K, dev_error,
                         kWaitLimitNs);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace unstep
