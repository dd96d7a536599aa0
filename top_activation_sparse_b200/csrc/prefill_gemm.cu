// Prefill masked-dense GEMM on the 5th-generation tensor cores:
//   Y[M, N] = X_sparse[M, K] . W^T[K, N]      (bf16 in, f32 accumulate, bf16 out)
//
// Source: Q-Sparse paper summary (shd-paper.top), abstract and method
// sections (Block Q-Sparse makes the sparsity usable for batched training and
// inference); with thousands of tokens each keeping its own top-K, almost
// every weight row is needed by some token, so the projection is a dense
// contraction over the masked activations and belongs on the tensor cores.
//
// sm_100a design (persistent: one CTA per SM walks output tiles of 128 x 256):
//   * TMA (cp.async.bulk.tensor, 128-byte swizzle, one CTA per copy) loads an A
//     tile of X_sparse (128 rows x 64 K, K-major) and a B tile of W^T (64 K x
//     256 N, N-major, as four 64-column boxes) per stage into a 4-stage ring;
//   * one thread issues tcgen05.mma.kind::f16 (bf16 x bf16 -> f32) with the
//     accumulator in tensor memory (two accumulators of 256 columns x 128
//     lanes, used by alternate tiles) and frees each stage with
//     tcgen05.commit on that stage's "empty" mbarrier;
//   * four epilogue warps read a finished accumulator with tcgen05.ld (each
//     warp its 32 TMEM lanes = 32 rows), round to bf16 and store Y while the
//     MMAs of the next tile fill the other accumulator;
//   * CTAs are ordered M-block fastest, so the CTAs resident at one time share
//     W^T tiles through the L2;
//   * every mbarrier wait is bounded: on a timeout the CTA records
//     DEV_TIMEOUT, waits (bounded) for its own copies and MMAs in flight,
//     frees its TMEM and returns.
//
// The same kernel serves the backward of the projection under the
// straight-through estimator (Q-Sparse news article, section "Top-K
// sparsification", STE paragraphs), through two compile-time choices: the
// major-ness of each operand (K-major: the reduction index is contiguous in
// memory; MN-major: the output index is) and the epilogue (bf16 store, f32
// store, or f32 accumulate into an existing matrix):
//   dL/dX   = dL/dY . W       A = dL/dY [T, d_out] K-major, B = W^T [d_in, d_out] K-major
//   dL/dW^T = X_sparse^T . dL/dY   A = X_sparse [T, d_in] read MN-major,
//                                  B = dL/dY [T, d_out] MN-major, added to dL/dW^T
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;                 // 16 KB
constexpr int kBBox = 64 * BK * 2;                   // one 64-column box of B: 8 KB
constexpr int kBBytes = (BN / 64) * kBBox;           // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;       // 48 KB
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kThreads = 192;                        // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 512;                  // two 256-column accumulators

// tcgen05 instruction descriptor, kind::f16: D f32, A and B bf16, N = 256,
// M = 128; bits 15 / 16 select MN-major A / B.
template <bool A_MN, bool B_MN>
constexpr uint32_t idesc() {
  return (1u << 4)                               // accumulator format: f32
         | (1u << 7)                             // A format: bf16
         | (1u << 10)                            // B format: bf16
         | ((A_MN ? 1u : 0u) << 15)              // A major-ness
         | ((B_MN ? 1u : 0u) << 16)              // B major-ness
         | ((uint32_t)(BN >> 3) << 17)
         | ((uint32_t)(BM >> 4) << 24);
}

// Epilogue kinds.
enum Epi { EPI_BF16 = 0, EPI_F32 = 1, EPI_F32_ADD = 2 };

// Shared-memory matrix descriptor (sm_100 version bits), 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc_bits, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc_bits), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive f32 accumulator columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo_f32, uint32_t hi_f32) {
  return (uint32_t)f32_to_bf16_bits(__uint_as_float(lo_f32)) |
         ((uint32_t)f32_to_bf16_bits(__uint_as_float(hi_f32)) << 16);
}

// out[M, N] (row pitch ldo elements) = A[M, K] . B[K, N]  (or out += that, EPI_F32_ADD)
template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b, void* __restrict__ out, int ldo,
                     int M, int N, int K, DevStatus* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  pdl_begin();
  __shared__ __align__(8) uint64_t s_full[kStages];
  __shared__ __align__(8) uint64_t s_empty[kStages];
  __shared__ __align__(8) uint64_t s_tfull[2];      // accumulator b complete (MMA -> epilogue)
  __shared__ __align__(8) uint64_t s_tempty[2];     // accumulator b drained (epilogue -> MMA)
  __shared__ __align__(8) uint64_t s_done;          // every MMA issued has completed
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  // 1024-byte aligned ring (128-byte swizzle atoms repeat every 1 KB)
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mblocks = (M + BM - 1) / BM;
  const int ntiles = mblocks * ((N + BN - 1) / BN);
  const int nk = (K + BK - 1) / BK;
  // tiles of this CTA: blockIdx.x, + gridDim.x, ...  (M-block fastest, so the
  // CTAs busy at one time share W^T tiles through the L2)
  const int my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_tfull[b], 1);
      mbar_init(&s_tempty[b], kEpiThreads);
    }
    mbar_init(&s_done, 1);
    mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) {   // whole warp: two accumulators of 256 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer: the ring runs on across this CTA's tiles ----
    int it = 0;
    for (int lt = 0; lt < my_tiles && !*(volatile int*)&s_abort; ++lt) {
      const int t = (int)blockIdx.x + lt * (int)gridDim.x;
      const int m0 = (t % mblocks) * BM, n0 = (t / mblocks) * BN;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait(&s_empty[s], (uint32_t)((it / kStages) - 1) & 1u)) {
          dev_fail(status, DEV_TIMEOUT, 20, (uint32_t)it);
          atomicExch(&s_abort, 1);
          break;
        }
        if (*(volatile int*)&s_abort) break;
        const uint32_t sa = base + (uint32_t)(s * kStageBytes);
        const uint32_t sb = sa + kABytes;
        mbar_arrive_expect_tx(&s_full[s], (uint32_t)kStageBytes);
        if constexpr (A_MN) {                    // two 64-row (M) x 64 (K) boxes
#pragma unroll
          for (int j = 0; j < BM / 64; ++j)
            tma_load_2d(sa + j * kBBox, &map_a, m0 + 64 * j, kb * BK, &s_full[s]);
        } else {                                 // one 64 (K) x 128 (M) box
          tma_load_2d(sa, &map_a, kb * BK, m0, &s_full[s]);
        }
        if constexpr (B_MN) {                    // four 64-column (N) x 64 (K) boxes
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sb + j * kBBox, &map_b, n0 + 64 * j, kb * BK, &s_full[s]);
        } else {                                 // one 64 (K) x 256 (N) box
          tma_load_2d(sb, &map_b, kb * BK, n0, &s_full[s]);
        }
      }
    }
    // on an abort, let the copies already issued land before the CTA exits
    if (*(volatile int*)&s_abort) {
      for (int i = 0; i < kStages && i < it; ++i) {
        const int g = it - 1 - i;
        mbar_wait(&s_full[g % kStages], (uint32_t)(g / kStages) & 1u);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: accumulator lt & 1, reused once the epilogue drained it ----
    int it = 0;
    bool issued = false;
    for (int lt = 0; lt < my_tiles && !*(volatile int*)&s_abort; ++lt) {
      const int b = lt & 1;
      if (lt >= 2 && !mbar_wait(&s_tempty[b], (uint32_t)((lt >> 1) - 1) & 1u)) {
        dev_fail(status, DEV_TIMEOUT, 23, (uint32_t)lt);
        atomicExch(&s_abort, 1);
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&s_full[s], (uint32_t)(it / kStages) & 1u)) {
          dev_fail(status, DEV_TIMEOUT, 21, (uint32_t)it);
          atomicExch(&s_abort, 1);
          break;
        }
        if (*(volatile int*)&s_abort) break;
        tc_fence_after();
        const uint32_t sa = base + (uint32_t)(s * kStageBytes);
        const uint32_t sb = sa + kABytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // K-major operand: 128-byte rows, 8-row groups 1 KB apart; K step = 32 bytes.
          // MN-major operand: 128-byte K rows, 8-row groups 1 KB apart (SBO),
          //   64-element M/N boxes 8 KB apart (LBO); K step = 16 rows = 2 KB.
          const uint64_t ad = A_MN ? smem_desc(sa + kk * 2048, kBBox, 1024) : smem_desc(sa + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc(sb + kk * 2048, kBBox, 1024) : smem_desc(sb + kk * 32, 16, 1024);
          umma_bf16(acc, ad, bd, idesc<A_MN, B_MN>(), (kb > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&s_empty[s]);          // frees the stage once these MMAs have read it
        issued = true;
      }
      umma_commit(&s_tfull[b]);            // accumulator b complete (or abandoned)
    }
    // every MMA issued has completed before TMEM is freed
    if (issued) {
      umma_commit(&s_done);
      mbar_wait(&s_done, 0u);
    }
  } else if (warp >= 2) {
    // ---- epilogue: TMEM -> registers -> bf16 -> global, overlapping the next tile's MMAs ----
    const int q = warp & 3;                      // this warp's TMEM lane quarter
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int b = lt & 1;
      const int t = (int)blockIdx.x + lt * (int)gridDim.x;
      const int m0 = (t % mblocks) * BM, n0 = (t / mblocks) * BN;
      if (!mbar_wait_backoff(&s_tfull[b], (uint32_t)(lt >> 1) & 1u)) {
        if (lane == 0) dev_fail(status, DEV_TIMEOUT, 22, (uint32_t)lt);
        atomicExch(&s_abort, 1);
        break;
      }
      tc_fence_after();
      const bool abort = *(volatile int*)&s_abort;
      const int row = m0 + q * 32 + lane;
      const uint32_t acc = tmem + (uint32_t)(b * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(acc + (uint32_t)c, r);
        if (abort || row >= M) continue;
        if constexpr (EPI == EPI_BF16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out) + (size_t)row * ldo + n0 + c;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (n0 + c + 8 * v + 8 > N) break;     // N is a multiple of 8
            uint4 o;
            o.x = pack_bf16x2(r[8 * v + 0], r[8 * v + 1]);
            o.y = pack_bf16x2(r[8 * v + 2], r[8 * v + 3]);
            o.z = pack_bf16x2(r[8 * v + 4], r[8 * v + 5]);
            o.w = pack_bf16x2(r[8 * v + 6], r[8 * v + 7]);
            *reinterpret_cast<uint4*>(dst + 8 * v) = o;
          }
        } else {
          float* dst = reinterpret_cast<float*>(out) + (size_t)row * ldo + n0 + c;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            if (n0 + c + 4 * v + 4 > N) break;     // N is a multiple of 4
            float4 o = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            if constexpr (EPI == EPI_F32_ADD) {
              // add into the existing values; a sum of exactly zero (no kept
              // input in this row) leaves them untouched
              if (o.x == 0.0f && o.y == 0.0f && o.z == 0.0f && o.w == 0.0f) continue;
              const float4 p = *reinterpret_cast<const float4*>(dst + 4 * v);
              if (o.x != 0.0f) o.x += p.x; else o.x = p.x;
              if (o.y != 0.0f) o.y += p.y; else o.y = p.y;
              if (o.z != 0.0f) o.z += p.z; else o.z = p.z;
              if (o.w != 0.0f) o.w += p.w; else o.w = p.w;
            }
            *reinterpret_cast<float4*>(dst + 4 * v) = o;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s_tempty[b]);                   // this thread's reads of accumulator b are done
      if (abort) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}


// ---- prefill forward with 2-SM tiles (tcgen05 cta_group::2) -----------------
// A cluster of two CTAs (on two SMs) computes a 256 x 256 tile of Y: each CTA
// loads its own 128 rows of X_sparse and its own 128-column half of the W^T
// tile (so each SM reads half of B from L2: 32 KB per stage instead of 48), the
// first CTA of the pair issues tcgen05.mma.cta_group::2 (M = 256: the
// accumulator rows are split over the two CTAs' tensor memory, the B operand
// is read from both CTAs' shared memory), and each CTA's epilogue stores its
// own 128 rows.  Each copy writes only its own CTA's shared memory and
// signals the first CTA's stage barrier (its address through mapa); each MMA
// commit arrives on the barriers of both CTAs (a tcgen05.commit with a CTA mask).
constexpr int k2Stages = 6;
constexpr int k2ABytes = 128 * BK * 2;               // 16 KB: this CTA's 128 rows
constexpr int k2BBytes = 2 * kBBox;                  // 16 KB: this CTA's 128 columns (two boxes)
constexpr int k2StageBytes = k2ABytes + k2BBytes;    // 32 KB
// + 16 KB of slack after the ring: no operand read can leave the allocation
constexpr int k2SmemBytes = k2Stages * k2StageBytes + 16 * 1024 + 1024;
constexpr int k2EpiWarps = 4;

// kind::f16: D f32, A and B bf16 (bits 15 / 16: MN-major A / B), N = 256,
// M = 256 (the pair)
template <bool A_MN, bool B_MN>
constexpr uint32_t idesc_2sm() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16) |
         ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc_bits, uint32_t accumulate) {
  const uint32_t z = 0u;                           // no output lane is disabled
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc_bits), "r"(accumulate), "r"(z)
      : "memory");
}

// arrives on the barrier at the same offset in both CTAs of the pair once the
// MMAs issued so far have completed
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The operand major-ness and the epilogue as in umma_gemm_kernel: the forward
// prefill is <K-major A, MN-major B, bf16>, the STE backward's dL/dX
// <K-major, K-major, f32> and dL/dW^T <MN-major, MN-major, f32 add>.
template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    umma_gemm_2sm_kernel(const __grid_constant__ CUtensorMap map_a,
                         const __grid_constant__ CUtensorMap map_b, void* __restrict__ out,
                         int ldo, int M, int N, int K, DevStatus* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  pdl_begin();
  __shared__ __align__(8) uint64_t s_full[k2Stages];   // first CTA: both CTAs' copies of a stage
  __shared__ __align__(8) uint64_t s_empty[k2Stages];  // each CTA: the stage's MMAs are done
  __shared__ __align__(8) uint64_t s_tfull[2];         // each CTA: accumulator b complete
  __shared__ __align__(8) uint64_t s_tempty[2];        // first CTA: both epilogues drained b
  __shared__ __align__(8) uint64_t s_done;             // first CTA: every MMA has completed
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = blockIdx.x & 1u;             // position in the pair (cluster of 2)
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int mblocks = (M + 255) / 256;
  const int ntiles = mblocks * ((N + BN - 1) / BN);
  const int nk = (K + BK - 1) / BK;
  const int my_tiles = pair < ntiles ? (ntiles - 1 - pair) / npairs + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_tfull[b], 1);
      mbar_init(&s_tempty[b], 2 * k2EpiWarps);
    }
    mbar_init(&s_done, 1);
    mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 0) {   // the same warp of both CTAs: the pair's accumulators (2 x 256 columns)
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                                // the peer's barriers exist before any signal
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer (both CTAs) ----
    int it = 0;
    for (int lt = 0; lt < my_tiles && !*(volatile int*)&s_abort; ++lt) {
      const int t = pair + lt * npairs;
      const int m0 = (t % mblocks) * 256 + (int)rank * 128, n0 = (t / mblocks) * BN + (int)rank * 128;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % k2Stages;
        if (it >= k2Stages && !mbar_wait(&s_empty[s], (uint32_t)((it / k2Stages) - 1) & 1u)) {
          dev_fail(status, DEV_TIMEOUT, 24, (uint32_t)it);
          atomicExch(&s_abort, 1);
          break;
        }
        if (*(volatile int*)&s_abort) break;
        const uint32_t sa = base + (uint32_t)(s * k2StageBytes);
        const uint32_t sb = sa + k2ABytes;
        const uint32_t full0 = cluster_addr(smem_u32(&s_full[s]), 0);
        if (leader) mbar_arrive_expect_tx(&s_full[s], (uint32_t)(2 * k2StageBytes));
        if constexpr (A_MN) {                      // 2 x 64 (M) x 64 (K)
#pragma unroll
          for (int j = 0; j < 2; ++j) tma_load_2d_pair(sa + j * kBBox, &map_a, m0 + 64 * j, kb * BK, full0);
        } else {                                   // 64 (K) x 128 (M)
          tma_load_2d_pair(sa, &map_a, kb * BK, m0, full0);
        }
        if constexpr (B_MN) {                      // 2 x 64 (N) x 64 (K)
#pragma unroll
          for (int j = 0; j < 2; ++j) tma_load_2d_pair(sb + j * kBBox, &map_b, n0 + 64 * j, kb * BK, full0);
        } else {                                   // 64 (K) x 128 (N)
          tma_load_2d_pair(sb, &map_b, kb * BK, n0, full0);
        }
      }
    }
    // on an abort, the first CTA lets the copies already issued (both CTAs') land
    if (leader && *(volatile int*)&s_abort) {
      for (int i = 0; i < k2Stages && i < it; ++i) {
        const int g = it - 1 - i;
        mbar_wait(&s_full[g % k2Stages], (uint32_t)(g / k2Stages) & 1u);
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---- MMA issuer (first CTA only) ----
    int it = 0;
    bool issued = false;
    for (int lt = 0; lt < my_tiles && !*(volatile int*)&s_abort; ++lt) {
      const int b = lt & 1;
      if (lt >= 2 && !mbar_wait(&s_tempty[b], (uint32_t)((lt >> 1) - 1) & 1u)) {
        dev_fail(status, DEV_TIMEOUT, 25, (uint32_t)lt);
        atomicExch(&s_abort, 1);
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % k2Stages;
        if (!mbar_wait(&s_full[s], (uint32_t)(it / k2Stages) & 1u)) {
          dev_fail(status, DEV_TIMEOUT, 26, (uint32_t)it);
          atomicExch(&s_abort, 1);
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + (uint32_t)(s * k2StageBytes);
        const uint32_t sb = sa + k2ABytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc(sa + kk * 2048, kBBox, 1024) : smem_desc(sa + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc(sb + kk * 2048, kBBox, 1024) : smem_desc(sb + kk * 32, 16, 1024);
          umma_bf16_pair(acc, ad, bd, idesc_2sm<A_MN, B_MN>(), (kb > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_pair(&s_empty[s]);     // frees the stage in both CTAs
        issued = true;
      }
      umma_commit_pair(&s_tfull[b]);       // accumulator b complete in both CTAs
    }
    if (issued) {
      umma_commit_pair_local(&s_done);
      mbar_wait(&s_done, 0u);
    }
  } else if (warp >= 2) {
    // ---- epilogue (both CTAs): this CTA's 128 rows of the tile ----
    const int q = warp & 3;
    const uint32_t tempty0[2] = {cluster_addr(smem_u32(&s_tempty[0]), 0),
                                 cluster_addr(smem_u32(&s_tempty[1]), 0)};
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int b = lt & 1;
      const int t = pair + lt * npairs;
      const int m0 = (t % mblocks) * 256 + (int)rank * 128, n0 = (t / mblocks) * BN;
      if (!mbar_wait_backoff(&s_tfull[b], (uint32_t)(lt >> 1) & 1u)) {
        if (lane == 0) dev_fail(status, DEV_TIMEOUT, 27, (uint32_t)lt);
        atomicExch(&s_abort, 1);
        break;
      }
      tc_fence_after();
      const bool abort = *(volatile int*)&s_abort;
      const int row = m0 + q * 32 + lane;
      const uint32_t acc = tmem + (uint32_t)(b * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(acc + (uint32_t)c, r);
        if (abort || row >= M) continue;
        if constexpr (EPI == EPI_BF16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out) + (size_t)row * ldo + n0 + c;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (n0 + c + 8 * v + 8 > N) break;     // N is a multiple of 8
            uint4 o;
            o.x = pack_bf16x2(r[8 * v + 0], r[8 * v + 1]);
            o.y = pack_bf16x2(r[8 * v + 2], r[8 * v + 3]);
            o.z = pack_bf16x2(r[8 * v + 4], r[8 * v + 5]);
            o.w = pack_bf16x2(r[8 * v + 6], r[8 * v + 7]);
            *reinterpret_cast<uint4*>(dst + 8 * v) = o;
          }
        } else {
          float* dst = reinterpret_cast<float*>(out) + (size_t)row * ldo + n0 + c;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            if (n0 + c + 4 * v + 4 > N) break;     // N is a multiple of 4
            float4 o = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            if constexpr (EPI == EPI_F32_ADD) {
              // add into the existing values; a sum of exactly zero (no kept
              // input in this row) leaves them untouched
              if (o.x == 0.0f && o.y == 0.0f && o.z == 0.0f && o.w == 0.0f) continue;
              const float4 p = *reinterpret_cast<const float4*>(dst + 4 * v);
              if (o.x != 0.0f) o.x += p.x; else o.x = p.x;
              if (o.y != 0.0f) o.y += p.y; else o.y = p.y;
              if (o.z != 0.0f) o.z += p.z; else o.z = p.z;
              if (o.w != 0.0f) o.w += p.w; else o.w = p.w;
            }
            *reinterpret_cast<float4*>(dst + 4 * v) = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0[b]);   // this warp's reads of accumulator b are done
      if (abort) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                                // both CTAs are done with the pair's TMEM
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map: dims {inner, outer}, row pitch in bytes, box {bx, by}.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t pitch,
              uint32_t bx, uint32_t by) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {bx, by};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_supported(int M, int N, int K) {
  // TMA needs 16-byte row pitches; the epilogue stores 8 columns at a time
  return M >= 1 && N >= 8 && K >= 8 && (N % 8) == 0 && (K % 8) == 0 && encode_fn() != nullptr;
}

namespace {

template <bool A_MN, bool B_MN, int EPI>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, void* out, int ldo, int M,
                        int N, int K, DevStatus* status, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(umma_gemm_kernel<A_MN, B_MN, EPI>, kSmemBytes, &configured);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM, each walking tiles blockIdx.x + i * gridDim.x
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  dim3 grid(tiles < kNumSMs ? tiles : kNumSMs);
  e = launch_pdl(umma_gemm_kernel<A_MN, B_MN, EPI>, grid, dim3(kThreads), (size_t)kSmemBytes, s, ma,
                 mb, out, ldo, M, N, K, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Pairs of CTAs resident at once for one 2-SM kernel instance (0: not available).
template <bool A_MN, bool B_MN, int EPI>
int pair_clusters() {
  static int n = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    n = 0;
    if (cudaFuncSetAttribute(umma_gemm_2sm_kernel<A_MN, B_MN, EPI>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, k2SmemBytes) != cudaSuccess)
      return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * kNumSMs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)k2SmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, umma_gemm_2sm_kernel<A_MN, B_MN, EPI>, &cfg) == cudaSuccess &&
        c > 0)
      n = c;
    (void)cudaGetLastError();
  });
  return n;
}

template <bool A_MN, bool B_MN, int EPI>
cudaError_t launch_gemm_2sm(const CUtensorMap& ma, const CUtensorMap& mb, void* out, int ldo, int M,
                            int N, int K, DevStatus* status, int clusters, cudaStream_t s) {
  const int tiles = ((M + 255) / 256) * ((N + BN - 1) / BN);
  const int pairs = tiles < clusters ? tiles : clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)k2SmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, umma_gemm_2sm_kernel<A_MN, B_MN, EPI>, ma, mb, out, ldo, M,
                                     N, K, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_gemm(const PrefillArgs& a, cudaStream_t s) {
  CUtensorMap ma, mb;
  // A = X_sparse [M, K] row-major: inner K, box 64 x 128
  if (!make_map(&ma, a.xs, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * 2, BK, BM))
    return cudaErrorInvalidValue;
  // B = W^T [K, N] row-major: inner N, box 64 (N) x 64 (K)
  if (!make_map(&mb, a.wt, (uint64_t)a.N, (uint64_t)a.K, (uint64_t)a.N * 2, 64, BK))
    return cudaErrorInvalidValue;
  // pairs of SMs on one 256 x 256 tile (each loads half of the W^T tile)
  const int clusters = pair_clusters<false, true, EPI_BF16>();
  if (clusters > 0)
    return launch_gemm_2sm<false, true, EPI_BF16>(ma, mb, a.y, a.N, a.M, a.N, a.K, a.status, clusters, s);
  return launch_gemm<false, true, EPI_BF16>(ma, mb, a.y, a.N, a.M, a.N, a.K, a.status, s);
}

bool backward_gemm_supported(int T, int d_in, int d_out) {
  return T >= 1 && d_in >= 8 && d_out >= 8 && (d_in % 8) == 0 && (d_out % 8) == 0 &&
         encode_fn() != nullptr;
}

cudaError_t launch_grad_x_gemm(const BackwardGemmArgs& a, cudaStream_t s) {
  // grad_x [T, d_in] = dL/dY [T, d_out] . (W^T [d_in, d_out])^T
  CUtensorMap ma, mb;
  // A = dL/dY: M = T rows, K = d_out contiguous (K-major), box 64 (K) x 128 (M)
  if (!make_map(&ma, a.grad_y, (uint64_t)a.d_out, (uint64_t)a.T, (uint64_t)a.d_out * 2, BK, BM))
    return cudaErrorInvalidValue;
  // B = W^T: N = d_in rows, K = d_out contiguous (K-major): box 64 (K) x 128 (N) for a CTA of a
  // pair (2-SM tiles), else 64 x 256
  const int clusters = pair_clusters<false, false, EPI_F32>();
  if (!make_map(&mb, a.wt, (uint64_t)a.d_out, (uint64_t)a.d_in, (uint64_t)a.d_out * 2, BK,
                clusters > 0 ? 128 : BN))
    return cudaErrorInvalidValue;
  if (clusters > 0)
    return launch_gemm_2sm<false, false, EPI_F32>(ma, mb, a.grad_x, a.d_in, a.T, a.d_in, a.d_out,
                                                  a.status, clusters, s);
  return launch_gemm<false, false, EPI_F32>(ma, mb, a.grad_x, a.d_in, a.T, a.d_in, a.d_out,
                                            a.status, s);
}

cudaError_t launch_grad_wt_gemm(const BackwardGemmArgs& a, cudaStream_t s) {
  // grad_wt [d_in, d_out] += X_sparse^T [d_in, T] . dL/dY [T, d_out]
  CUtensorMap ma, mb;
  // A = X_sparse^T: M = d_in contiguous in X_sparse [T, d_in] (MN-major), K = T; box 64 x 64
  if (!make_map(&ma, a.xs, (uint64_t)a.d_in, (uint64_t)a.T, (uint64_t)a.d_in * 2, 64, BK))
    return cudaErrorInvalidValue;
  // B = dL/dY [T, d_out]: N = d_out contiguous (MN-major), K = T; box 64 x 64
  if (!make_map(&mb, a.grad_y, (uint64_t)a.d_out, (uint64_t)a.T, (uint64_t)a.d_out * 2, 64, BK))
    return cudaErrorInvalidValue;
  const int clusters = pair_clusters<true, true, EPI_F32_ADD>();
  if (clusters > 0)
    return launch_gemm_2sm<true, true, EPI_F32_ADD>(ma, mb, a.grad_wt, a.d_out, a.d_in, a.d_out, a.T,
                                                    a.status, clusters, s);
  return launch_gemm<true, true, EPI_F32_ADD>(ma, mb, a.grad_wt, a.d_out, a.d_in, a.d_out, a.T,
                                              a.status, s);
}

}  // namespace qs
