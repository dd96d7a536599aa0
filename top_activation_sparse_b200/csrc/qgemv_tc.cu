// int8 x ternary projection for 8 to 64 tokens on the 5th-generation tensor
// cores (tcgen05.mma kind::i8, int32 accumulators in tensor memory).
//
// Source: Q-Sparse news article (zxwl-tech.com), Top-K section, paragraphs on
// quantized models (BitNet b1.58 + Q-Sparse): int8 activation codes q (the
// kept entries of each token, zero elsewhere) times ternary weights t, summed
// exactly in int32: acc[t, j] = sum_i q[t, i] * t[i, j]; y = f32(acc) * r_t.
//
// With 8 or more tokens the union of the tokens' kept inputs covers about
// every input (1 - 0.61^8 = 98% at 39% kept), so this kernel streams every
// packed row of W^T in order (2-D TMA, no gather) and multiplies it with the
// dense masked codes (zero where a token dropped the input):
//   * a CTA owns 256 output columns (two MMAs of M = 128) and a range of
//     rows; per step of 64 rows (two of the MMA's K = 32) one TMA brings the
//     64 x 64-byte packed segment and two TMAs the tokens' codes (32 rows
//     each, K-major, 32-byte swizzle), into a ring of 4 stages (fewer barrier
//     handshakes per byte than 32-row steps: each costs shared-memory round
//     trips in the single-thread loops);
//   * eight decode warps, in four groups that take every fourth step (their
//     proxy fences overlap), expand the 2-bit codes (00 = 0, 01 = +1, 10 = -1) into
//     int8 (the codes are spread into nibbles, and one byte permute per four
//     codes selects from the bytes {0, +1, -1}) and write the two A tiles in
//     the MN-major 128-byte-swizzled layout
//     (each 64-row x 128-byte tile: row k holds columns 0..127, 16-byte chunk
//     c of row k at chunk c ^ (k mod 8)), then make them visible to the tensor
//     core (fence.proxy.async) and arrive on the stage's barrier;
//   * one thread issues tcgen05.mma.cta_group::1.kind::i8 (s8 x s8 -> s32,
//     M = 128, N = tokens rounded up to 16, K = 32; four per step) into two
//     accumulators and frees the stage with tcgen05.commit;
//   * the decode warps then read the accumulators (tcgen05.ld, one column per
//     lane) into the CTA's shared memory; the S CTAs that split the rows of
//     one column range form a thread-block cluster, and after a cluster
//     barrier each of them sums its slice of the columns over all S partial
//     tiles through distributed shared memory (exact int32), rescales
//     y = f32(acc) * r_t and stores it: no global atomics, no split-sum buffer.
// Every wait is bounded; a timeout records DEV_TIMEOUT, lets the copies and
// MMAs in flight finish and frees the tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr int kTcBlocks = 2;                       // 128-column MMA blocks per CTA
constexpr int kTcCols = 128 * kTcBlocks;           // output columns per CTA
constexpr int kTcWords = kTcCols / 16;             // packed words per row segment (16)
constexpr int kTcK = 32;                           // the MMA's K for int8 (rows per MMA)
constexpr int kTcKc = 2;                           // K chunks (MMAs per accumulator) per step
constexpr int kTcRows = kTcK * kTcKc;              // rows per step: fewer handshakes per byte
constexpr int kTcStages = 4;                       // two CTAs per SM fit (2 x 97 KB)
constexpr int kTcATile = kTcRows * 128;            // one 128-column A tile: 8 KB
constexpr int kTcPacked = kTcRows * kTcWords * 4;  // 4 KB
constexpr int kTcBChunk = 64 * kTcK;               // codes of up to 64 tokens for one K chunk: 2 KB
constexpr int kTcBMax = kTcKc * kTcBChunk;         // 4 KB
constexpr int kTcStage = kTcBlocks * kTcATile + kTcPacked + kTcBMax;   // 24 KB (multiple of 1 KB)
constexpr int kTcSmem = kTcStages * kTcStage + 1024;
constexpr int kTcThreads = 320;                    // warp 0 TMA, warp 1 MMA, warps 2-9 decode + epilogue
constexpr int kTcDecoders = 256;
constexpr int kTcGroups = 4;                       // decode groups working on different steps
// A slot is always decoded by the same group (step % stages fixes step % groups),
// so a group that waits on a slot has seen that slot's previous phase itself.
static_assert(kTcStages % kTcGroups == 0, "each ring slot must belong to one decode group");
static_assert(kTcBlocks * 4 == (kTcThreads - 64) / 32, "one epilogue warp per (accumulator, TMEM lane quarter)");

// instruction descriptor, kind::i8: D s32, A and B signed 8-bit, A MN-major,
// B K-major, M = 128, N = NPAD
template <int NPAD>
constexpr uint32_t i8_idesc() {
  return (2u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (0u << 16) |
         ((uint32_t)(NPAD >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                                 uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                          // sm_100 descriptor version
  d |= (uint64_t)layout << 61;
  return d;
}

__device__ __forceinline__ void tc_tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait on a stage barrier that gives up early once another role has
// aborted.  The abort flag is read only after failed polls: a shared-memory
// load costs hundreds of cycles while the ring, the decoders and the tensor
// core keep shared memory busy, so the fast path (phase already complete)
// touches nothing but the barrier.
enum TcWait { TC_READY = 0, TC_ABORTED = 1, TC_TIMEOUT = 2 };
__device__ __forceinline__ int tc_wait(uint64_t* bar, uint32_t parity, const int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return TC_READY;
    if ((i & 15u) == 15u && *(volatile const int*)abort_flag) return TC_ABORTED;
  }
  return TC_TIMEOUT;
}

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc_bits, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc_bits), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit accumulator columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 8 packed 2-bit codes (16 bits) -> 8 nibbles: code k moves to bits 4k..4k+1
__device__ __forceinline__ uint32_t spread_codes(uint32_t x) {
  x &= 0xFFFFu;
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  return (x | (x << 2)) & 0x33333333u;
}

// one packed word (16 codes: 00 -> 0, 01 -> +1, 10 -> -1) -> 16 int8, in
// column order: each nibble selects a byte of {0, +1, -1} (byte permute)
__device__ __forceinline__ uint4 decode_word(uint32_t w) {
  constexpr uint32_t kVals = 0x00FF0100u;          // bytes 0, +1, -1
  const uint32_t lo = spread_codes(w), hi = spread_codes(w >> 16);
  return make_uint4(__byte_perm(kVals, 0u, lo & 0xFFFFu), __byte_perm(kVals, 0u, lo >> 16),
                    __byte_perm(kVals, 0u, hi & 0xFFFFu), __byte_perm(kVals, 0u, hi >> 16));
}

template <int NPAD>
__global__ void __launch_bounds__(kTcThreads, 1)
    qgemv_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_q,
                    QGemvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t s_full[kTcStages];     // TMA -> decoders
  __shared__ __align__(8) uint64_t s_dec[kTcStages];      // decoders -> MMA
  __shared__ __align__(8) uint64_t s_empty[kTcStages];    // MMA (commit) -> TMA
  __shared__ __align__(8) uint64_t s_accum;               // every MMA done -> epilogue
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  constexpr uint32_t kTmemCols = (kTcBlocks * NPAD) <= 32 ? 32 : ((kTcBlocks * NPAD) <= 64 ? 64 : 128);
  constexpr int kBBytes = NPAD * kTcK;             // codes of one K chunk

  pdl_begin();
  grid_zero(a.zero, a.zero_n);
  const GemvPlan& P = a.plan;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ct = blockIdx.x, s = blockIdx.y;
  const int d_in = a.d_in, d_out = a.d_out;
  const int T = a.T;
  const int col0 = ct * kTcCols;
  // rows [r0, r1) of this split, in whole steps of 32
  const int steps_all = (d_in + kTcRows - 1) / kTcRows;
  const int st0 = (int)(((long long)steps_all * s) / P.S);
  const int st1 = (int)(((long long)steps_all * (s + 1)) / P.S);
  const int nsteps = st1 - st0;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_dec[i], kTcDecoders / 32 / kTcGroups);   // one arrive per warp of the step's group
      mbar_init(&s_empty[i], 1);
    }
    mbar_init(&s_accum, 1);
    mbar_fence_init();
    s_abort = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ----
      int it = 0;
      for (; it < nsteps; ++it) {
        const int sl = it % kTcStages;
        if (it >= kTcStages) {
          const int w = tc_wait(&s_empty[sl], (uint32_t)((it / kTcStages) - 1) & 1u, &s_abort);
          if (w == TC_TIMEOUT) {
            dev_fail(a.status, DEV_TIMEOUT, 50, (uint32_t)it);
            atomicExch(&s_abort, 1);
          }
          if (w != TC_READY) break;
        }
        const uint32_t sp = base + (uint32_t)(sl * kTcStage) + kTcBlocks * kTcATile;
        const uint32_t sq = sp + kTcPacked;
        mbar_arrive_expect_tx(&s_full[sl], (uint32_t)(kTcPacked + kTcKc * kBBytes));
        const int row = (st0 + it) * kTcRows;
        tc_tma_2d(sp, &map_w, col0 / 16, row, &s_full[sl]);
#pragma unroll
        for (int kc = 0; kc < kTcKc; ++kc)        // one 32-row codes box per K chunk
          tc_tma_2d(sq + (uint32_t)(kc * kTcBChunk), &map_q, row + kc * kTcK, 0, &s_full[sl]);
      }
      // on an abort, let the copies already issued land
      if (*(volatile int*)&s_abort) {
        for (int i = 0; i < kTcStages && i < it; ++i) {
          const int g = it - 1 - i;
          mbar_wait(&s_full[g % kTcStages], (uint32_t)(g / kTcStages) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      bool issued = false;
      for (int it = 0; it < nsteps; ++it) {
        const int sl = it % kTcStages;
        const int w = tc_wait(&s_dec[sl], (uint32_t)(it / kTcStages) & 1u, &s_abort);
        if (w == TC_TIMEOUT) {
          dev_fail(a.status, DEV_TIMEOUT, 51, (uint32_t)it);
          atomicExch(&s_abort, 1);
        }
        if (w != TC_READY) break;
        tc_after();
        const uint32_t sa = base + (uint32_t)(sl * kTcStage);
        const uint32_t sq = sa + kTcBlocks * kTcATile + kTcPacked;
#pragma unroll
        for (int kc = 0; kc < kTcKc; ++kc) {
          // B: K-major codes, 32-byte rows (one token each), 32-byte swizzle, 8-row groups 256 B apart
          const uint64_t bd = tc_smem_desc(sq + (uint32_t)(kc * kTcBChunk), 16, 256, 6);
#pragma unroll
          for (int b = 0; b < kTcBlocks; ++b) {
            // A: MN-major, 128-byte rows (one input row each), 128-byte swizzle, 8-row groups
            // 1 KB apart; K chunk kc starts kTcK rows in
            const uint64_t ad = tc_smem_desc(sa + (uint32_t)(b * kTcATile + kc * kTcK * 128), 16, 1024, 2);
            umma_i8(tmem + (uint32_t)(b * NPAD), ad, bd, i8_idesc<NPAD>(), (it > 0 || kc > 0) ? 1u : 0u);
          }
        }
        tc_commit(&s_empty[sl]);                   // frees the stage once these MMAs have read it
        issued = true;
      }
      tc_commit(&s_accum);                         // the accumulators are complete (or abandoned)
      if (!issued) {
        // no MMA was issued: the commit above still arrives once nothing is pending
      }
    }
  } else {
    // ---- decoders: 2-bit codes -> int8 A tiles ----
    // Four groups of two warps take every fourth step, so that the steps'
    // proxy fences (decoded tiles -> tensor core) overlap; a thread decodes
    // one 128-column row segment (8 words) of its group's step.
    const int dt = threadIdx.x - 64;               // 0..255
    const int grp = dt >> 6;                       // decode group (0..3)
    const int gt = dt & 63;
    const int r0 = gt >> 1;                        // rows r0 and r0 + 32 of the step
    const int blk = gt & 1;                        // A tile (columns 0..127 or 128..255)
    for (int it = grp; it < nsteps; it += kTcGroups) {
      const int sl = it % kTcStages;
      // the decode warps are the stage's only consumers: poll without sleeping
      // (a stage holds a fraction of a microsecond of work)
      const int w = tc_wait(&s_full[sl], (uint32_t)(it / kTcStages) & 1u, &s_abort);
      const bool ready = w == TC_READY;
      if (w == TC_TIMEOUT) {
        if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 52, (uint32_t)it);
        atomicExch(&s_abort, 1);
      }
      if (ready) {
        unsigned char* st = smem_raw + ((base - smem_u32(smem_raw)) + (uint32_t)(sl * kTcStage));
#pragma unroll
        for (int rr = 0; rr < kTcKc; ++rr) {
          const int r = r0 + rr * kTcK;
          const uint4* pw = reinterpret_cast<const uint4*>(st + kTcBlocks * kTcATile + r * (kTcWords * 4) + blk * 32);
          const uint4 p0 = pw[0], p1 = pw[1];
          const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
          unsigned char* at = st + blk * kTcATile + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)              // 16-byte chunk c holds columns 16c..16c+15
            *reinterpret_cast<uint4*>(at + ((c ^ (r & 7)) * 16)) = decode_word(words[c]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_dec[sl]);
    }
    // ---- epilogue: this CTA's partial sums -> its shared memory ----
    // (token-major [t][256 columns] int32; the ring is free: every MMA has
    // completed, so every stage has been read)
    const bool done = mbar_wait_backoff(&s_accum, 0u);
    if (!done && lane == 0) dev_fail(a.status, DEV_TIMEOUT, 53, 0u);
    tc_after();
    const int q = warp & 3;                        // this warp's TMEM lane quarter
    const int b = (warp - 2) >> 2;                 // its accumulator (128-column block)
    const bool abort = *(volatile int*)&s_abort || !done;
    int32_t* part = reinterpret_cast<int32_t*>(smem_raw + (base - smem_u32(smem_raw)));
    const int cl = b * 128 + q * 32 + lane;        // column within the CTA's 256
#pragma unroll
    for (int c0 = 0; c0 < NPAD; c0 += 16) {
      uint32_t v[16];
      tc_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * NPAD + c0), v);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c0 + e < T) part[(c0 + e) * kTcCols + cl] = abort ? 0 : (int32_t)v[e];
    }
  }
  // ---- free the tensor memory once every read of it is done ----
  tc_before();
  __syncthreads();
  if (warp == 1) {
    tc_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
  // per-token scales
  __shared__ float s_r[64];
  for (int t = threadIdx.x; t < T; t += kTcThreads) s_r[t] = __fdiv_rn(__fmul_rn(a.alpha, a.gamma[t]), 127.0f);

  // ---- the split CTAs of this column range are one cluster: after the
  // barrier each sums its slice of columns over every CTA's shared memory
  // (distributed shared memory), exactly in int32, and writes y.  Every
  // thread of every CTA reaches both cluster barriers (no early return). ----
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  const int S = P.S;
  const int rank = blockIdx.y;                     // the cluster spans blockIdx.y
  const int ncols = min(kTcCols, d_out - col0);
  const int slice = (((kTcCols + S - 1) / S + 3) / 4) * 4;   // ceil(256 / S), a multiple of 4
  const int cA = min(rank * slice, ncols), cB = min(cA + slice, ncols);
  const int ng = (cB - cA + 3) / 4;                // 4-column groups (ncols % 4 == 0)
  const uint32_t part_addr = base;
  for (int i = threadIdx.x; i < T * ng; i += kTcThreads) {
    const int t = i / ng, g = i - t * ng;
    const int c = cA + 4 * g;
    const uint32_t local = part_addr + (uint32_t)((t * kTcCols + c) * 4);
    int4 sum = make_int4(0, 0, 0, 0);
    for (int rr = 0; rr < S; ++rr) {
      uint32_t remote;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rr));
      int4 v;
      asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(remote)
                   : "memory");
      sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
    }
    const int iv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = col0 + c + e;
      if (c + e >= cB) break;
      const size_t o = (size_t)t * d_out + col;
      float yv = __fmul_rn(__int2float_rn(iv[e]), s_r[t]);
      if (a.gating) {                              // the quantized FFN's gate projection
        const float bu = (a.gating == 2 && a.b_up) ? a.b_up[col] : 0.0f;
        const float bg = (a.gating == 2 && a.b_gate) ? a.b_gate[col] : 0.0f;
        yv = quant_gate_value(a.gating, __ldcg(a.gate_u + o), yv, bu, bg);
      }
      a.y[o] = yv;
      if (a.acc) a.acc[o] = iv[e];
    }
  }
  // no CTA leaves while another may still read its shared memory
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
                 uint64_t outer, uint64_t pitch, uint32_t bx, uint32_t by, CUtensorMapSwizzle sw) {
  auto fn = tc_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {bx, by};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NPAD>
cudaError_t tc_launch(const QGemvArgs& a, const CUtensorMap& mw, const CUtensorMap& mq, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(qgemv_tc_kernel<NPAD>, kTcSmem, &configured);
  if (e != cudaSuccess) return e;
  // one cluster per column range: its S split CTAs (S <= 8, portable)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.plan.n_ct, a.plan.S, 1);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = (size_t)kTcSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = (unsigned)a.plan.S;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, qgemv_tc_kernel<NPAD>, mw, mq, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool qgemv_tc_supported(int T, int d_in, int d_out) {
  return T >= 8 && T <= 64 && d_in >= 1 && (d_in % 16) == 0 && (d_out % 64) == 0 &&
         tc_encode_fn() != nullptr;
}

GemvPlan plan_qgemv_tc(int T, int d_in, int d_out) {
  GemvPlan p{};
  p.mma = 2;
  p.TT = ((T + 15) / 16) * 16;
  p.groups = 1;
  p.mats = 1;
  p.n_ct = (d_out + kTcCols - 1) / kTcCols;
  p.vec_tile = kTcWords;
  p.threads = kTcThreads;
  p.rps = kTcRows;
  p.nst = kTcStages;
  p.rcap = 0;
  p.smem = kTcSmem;
  // splits: about two CTAs per SM, at most 8 (each split adds T x d_out exact
  // partial sums), at least 4 steps of 64 rows each
  const int steps = (d_in + kTcRows - 1) / kTcRows;
  long S = (2L * kNumSMs) / p.n_ct;
  if (S > 8) S = 8;
  if (S > steps / 4) S = steps / 4;
  if (S < 1) S = 1;
  p.S = (int)S;
  p.copies = 1;
  p.parts_elems = 0;                              // split sums meet in distributed shared memory
  p.tickets = 0;
  return p;
}

cudaError_t launch_qgemv_tc(const QGemvArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  if (a.xq == nullptr || a.plan.mma != 2) return cudaErrorInvalidValue;
  CUtensorMap mw, mq;
  const int row_words = a.d_out / 16;
  // packed W^T [d_in rows][row_words] u32: box 16 words (64 B) x 64 rows, no swizzle
  if (!make_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.wp, (uint64_t)row_words, (uint64_t)a.d_in,
                   (uint64_t)row_words * 4, kTcWords, kTcRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const int npad = a.plan.TT;
  // dense masked codes [T][d_in] int8: box 32 (rows, one K chunk) x npad tokens, 32-byte swizzle
  if (!make_map_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.xq, (uint64_t)a.d_in, (uint64_t)a.T,
                   (uint64_t)a.d_in, kTcK, (uint32_t)npad, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  switch (npad) {
    case 16: return tc_launch<16>(a, mw, mq, s);
    case 32: return tc_launch<32>(a, mw, mq, s);
    case 48: return tc_launch<48>(a, mw, mq, s);
    case 64: return tc_launch<64>(a, mw, mq, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qs
