// One-token sparse FFN layer as ONE persistent kernel (every CTA resident).
//
// Q-Sparse news article (zxwl-tech.com), "Top-K sparsification": the K
// largest |x| of the token are kept, the rest set to zero; the projections
// then only need the weight rows of the kept inputs.  Turbo Sparse summary
// (blog.csdn.net), Eq. 2 (dReLU) and the squared-ReLU GLU of the Q-Sparse
// paper summary (shd-paper.top, method section): h = act(u, g) with
// u = x_s W_up^T, g = x_s W_gate^T; the down projection takes the top-K of
// |h|.  aibase.com summary, "Vantagens da ativação esparsa": one-token decode
// is bound by the weight bytes read, so this path is about latency between
// the steps: the separate kernels of the general path pay a grid completion
// and a wake-up at each of their four boundaries, here the steps are phases
// of one grid separated by grid barriers.
//
// Phases (every CTA takes part in every barrier; none returns early):
//   A  top-K on |x|: every CTA finds the K-th largest key of the whole row by a
//      radix select (x staged in shared memory) and lists the kept inputs of
//      its own index range, with its position in the global list (the
//      lower index wins a tie, the oracle's rule);
//   B  up and gate projections over those rows (bulk-copy ring of row tiles);
//      each CTA stores its partial sums in its own slot (no accumulator to
//      clear, a fixed summation order later);
//   -- grid barrier --
//   C  h = act(u, g) for one index range of d_ff per CTA (sum of the slots in
//      split order) and its nonzero h;
//   D  down projection over those nonzero h, partial sums added into the
//      accumulator (cleared in phase A): these are the kept h whenever the
//      whole row has at most K_h nonzero h;
//   -- grid barrier --
//      the nonzero count of the row decides: at most K_h, the h list is
//      written; otherwise the accumulator is cleared, -- grid barrier --,
//      every CTA finds the K_h-th largest |h| by a radix select over h and D
//      runs again over the kept rows, -- grid barrier --;
//   E  y = the accumulator rounded to bf16; the last CTA to leave resets the
//      barrier counters.
// The row lists and their counts are written as by the general path (so the
// workspace statistics and list read-back stay valid).
#include <mutex>

#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr int kFThreads = 384;                     // 11 consumer warps + 1 producer warp
constexpr int kFConsumers = kFThreads - 32;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFStages = 5;
constexpr int kFStageBytes = 16896;                // 3 row tiles of <= 5632 B
constexpr int kFMaxRange = 1024;                   // rows one CTA may list per phase
constexpr int kFMaxDModel = 8192;                  // x staged in shared memory (bf16)
constexpr uint32_t kBarLimit = 1u << 20;           // grid-barrier polls before giving up

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every CTA arrives once; the waits are bounded (the occupancy-sized grid is
// resident when these layers run alone on the device, and always under a
// cooperative launch; a wait that runs out records DEV_TIMEOUT and the kernel
// goes on, it never hangs).
__device__ __forceinline__ void grid_barrier(int32_t* ctr, int G, DevStatus* st, int where,
                                             int* s_err) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1);
    uint32_t it = 0;
    while (ld_acquire_gpu(ctr) < G) {
      if (++it > kBarLimit) {
        dev_fail(st, DEV_TIMEOUT, 60 + where, (uint32_t)ld_acquire_gpu(ctr));
        *s_err = 1;
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
  }
  __syncthreads();
}

// Exclusive block-wide prefix of two predicates (ballots, then the warps'
// counts); returns this thread's prefixes and the block totals.
__device__ __forceinline__ void block_scan_pred2(bool p, bool q, uint32_t* s_w, int& ep, int& eq,
                                                 int& tp, int& tq) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bp = __ballot_sync(0xffffffffu, p), bq = __ballot_sync(0xffffffffu, q);
  if (lane == 0) s_w[warp] = (uint32_t)__popc(bp) | ((uint32_t)__popc(bq) << 16);
  __syncthreads();
  int pp = 0, pq = 0, sp = 0, sq = 0;
  for (int w = 0; w < kFWarps; ++w) {
    const uint32_t v = s_w[w];
    if (w < warp) { pp += (int)(v & 0xffffu); pq += (int)(v >> 16); }
    sp += (int)(v & 0xffffu);
    sq += (int)(v >> 16);
  }
  ep = pp + __popc(bp & lanemask_lt());
  eq = pq + __popc(bq & lanemask_lt());
  tp = sp;
  tq = sq;
  __syncthreads();                                 // s_w is reused by the next call
}

__device__ __forceinline__ int block_sum(int v, int* s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) s_w[warp] = v;
  __syncthreads();
  int s = 0;
  for (int w = 0; w < kFWarps; ++w) s += s_w[w];
  __syncthreads();
  return s;
}

// The k-th largest of n magnitude keys (1 <= k <= n, keys < 2^nbits, nbits >=
// 11): returns tau (that key) and need (how many of the keys equal to tau are
// among the k largest).  Radix select from the top: the first pass counts the
// top 11 bits into one 2048-bin histogram (h2k: idle shared memory), which
// spreads the keys of a warp over many bins (a narrow first digit would be the
// exponent alone, a few bins for most data, and serialise the atomics); the
// later passes take up to 8 bits each into s_hist.
template <typename KeyFn>
__device__ void block_kth_largest(KeyFn key, int n, int k, int nbits, int* h2k, int* s_hist,
                                  int* s_pick, int* s_w, uint32_t& tau, int& need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sh1 = nbits - 11;
  for (int j = tid; j < 2048; j += kFThreads) h2k[j] = 0;
  for (int j = tid; j < 256; j += kFThreads) s_hist[j] = 0;
  __syncthreads();
  for (int e = tid; e < n; e += kFThreads) atomicAdd(&h2k[key(e) >> sh1], 1);
  __syncthreads();
  // threads 0..255 hold 8 bins each, in descending order from the top bin
  int c[8], sum = 0;
  if (tid < 256) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = h2k[2047 - 8 * tid - q];
      sum += c[q];
    }
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31 && warp < 8) s_w[warp] = incl;
  __syncthreads();
  if (tid < 256) {
    for (int w = 0; w < warp; ++w) incl += s_w[w];
    const int excl = incl - sum;
    if (excl < k && k <= incl) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + c[q] >= k) {
          s_pick[0] = 2047 - 8 * tid - q;
          s_pick[1] = run;
          break;
        }
        run += c[q];
      }
    }
  }
  __syncthreads();
  uint32_t prefix = (uint32_t)s_pick[0] << sh1, pmask = 0x7ffu << sh1;
  int rem = k - s_pick[1];
  int sh = sh1;
  while (sh > 0) {                                 // (block-uniform)
    const int w = sh < 8 ? sh : 8;
    sh -= w;
    const uint32_t dmask = (1u << w) - 1u;
    for (int e = tid; e < n; e += kFThreads) {
      const uint32_t kk = key(e);
      if ((kk & pmask) == prefix) atomicAdd(&s_hist[(kk >> sh) & dmask], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8l .. 248 - 8l (descending)
      int d[8], dsum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        d[q] = s_hist[255 - 8 * lane - q];
        dsum += d[q];
      }
      int dincl = dsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, dincl, o);
        if (lane >= o) dincl += v;
      }
      const int dexcl = dincl - dsum;
      if (dexcl < rem && rem <= dincl) {
        int run = dexcl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + d[q] >= rem) {
            s_pick[0] = 255 - 8 * lane - q;
            s_pick[1] = run;
            break;
          }
          run += d[q];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_pick[0] << sh;
    pmask |= dmask << sh;
    rem -= s_pick[1];
    if (sh > 0) {                                  // the next pass counts into a cleared s_hist
      for (int j = tid; j < 256; j += kFThreads) s_hist[j] = 0;
      __syncthreads();
    }
  }
  tau = prefix;
  need = rem;
}

struct Selection {
  uint32_t tau;        // the K-th largest key (0xffffffff: nothing kept)
  int need;            // keys equal to tau that are kept (lowest indices first)
  int gt_before;       // keys > tau below the range start
  int ties_before;     // keys == tau below the range start
};

// Kept inputs of [r0, r1) with a nonzero value, in index order, into s_rows /
// s_vals; returns their number.  valf(e) is the value, key(e) its magnitude key.
template <typename KeyFn, typename ValFn>
__device__ int list_range(const Selection& S, KeyFn key, ValFn valf, int r0, int r1, int* s_rows,
                          float* s_vals, uint32_t* s_w) {
  int tie_base = S.ties_before, pos = 0;
  for (int c0 = r0; c0 < r1; c0 += kFThreads) {
    const int e = c0 + (int)threadIdx.x;
    const bool valid = e < r1;
    const uint32_t kk = valid ? key(e) : 0u;
    const bool tie = valid && kk == S.tau;
    // tie rank first (a kept tie needs the ties before it)
    int et, unused_e, tt, unused_t;
    block_scan_pred2(tie, false, s_w, et, unused_e, tt, unused_t);
    const bool sel = valid && kk != 0u && (kk > S.tau || (tie && tie_base + et < S.need));
    int es, tsel;
    block_scan_pred2(sel, false, s_w, es, unused_e, tsel, unused_t);
    if (sel) {
      s_rows[pos + es] = e;
      s_vals[pos + es] = valf(e);
    }
    tie_base += tt;
    pos += tsel;
  }
  __syncthreads();
  return pos;
}

// Top-K selection of n keys restricted to [r0, r1): tau, need and the counts
// below r0.  k <= 0 keeps nothing, k >= n keeps everything.
template <typename KeyFn>
__device__ Selection select_topk(KeyFn key, int n, int k, int nbits, int r0, int* whist,
                                 int* s_hist, int* s_pick, int* s_w) {
  Selection S;
  if (k <= 0) {
    S.tau = 0xffffffffu; S.need = 0; S.gt_before = 0; S.ties_before = 0;
    return S;
  }
  if (k >= n) {
    S.tau = 0u; S.need = n;                        // every key is > 0 or a kept tie at 0
  } else {
    block_kth_largest(key, n, k, nbits, whist, s_hist, s_pick, s_w, S.tau, S.need);
  }
  int cnt = 0;                                     // (> tau) + (== tau) << 16, each < 65536
  for (int e = (int)threadIdx.x; e < r0; e += kFThreads) {
    const uint32_t kk = key(e);
    cnt += (kk > S.tau ? 1 : 0) + (kk == S.tau ? 0x10000 : 0);
  }
  const uint32_t both = (uint32_t)block_sum(cnt, s_w);   // (wraps as unsigned: exact)
  S.gt_before = (int)(both & 0xffffu);
  S.ties_before = (int)(both >> 16);
  return S;
}

// Position of the range's first listed (nonzero) kept input in the global list.
__device__ __forceinline__ int list_offset(const Selection& S) {
  if (S.tau == 0xffffffffu) return 0;
  const int ties = S.ties_before < S.need ? S.ties_before : S.need;
  return S.gt_before + (S.tau != 0u ? ties : 0);
}

__device__ __forceinline__ void red_add_f32x8(float* dst, const float (&v)[8]) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v[0]), "f"(v[1]),
               "f"(v[2]), "f"(v[3])
               : "memory");
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4), "f"(v[4]), "f"(v[5]),
               "f"(v[6]), "f"(v[7])
               : "memory");
}

// Stream the listed rows' tiles through the ring; acc += v * row.
__device__ __forceinline__ void stream_rows(const unsigned char* Wb, size_t row_bytes, int tbytes,
                                            int tvec, int tile_bytes, int rps, int n,
                                            const int* s_rows, const float* s_vals,
                                            unsigned char* ring, uint64_t* s_full,
                                            uint64_t* s_empty, int& gst, float (&acc)[8],
                                            int* s_err, const FfnFusedArgs& a) {
  DevStatus* st = a.status;
  const int tid = threadIdx.x, lane = tid & 31;
  const bool producer = tid >= kFConsumers;
  const int nstage = (n + rps - 1) / rps;
  if (producer) {
    for (int s = 0; s < nstage && !a.no_copies; ++s) {
      const int g = gst + s;
      const int slot = g % kFStages;
      int ok = 1;
      if (lane == 0 && g >= kFStages &&
          !mbar_wait(&s_empty[slot], (uint32_t)((g / kFStages) - 1) & 1u)) {
        dev_fail(st, DEV_TIMEOUT, 70, (uint32_t)g);
        atomicExch(s_err, 1);
        ok = 0;
      }
      if (__shfl_sync(0xffffffffu, ok, 0) == 0) break;
      const int j0 = s * rps;
      const int cnt = min(rps, n - j0);
      if (lane == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cnt * tbytes));
      __syncwarp();
      for (int r = lane; r < cnt; r += 32)
        bulk_g2s(ring + ((size_t)slot * rps + r) * tile_bytes, Wb + (size_t)s_rows[j0 + r] * row_bytes,
                 (uint32_t)tbytes, &s_full[slot]);
    }
  } else {
    for (int s = 0; s < nstage; ++s) {
      const int g = gst + s;
      const int slot = g % kFStages;
      bool ready = false;
      for (uint32_t i = 0; i < a.wait_limit; ++i) {  // abort flag read only after failed polls
        if (mbar_try_wait(&s_full[slot], (uint32_t)(g / kFStages) & 1u)) { ready = true; break; }
        if ((i & 15u) == 15u && *(volatile int*)s_err) break;
      }
      if (!ready && !*(volatile int*)s_err) {
        if (lane == 0) dev_fail(st, DEV_TIMEOUT, 71, (uint32_t)g);
        atomicExch(s_err, 1);
      }
      const int j0 = s * rps;
      const int cnt = min(rps, n - j0);
      if (ready && tid < tvec) {
        for (int r = 0; r < cnt; ++r) {
          const uint4 q = *reinterpret_cast<const uint4*>(ring + ((size_t)slot * rps + r) * tile_bytes +
                                                          (size_t)tid * 16);
          const float v = s_vals[j0 + r];
          const float w[8] = {bf16lo(q.x), bf16hi(q.x), bf16lo(q.y), bf16hi(q.y),
                              bf16lo(q.z), bf16hi(q.z), bf16lo(q.w), bf16hi(q.w)};
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(v, w[e], acc[e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[slot]);
    }
  }
  gst += nstage;
  __syncthreads();
}

__global__ void __launch_bounds__(kFThreads, 2) ffn_fused_kernel(FfnFusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[kFStages];
  __shared__ __align__(8) uint64_t s_empty[kFStages];
  __shared__ int s_hist[256];
  __shared__ int s_pick[2];
  __shared__ uint32_t s_w[kFWarps];
  __shared__ int s_err;
  __shared__ int s_tot[2];

  const FfnFusedPlan& P = a.plan;
  const int tid = threadIdx.x, lane = tid & 31;
  const int c = blockIdx.x;
  const int G = gridDim.x;
  const int d_model = a.d_model, d_ff = a.d_ff;
  unsigned char* ring = smem;
  int* whist = reinterpret_cast<int*>(ring);       // selection histograms: the ring is idle then
  int* s_rows = reinterpret_cast<int*>(smem + (size_t)kFStages * kFStageBytes);
  float* s_vals = reinterpret_cast<float*>(s_rows + kFMaxRange);
  uint16_t* s_x = reinterpret_cast<uint16_t*>(s_vals + kFMaxRange);

  // Programmatic dependent launch: the next launch may start its set-up now
  // (it waits for this grid's completion before it touches memory); this
  // grid touches nothing that the previous one reads or writes before its wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    for (int i = 0; i < kFStages; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kFConsumers / 32);
    }
    mbar_fence_init();
    s_err = 0;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ---- A: top-K on |x| (x loads first: the longest latency of the phase) ----
  const uint16_t* xg = reinterpret_cast<const uint16_t*>(a.x);
  for (int e = tid; e < d_model; e += kFThreads) s_x[e] = xg[e];
  // the down accumulator: cleared before the first barrier, added to after it
  for (int j = c * kFThreads + tid; j < d_model / 4; j += G * kFThreads)
    reinterpret_cast<float4*>(a.pdn)[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  __syncthreads();
  const int units_ug = 2 * P.n_ct_ug;
  const bool ug_active = c < units_ug * P.S_ug;
  const int ug_unit = c / P.S_ug, ug_rr = c - (c / P.S_ug) * P.S_ug;
  const int mat = ug_unit & 1, ct_ug = ug_unit >> 1;
  const int r0 = (int)(((long long)d_model * ug_rr) / P.S_ug);
  const int r1 = (int)(((long long)d_model * (ug_rr + 1)) / P.S_ug);
  auto xkey = [&](int e) -> uint32_t { return (uint32_t)s_x[e] & 0x7fffu; };
  auto xval = [&](int e) -> float { return __uint_as_float((uint32_t)s_x[e] << 16); };
  int n_x = 0;
  if (ug_active) {                                 // (block-uniform)
    // (an even split of the kept rows by list position measured slower: the
    // splits' finish times spread by about 4 us even with equal row counts,
    // from uneven bandwidth across the SMs, and the listing costs more)
    const Selection Sx = select_topk(xkey, d_model, a.k_in, 15, r0, whist, s_hist, s_pick,
                                     reinterpret_cast<int*>(s_w));
    n_x = list_range(Sx, xkey, xval, r0, r1, s_rows, s_vals, s_w);
    if (ug_unit == 0) {                            // one copy of the list
      const int off = list_offset(Sx);
      for (int j = tid; j < n_x; j += kFThreads) {
        a.list_x[off + j] = s_rows[j];
        a.lval_x[off + j] = s_vals[j];
      }
      if (ug_rr == P.S_ug - 1 && tid == 0) a.cnt[0] = off + n_x;
    }
  }

  // ---- B: up and gate projections -------------------------------------------
  int gst = 0;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  if (ug_active) {
    const size_t row_bytes = (size_t)d_ff * 2;
    const int tile_bytes = P.vt_ug * 16;
    const size_t cbyte = (size_t)ct_ug * tile_bytes;
    const int tbytes = (int)min((size_t)tile_bytes, row_bytes - cbyte);
    const int tvec = tbytes / 16;
    const unsigned char* Wb =
        reinterpret_cast<const unsigned char*>(mat == 0 ? a.w_up : a.w_gate) + cbyte;
    stream_rows(Wb, row_bytes, tbytes, tvec, tile_bytes, P.rps_ug, n_x, s_rows, s_vals, ring, s_full,
                s_empty, gst, acc, &s_err, a);
    if (tid < tvec) {                              // every slot entry is written (zeros too)
      float* dst = a.pug + ((size_t)ug_rr * 2 + mat) * d_ff + ((size_t)ct_ug * P.vt_ug + tid) * 8;
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  grid_barrier(a.bar + 0, G, a.status, 0, &s_err);

  // ---- C+D: h of this CTA's index range, then the down projection over its
  // nonzero h.  Taking the nonzero h is right when there are at most K_h of
  // them in the whole row (the count is known only after the next barrier;
  // otherwise the down phase is done again below with the full selection).
  const bool dn_active = c < P.n_ct_dn * P.S_dn;
  const int ct_dn = c / P.S_dn, dn_rr = c - (c / P.S_dn) * P.S_dn;
  const int q0 = (int)(((long long)d_ff * dn_rr) / P.S_dn);
  const int q1 = (int)(((long long)d_ff * (dn_rr + 1)) / P.S_dn);
  const size_t dn_row_bytes = (size_t)d_model * 2;
  const int dn_tile_bytes = P.vt_dn * 16;
  const size_t dn_cbyte = (size_t)ct_dn * dn_tile_bytes;
  const int dn_tbytes = dn_active ? (int)min((size_t)dn_tile_bytes, dn_row_bytes - dn_cbyte) : 0;
  const int dn_tvec = dn_tbytes / 16;
  const unsigned char* Wd = reinterpret_cast<const unsigned char*>(a.w_down) + dn_cbyte;
  int n_h = 0;
  if (dn_active) {
    const int len = q1 - q0;
    const int np = 2 * len;                        // (matrix, index) pairs
    const int H = min(8, max(1, kFThreads / max(np, 1)));   // split of the slots per pair
    float* s_part = reinterpret_cast<float*>(ring);          // the ring is idle here
    if (tid < np * H) {
      const int pr = tid % np, hh = tid / np;
      const int m = pr >= len ? 1 : 0, i = q0 + (pr - m * len);
      const int s0 = (P.S_ug * hh) / H, s1 = (P.S_ug * (hh + 1)) / H;
      const float* src = a.pug + (size_t)m * d_ff + i;
      float v = 0.0f;
      for (int sb = s0; sb < s1; sb += 24) {       // 24 loads in flight, summed in slot order
        float t[24];
#pragma unroll
        for (int j = 0; j < 24; ++j) t[j] = sb + j < s1 ? __ldcg(src + (size_t)(sb + j) * 2 * d_ff) : 0.0f;
#pragma unroll
        for (int j = 0; j < 24; ++j) v += t[j];
      }
      s_part[hh * np + pr] = v;
    }
    __syncthreads();
    // h of [q0, q1) from the two sums, its nonzero h listed in index order
    for (int c0 = 0; c0 < len; c0 += kFThreads) {
      const int j = c0 + tid;
      float hv = 0.0f;
      if (j < len) {
        float u = 0.0f, g = 0.0f;
        for (int hh = 0; hh < H; ++hh) {           // fixed order
          u += s_part[hh * np + j];
          g += s_part[hh * np + len + j];
        }
        const int i = q0 + j;
        if (a.act == 1) {
          const float r = fmaxf(u, 0.0f);
          hv = (r * r) * g;
        } else {
          const float bu = a.b_up ? a.b_up[i] : 0.0f;
          const float bg = a.b_gate ? a.b_gate[i] : 0.0f;
          hv = fmaxf(g + bg, 0.0f) * fmaxf(u + bu, 0.0f);
        }
        if (ct_dn == 0) a.h[i] = hv;
      }
      const bool nz = j < len && hv != 0.0f;
      int ep, unused_e, tp, unused_t;
      block_scan_pred2(nz, false, s_w, ep, unused_e, tp, unused_t);
      if (nz) {
        s_rows[n_h + ep] = q0 + j;
        s_vals[n_h + ep] = hv;
      }
      n_h += tp;
      __syncthreads();
    }
    if (ct_dn == 0 && tid == 0) a.hnz[dn_rr] = n_h;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;     // (phase B's sums are stored)
    stream_rows(Wd, dn_row_bytes, dn_tbytes, dn_tvec, dn_tile_bytes, P.rps_dn, n_h, s_rows, s_vals,
                ring, s_full, s_empty, gst, acc, &s_err, a);
    if (tid < dn_tvec) {
      float* dst = a.pdn + ((size_t)ct_dn * P.vt_dn + tid) * 8;
      red_add_f32x8(dst, acc);
    }
  }
  grid_barrier(a.bar + 1, G, a.status, 1, &s_err);

  // ---- the nonzero count of h: total and below this range ---------------------
  if (tid < 32) {
    int tot = 0, pre = 0;
    for (int j = lane; j < P.S_dn; j += 32) {
      const int v = __ldcg(a.hnz + j);
      tot += v;
      pre += j < dn_rr ? v : 0;
    }
    tot = __reduce_add_sync(0xffffffffu, tot);
    pre = __reduce_add_sync(0xffffffffu, pre);
    if (lane == 0) { s_tot[0] = tot; s_tot[1] = pre; }
  }
  __syncthreads();
  const bool fallback = s_tot[0] > a.k_h;          // (grid-uniform)
  if (!fallback) {
    if (dn_active && ct_dn == 0) {
      for (int j = tid; j < n_h; j += kFThreads) {
        a.list_h[s_tot[1] + j] = s_rows[j];
        a.lval_h[s_tot[1] + j] = s_vals[j];
      }
      if (dn_rr == P.S_dn - 1 && tid == 0) a.cnt[1] = s_tot[0];
    }
  } else {
    // ---- more than K_h nonzero h: the down phase again, over the top-K of |h| --
    for (int j = c * kFThreads + tid; j < d_model / 4; j += G * kFThreads)
      reinterpret_cast<float4*>(a.pdn)[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    grid_barrier(a.bar + 2, G, a.status, 2, &s_err);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    if (dn_active) {
      auto hkey = [&](int e) -> uint32_t { return __float_as_uint(__ldcg(a.h + e)) & 0x7fffffffu; };
      auto hval = [&](int e) -> float { return __ldcg(a.h + e); };
      const Selection Sh = select_topk(hkey, d_ff, a.k_h, 31, q0, whist, s_hist, s_pick,
                                       reinterpret_cast<int*>(s_w));
      n_h = list_range(Sh, hkey, hval, q0, q1, s_rows, s_vals, s_w);
      if (ct_dn == 0) {
        const int off = list_offset(Sh);
        for (int j = tid; j < n_h; j += kFThreads) {
          a.list_h[off + j] = s_rows[j];
          a.lval_h[off + j] = s_vals[j];
        }
        if (dn_rr == P.S_dn - 1 && tid == 0) a.cnt[1] = off + n_h;
      }
      stream_rows(Wd, dn_row_bytes, dn_tbytes, dn_tvec, dn_tile_bytes, P.rps_dn, n_h, s_rows, s_vals,
                  ring, s_full, s_empty, gst, acc, &s_err, a);
      if (tid < dn_tvec) {
        float* dst = a.pdn + ((size_t)ct_dn * P.vt_dn + tid) * 8;
        red_add_f32x8(dst, acc);
      }
    }
    grid_barrier(a.bar + 3, G, a.status, 3, &s_err);
  }

  // ---- E: y ------------------------------------------------------------------
  uint16_t* y = reinterpret_cast<uint16_t*>(a.y);
  for (int j = c * kFThreads + tid; j < d_model / 4; j += G * kFThreads) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(a.pdn) + j);
    uint2 q;
    q.x = (uint32_t)f32_to_bf16_bits(v.x) | ((uint32_t)f32_to_bf16_bits(v.y) << 16);
    q.y = (uint32_t)f32_to_bf16_bits(v.z) | ((uint32_t)f32_to_bf16_bits(v.w) << 16);
    reinterpret_cast<uint2*>(y)[j] = q;
  }
  if (s_err && tid == 0 && !a.no_copies) {
    // a stage wait gave up: let the copies already issued land before leaving
    for (int i = 0; i < kFStages && i < gst; ++i) {
      const int g_last = gst - 1 - i;
      mbar_wait(&s_full[g_last % kFStages], (uint32_t)(g_last / kFStages) & 1u);
    }
  }
  // the last CTA out resets the barrier counters (every CTA is past every wait)
  if (tid == 0 && atomicAdd(a.bar + 4, 1) == G - 1) {
    for (int i = 0; i < 5; ++i) a.bar[i] = 0;
  }
}

int fused_grid() {
  static int G = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0, sms = 0, nb = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      G = 0;
      return;
    }
    if (cudaFuncSetAttribute(ffn_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)ffn_fused_smem()) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, ffn_fused_kernel, kFThreads,
                                                      ffn_fused_smem()) != cudaSuccess) {
      G = 0;
      return;
    }
    nb = nb > 2 ? 2 : nb;
    G = nb * sms;
    if (G > 2 * kNumSMs) G = 2 * kNumSMs;
  });
  return G;
}

// Column tiles of a bf16 row of `d` outputs for 352 consumer threads (one
// 16-byte vector each), preferring equal tiles.
void fused_tiles(int d, int* n_ct, int* vt) {
  const int vec_row = d / 8;
  int nct = (vec_row + kFConsumers - 1) / kFConsumers;
  for (int c = nct; c <= nct + 8 && c <= vec_row; ++c)
    if (vec_row % c == 0) { nct = c; break; }
  *n_ct = nct;
  *vt = (vec_row + nct - 1) / nct;
}

}  // namespace

size_t ffn_fused_smem() {
  return (size_t)kFStages * kFStageBytes + (size_t)kFMaxRange * 8 + (size_t)kFMaxDModel * 2;
}

bool plan_ffn_fused(int d_model, int d_ff, int G, FfnFusedPlan* p) {
  *p = FfnFusedPlan{};
  if (G < 2 || d_model < 8 || d_ff < 8 || d_model % 8 != 0 || d_ff % 8 != 0 || d_model > kFMaxDModel)
    return false;
  fused_tiles(d_ff, &p->n_ct_ug, &p->vt_ug);
  fused_tiles(d_model, &p->n_ct_dn, &p->vt_dn);
  if (p->vt_ug * 16 > kFStageBytes || p->vt_dn * 16 > kFStageBytes) return false;
  p->rps_ug = kFStageBytes / (p->vt_ug * 16);
  p->rps_dn = kFStageBytes / (p->vt_dn * 16);
  p->S_ug = G / (2 * p->n_ct_ug);
  p->S_dn = G / p->n_ct_dn;
  if (p->S_ug < 1 || p->S_dn < 1) return false;
  // rows one CTA lists: its index range of x, of h
  if ((d_model + p->S_ug - 1) / p->S_ug > kFMaxRange || (d_ff + p->S_dn - 1) / p->S_dn > kFMaxRange)
    return false;
  // h sums: (matrix, index) pairs of one range fit one block
  if (2 * ((d_ff + p->S_dn - 1) / p->S_dn) > kFThreads) return false;
  p->G = G;
  return true;
}

size_t ffn_fused_pug_elems(int d_model, int d_ff) {
  FfnFusedPlan p;
  if (!plan_ffn_fused(d_model, d_ff, 2 * kNumSMs, &p)) return 0;
  return (size_t)p.S_ug * 2 * d_ff;
}

int ffn_fused_grid() { return fused_grid(); }

// The grid is the occupancy-sized count of CTAs (ffn_fused_grid), all of which
// must be resident together for the grid barriers.  An ordinary launch with
// programmatic dependent launch is the default: a grid that follows another
// one-kernel layer on the stream is scheduled only after every CTA of that
// layer has started (each one triggers at entry) and takes their places as
// they leave, so on a device that runs these layers alone every CTA becomes
// resident, and the next layer's set-up overlaps this one's exit (about 1.7 us
// a launch less than a cooperative launch, with which the driver does not
// overlap launches).  `cooperative` asks for a cooperative launch instead,
// which the driver admits only when the whole grid can be resident: for
// callers that run other kernels concurrently on the device, where CTAs of an
// ordinary launch could wait for SMs that another kernel holds (every grid
// barrier wait is bounded and would end in DEV_TIMEOUT, never a hang).
cudaError_t launch_ffn_fused(const FfnFusedArgs& a_in, bool cooperative, cudaStream_t s) {
  FfnFusedArgs a = a_in;
  a.wait_limit = kWaitLimit;
  if (g_fault.mode == QS_FAULT_GATHER_NO_COPIES) {   // failure-detection tests only
    a.no_copies = 1;
    if (g_fault.wait_polls != 0) a.wait_limit = g_fault.wait_polls;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.plan.G);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = ffn_fused_smem();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (cooperative) {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, ffn_fused_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qs
