// Decode-regime gather-GEMV:  y[t, :] = sum_{i in rows} xs[t, i] * W^T[i, :]
//
// Source: Q-Sparse news article (zxwl-tech.com), section "Top-K
// sparsification" (X_sparse replaces X in Y = X.W^T, so the zeroed inputs
// need neither arithmetic nor their weights), and the aibase.com summary,
// "Vantagens da ativacao esparsa" (memory traffic, not arithmetic, bounds
// inference).  With W stored input-major (W^T, [d_in, d_out]) the weights of
// one kept input are one contiguous row, so the kernel streams exactly the
// rows listed by the top-K kernel (the union over the batch's tokens) and
// nothing else.
//
// Mapping (B200: 148 SMs, HBM3e).  Measured on this pattern (2867 kept rows
// of 22 KB): 512-byte segments per request stream at ~3.4 TB/s whatever the
// load depth, while 1-D bulk copies (TMA) of multi-KB row segments reach
// 6.0 TB/s over 4 GiB (5.5 KB every 22 KB; plain reads peak at 7.1 TB/s).  So:
//   * a row is cut into n_ct equal column tiles of a few KB (e.g. 4 x 5.5 KB
//     for 11008 bf16 columns); a CTA owns one tile, one weight matrix and a
//     contiguous slice of the row list (split-K);
//   * the producer warp issues a cp.async.bulk per kept row (a stage's rows
//     from its lanes side by side) into a ring of shared-memory stages guarded
//     by mbarriers (transaction-count completion); each wait is bounded and
//     reports DEV_TIMEOUT if it runs out;
//   * each consumer thread owns one 16-byte column vector of the tile for the
//     whole stream (f32 accumulators in registers, one per token), so no
//     cross-warp reduction is needed;
//   * the slice's row indices and per-token values are staged in shared
//     memory first (one round trip: the top-K kernel stores each listed row's
//     values next to the list);
//   * split partials are added with f32 vector reductions (red.add.v4.f32)
//     into an accumulator that the previous kernel of the call zeroed; the
//     last CTA of a column tile to arrive (an atomic ticket, nobody waits)
//     reads the sums once and runs the epilogue.  The epilogue
//     is the output cast, or the FFN gating h = ReLU(u)^2 * g (Q-Sparse
//     squared ReLU) or h = ReLU(g + b_g) * ReLU(u + b_u) (Turbo Sparse dReLU,
//     Eq. 2).  The order of the split additions is not fixed, so the last
//     bits of a split sum may differ between runs.
#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr int kMaxConsumers = 384;
constexpr int kMaxStages = 32;

template <typename WT> struct VecTraits;
template <> struct VecTraits<float> { static constexpr int V = 4; };
template <> struct VecTraits<__nv_bfloat16> { static constexpr int V = 8; };

template <typename WT>
__device__ __forceinline__ void unpack(const uint4& q, float (&w)[VecTraits<WT>::V]) {
  if constexpr (VecTraits<WT>::V == 8) {
    w[0] = bf16lo(q.x); w[1] = bf16hi(q.x);
    w[2] = bf16lo(q.y); w[3] = bf16hi(q.y);
    w[4] = bf16lo(q.z); w[5] = bf16hi(q.z);
    w[6] = bf16lo(q.w); w[7] = bf16hi(q.w);
  } else {
    w[0] = __uint_as_float(q.x); w[1] = __uint_as_float(q.y);
    w[2] = __uint_as_float(q.z); w[3] = __uint_as_float(q.w);
  }
}

__device__ __forceinline__ void red_add_v4(float* dst, float a0, float a1, float a2, float a3) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a0), "f"(a1), "f"(a2),
               "f"(a3)
               : "memory");
}

template <int V>
__device__ __forceinline__ void store_f32(float* dst, const float (&v)[V]) {
#pragma unroll
  for (int q = 0; q < V / 4; ++q)
    reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

template <typename WT>
__device__ __forceinline__ void store_y(void* y, size_t o, const float (&v)[VecTraits<WT>::V]) {
  if constexpr (VecTraits<WT>::V == 8) {
    uint4 q;
    q.x = (uint32_t)f32_to_bf16_bits(v[0]) | ((uint32_t)f32_to_bf16_bits(v[1]) << 16);
    q.y = (uint32_t)f32_to_bf16_bits(v[2]) | ((uint32_t)f32_to_bf16_bits(v[3]) << 16);
    q.z = (uint32_t)f32_to_bf16_bits(v[4]) | ((uint32_t)f32_to_bf16_bits(v[5]) << 16);
    q.w = (uint32_t)f32_to_bf16_bits(v[6]) | ((uint32_t)f32_to_bf16_bits(v[7]) << 16);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + o) = q;
  } else {
    store_f32<4>(reinterpret_cast<float*>(y) + o, v);
  }
}

// Output of one column vector: y (MODE 0) or the gated hidden h (MODE 1/2).
// Returns how many of its h are nonzero when the launch counts them
// (a.hcount), for the caller to add once per warp.
template <typename WT, int MODE>
__device__ __forceinline__ int epilogue(const GemvArgs& a, int tok, int col,
                                         const float (&u)[VecTraits<WT>::V],
                                         const float (&g)[VecTraits<WT>::V]) {
  constexpr int V = VecTraits<WT>::V;
  const size_t o = (size_t)tok * a.d_out + col;
  int nz = 0;
  if constexpr (MODE == 0) {
    store_y<WT>(a.y, o, u);
  } else {
    float hv[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
      if constexpr (MODE == 1) {
        const float r = fmaxf(u[e], 0.0f);           // u (up), g (gate)
        hv[e] = (r * r) * g[e];
      } else {
        const float bu = a.b_up ? a.b_up[col + e] : 0.0f;
        const float bg = a.b_gate ? a.b_gate[col + e] : 0.0f;
        hv[e] = fmaxf(g[e] + bg, 0.0f) * fmaxf(u[e] + bu, 0.0f);
      }
    }
    store_f32<V>(a.h + o, hv);
    if (a.hbits != nullptr) {                      // one token: publish which h are nonzero
      uint32_t m = 0;
#pragma unroll
      for (int e = 0; e < V; ++e) m |= (hv[e] != 0.0f ? 1u : 0u) << e;
      if (m != 0u) atomicOr(a.hbits + col / 32, m << (col % 32));
      if (a.hcount != nullptr) nz = __popc(m);
    }
  }
  return nz;
}

// One atomic per warp for the nonzero-h counter (every lane calls this).
__device__ __forceinline__ void add_hcount(int32_t* hcount, int nz) {
  if (hcount == nullptr) return;
  nz = __reduce_add_sync(0xffffffffu, nz);
  if ((threadIdx.x & 31) == 0 && nz != 0) atomicAdd(hcount, nz);
}

template <typename WT, int TT, int MODE>
__global__ void __launch_bounds__(kMaxConsumers + 32, (TT <= 4) ? 2 : 1) gemv_kernel(GemvArgs a) {
  constexpr int V = VecTraits<WT>::V;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[kMaxStages];
  __shared__ __align__(8) uint64_t s_empty[kMaxStages];
  __shared__ int s_flag;
  __shared__ int s_err;

  const GemvPlan& P = a.plan;
  const int NC = P.threads - 32;                 // consumer threads; the last warp produces
  const int tid = threadIdx.x, lane = tid & 31;
  const bool producer = tid >= NC;
  const int tile_bytes = P.vec_tile * 16;
  unsigned char* s_stage = smem;
  int* s_rows = reinterpret_cast<int*>(smem + (size_t)P.nst * P.rps * tile_bytes);
  float* s_vals = reinterpret_cast<float*>(s_rows + P.rcap);

  const int S = P.S;
  const int ct = blockIdx.x;
  const int mat = blockIdx.y / S;
  const int s = blockIdx.y - mat * S;
  const int grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const size_t row_bytes = (size_t)d_out * sizeof(WT);
  const size_t cbyte = (size_t)ct * tile_bytes;
  const int tbytes = (int)min((size_t)tile_bytes, row_bytes - cbyte);   // ragged last tile
  const int tvec = tbytes / 16;
  const unsigned char* Wb = reinterpret_cast<const unsigned char*>(a.w[mat]) + cbyte;
  const int col = (ct * P.vec_tile + tid) * V;                            // this thread's columns

  // The down projection of a one-token FFN (a.hcount): the launch before this
  // one (the top-K on h) releases this grid as soon as it starts, and its
  // completion, which the wait below waits for, follows that of the up/gate
  // projection; so h and its nonzero count are complete after the wait.  With
  // at most k_sel nonzero h the kept rows are exactly the nonzero h: this CTA
  // lists those of its own index range and streams them (the top-K's list is
  // used otherwise).  The counter is zeroed by the next call's first kernel.
  bool hrange = false;
  if (MODE == 0 && a.hcount != nullptr) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    hrange = __ldcg(a.hcount) <= a.k_sel;
  } else {
    pdl_begin();
  }
  grid_zero(a.zero, a.zero_n);
  int r0, r1;
  if (hrange) {
    r0 = (int)(((long long)d_in * s) / S);
    r1 = (int)(((long long)d_in * (s + 1)) / S);
  } else {
    const int n = min(max(*a.list_count, 0), d_in);
    r0 = (int)(((long long)n * s) / S);
    r1 = (int)(((long long)n * (s + 1)) / S);
  }

  if (tid == 0) {
    for (int i = 0; i < P.nst; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], NC / 32);
    }
    mbar_fence_init();
    s_err = 0;
  }
  __syncthreads();
  if (hrange) {
    // the nonzero h of [r0, r1) in index order (r1 - r0 <= rcap, checked on the
    // host): one ballot per warp, the warps' counts in shared memory
    __shared__ int s_wcnt[(kMaxConsumers + 32) / 32];
    const int nw = P.threads / 32;
    const int len = r1 - r0;
    int base = 0;
    for (int c0 = 0; c0 < len; c0 += P.threads) {
      const int i = c0 + tid;
      const float v = i < len ? __ldcg(a.hsrc + r0 + i) : 0.0f;
      const bool nz = v != 0.0f;
      const unsigned b = __ballot_sync(0xffffffffu, nz);
      if (lane == 0) s_wcnt[tid >> 5] = __popc(b);
      __syncthreads();
      int pre = base;
      for (int w = 0; w < (tid >> 5); ++w) pre += s_wcnt[w];
      if (nz) {
        const int pos = pre + __popc(b & lanemask_lt());
        s_rows[pos] = r0 + i;
        s_vals[pos] = v;
      }
      for (int w = 0; w < nw; ++w) base += s_wcnt[w];
      __syncthreads();
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0 && a.rows_out) *a.rows_out = __ldcg(a.hcount);
    r1 = r0 + base;                                // rows of this split's piece
  }

  float acc[TT][V];
#pragma unroll
  for (int t = 0; t < TT; ++t)
#pragma unroll
    for (int e = 0; e < V; ++e) acc[t][e] = 0.0f;

  int gst = 0;                                   // stages issued so far (slot/phase)
  for (int pb = r0; pb < r1; pb += P.rcap) {
    const int np = min(P.rcap, r1 - pb);
    for (int j = tid; j < np && !hrange; j += P.threads) {
      int r = a.list[pb + j];
      const bool ok = (unsigned)r < (unsigned)d_in;
      if (!ok) {                                 // a corrupted list is reported, never followed
        dev_fail(a.status, DEV_CHECK, 3, (uint32_t)r);
        r = 0;
      }
      s_rows[j] = r;
      if (a.list_val) {
        const float* lv = a.list_val + (size_t)(pb + j) * a.T + tok0;
#pragma unroll
        for (int t = 0; t < TT; ++t) s_vals[t * P.rcap + j] = (ok && t < ntok) ? lv[t] : 0.0f;
      } else {
#pragma unroll
        for (int t = 0; t < TT; ++t)
          s_vals[t * P.rcap + j] = (ok && t < ntok) ? a.xsf[(size_t)(tok0 + t) * d_in + r] : 0.0f;
      }
    }
    __syncthreads();
    const int nstage = (np + P.rps - 1) / P.rps;
    if (producer) {
      // the producer warp's lanes issue a stage's copies side by side (none at
      // all under the failure-detection test's no-copies injection)
      for (int st = 0; st < nstage && !a.no_copies; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        int ok = 1;
        if (lane == 0 && g >= P.nst &&
            !mbar_wait(&s_empty[slot], (uint32_t)((g / P.nst) - 1) & 1u, a.wait_limit)) {
          dev_fail(a.status, DEV_TIMEOUT, 10, (uint32_t)g);
          atomicExch(&s_err, 1);
          ok = 0;
        }
        if (__shfl_sync(0xffffffffu, ok, 0) == 0) break;
        const int j0 = st * P.rps;
        const int cnt = min(P.rps, np - j0);
        if (lane == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cnt * tbytes));
        __syncwarp();
        for (int rr = lane; rr < cnt; rr += 32)
          bulk_g2s(s_stage + ((size_t)slot * P.rps + rr) * tile_bytes,
                   Wb + (size_t)s_rows[j0 + rr] * row_bytes, (uint32_t)tbytes, &s_full[slot]);
      }
    } else {
      for (int st = 0; st < nstage; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        // once a wait of this CTA has given up, the later stages are not waited for
        const bool ready = !*(volatile int*)&s_err &&
                           mbar_wait_backoff(&s_full[slot], (uint32_t)(g / P.nst) & 1u, a.wait_limit);
        if (!ready && !*(volatile int*)&s_err) {
          if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 11, (uint32_t)g);
          atomicExch(&s_err, 1);
        }
        const int j0 = st * P.rps;
        const int cnt = min(P.rps, np - j0);
        if (ready && tid < tvec) {
          for (int r = 0; r < cnt; ++r) {
            const uint4 q = *reinterpret_cast<const uint4*>(
                s_stage + ((size_t)slot * P.rps + r) * tile_bytes + (size_t)tid * 16);
            float w[V];
            unpack<WT>(q, w);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              const float v = s_vals[t * P.rcap + j0 + r];
#pragma unroll
              for (int e = 0; e < V; ++e) acc[t][e] = fmaf(v, w[e], acc[t][e]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[slot]);
      }
    }
    gst += nstage;
    __syncthreads();                             // piece consumed before restaging
  }
  if (s_err && tid == 0 && !a.no_copies) {
    // a wait gave up: let the copies already issued land before the CTA exits
    // (with no copies issued at all there is nothing to wait for)
    for (int i = 0; i < P.nst && i < gst; ++i) {
      const int g_last = gst - 1 - i;            // the newest stage of each slot
      mbar_wait(&s_full[g_last % P.nst], (uint32_t)(g_last / P.nst) & 1u, a.wait_limit);
    }
  }

  // ---- add this split's partial sums --------------------------------------
  const bool mine = !producer && tid < tvec;
  const bool direct = (MODE == 0) && (S == 1);
  const size_t per_mat = (size_t)a.T * d_out;
  if (mine) {
    for (int t = 0; t < ntok; ++t) {
      const int tok = tok0 + t;
      if (direct) {
        store_y<WT>(a.y, (size_t)tok * d_out + col, acc[t]);
      } else {
        float* dst = a.parts + (size_t)(s % P.copies) * P.mats * per_mat + (size_t)mat * per_mat +
                     (size_t)tok * d_out + col;
#pragma unroll
        for (int q = 0; q < V / 4; ++q)
          red_add_v4(dst + 4 * q, acc[t][4 * q], acc[t][4 * q + 1], acc[t][4 * q + 2], acc[t][4 * q + 3]);
      }
    }
  }
  if (direct) return;

  // ---- the last CTA of this column tile: epilogue, then zero the sums -------
  int32_t* ticket = a.tickets + (size_t)grp * P.n_ct + ct;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = (atomicAdd(ticket, 1) == P.mats * S - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0) *ticket = 0;                     // leave the counter clean
  int nzc = 0;
  if (mine) {
    const size_t copy_stride = (size_t)P.mats * per_mat;
    for (int t = 0; t < ntok; ++t) {
      const int tok = tok0 + t;
      const float* pu = a.parts + (size_t)tok * d_out + col;
      float u[V], g[V];
#pragma unroll
      for (int e = 0; e < V; ++e) { u[e] = 0.0f; g[e] = 0.0f; }
      for (int c = 0; c < P.copies; ++c) {
#pragma unroll
        for (int q = 0; q < V / 4; ++q) {
          const float4 r = __ldcg(reinterpret_cast<const float4*>(pu + c * copy_stride) + q);
          u[4 * q] += r.x; u[4 * q + 1] += r.y; u[4 * q + 2] += r.z; u[4 * q + 3] += r.w;
        }
        if (P.mats == 2) {
#pragma unroll
          for (int q = 0; q < V / 4; ++q) {
            const float4 r = __ldcg(reinterpret_cast<const float4*>(pu + c * copy_stride + per_mat) + q);
            g[4 * q] += r.x; g[4 * q + 1] += r.y; g[4 * q + 2] += r.z; g[4 * q + 3] += r.w;
          }
        }
      }
      nzc += epilogue<WT, MODE>(a, tok, col, u, g);
    }
  }
  if constexpr (MODE != 0) add_hcount(a.hcount, nzc);
}

// ---- batched decode on the tensor cores ------------------------------------
// With 4 or 8 tokens the FMA path spends 32-64 FMAs per 16-byte weight vector
// and stops being HBM-bound.  Here the staged rows feed warp-level
// mma.sync m16n8k16 (bf16 x bf16 -> f32): A = the weight tile read as
// [16 columns x 16 rows] with ldmatrix.trans (rows sit in shared memory with
// their columns contiguous), B = the 16 rows' values for 8 token slots
// (rounded to bf16), C = 16 columns x 8 tokens in registers.  Rows are staged
// 16 per ring stage at a padded pitch (tile bytes + 16), which keeps the
// ldmatrix row addresses in distinct bank groups.  Split sums, tickets and
// the epilogue are those of gemv_kernel.
constexpr int kMmaWarps = 8;                       // consumer warps
constexpr int kMmaBPW = 12;                        // 16-column blocks per warp (max)
constexpr int kMmaRows = 16;                       // rows per stage (the MMA's K)

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int TT, int MODE, int MINB>
__global__ void __launch_bounds__(kMmaWarps * 32 + 32, MINB) gemv_mma_kernel(GemvArgs a) {
  constexpr int V = 8;
  constexpr int NC = kMmaWarps * 32;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[kMaxStages];
  __shared__ __align__(8) uint64_t s_empty[kMaxStages];
  __shared__ int s_flag;
  __shared__ int s_err;

  const GemvPlan& P = a.plan;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == kMmaWarps;
  const int pitch = P.vec_tile * 16 + 16;
  const int stage_bytes = kMmaRows * pitch;
  unsigned char* s_stage = smem;
  int* s_rows = reinterpret_cast<int*>(smem + (size_t)P.nst * stage_bytes);
  float* s_vals = reinterpret_cast<float*>(s_rows + P.rcap);

  const int S = P.S;
  const int ct = blockIdx.x;
  const int mat = blockIdx.y / S;
  const int s = blockIdx.y - mat * S;
  const int grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const size_t row_bytes = (size_t)d_out * 2;
  const size_t cbyte = (size_t)ct * P.vec_tile * 16;
  const int tbytes = (int)min((size_t)P.vec_tile * 16, row_bytes - cbyte);
  const int tvec = tbytes / 16;
  const int nblk = tbytes / 32;                    // 16-column blocks (d_out % 16 == 0)
  const unsigned char* Wb = reinterpret_cast<const unsigned char*>(a.w[mat]) + cbyte;

  pdl_begin();
  grid_zero(a.zero, a.zero_n);
  const int n = min(max(*a.list_count, 0), d_in);
  const int r0 = (int)(((long long)n * s) / S);
  const int r1 = (int)(((long long)n * (s + 1)) / S);

  if (tid == 0) {
    for (int i = 0; i < P.nst; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kMmaWarps);
    }
    mbar_fence_init();
    s_err = 0;
  }
  __syncthreads();

  float acc[kMmaBPW][4];
#pragma unroll
  for (int b = 0; b < kMmaBPW; ++b)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[b][e] = 0.0f;

  // ldmatrix row address of this lane inside a 16 x 16 block: matrices
  // (k 0-7, m 0-7), (k 0-7, m 8-15), (k 8-15, m 0-7), (k 8-15, m 8-15)
  const int q = lane >> 3;
  const uint32_t lane_off = (uint32_t)(((q >> 1) * 8 + (lane & 7)) * pitch + (q & 1) * 16);
  const uint32_t ring_addr = (uint32_t)__cvta_generic_to_shared(s_stage);
  const int bn = lane >> 2;                         // token slot of this lane's B values
  const int bk = (lane & 3) * 2;                    // first row of this lane's B values

  int gst = 0;
  for (int pb = r0; pb < r1; pb += P.rcap) {
    const int np = min(P.rcap, r1 - pb);
    for (int j = tid; j < np; j += blockDim.x) {
      int r = a.list[pb + j];
      const bool ok = (unsigned)r < (unsigned)d_in;
      if (!ok) {
        dev_fail(a.status, DEV_CHECK, 3, (uint32_t)r);
        r = 0;
      }
      s_rows[j] = r;
#pragma unroll
      for (int t = 0; t < TT; ++t)
        s_vals[t * P.rcap + j] = (ok && t < ntok)
                                     ? (a.list_val ? a.list_val[(size_t)(pb + j) * a.T + tok0 + t]
                                                   : a.xsf[(size_t)(tok0 + t) * d_in + r])
                                     : 0.0f;
    }
    __syncthreads();
    const int nstage = (np + kMmaRows - 1) / kMmaRows;
    if (producer) {
      // the producer warp's lanes issue a stage's copies side by side
      for (int st = 0; st < nstage; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        int ok = 1;
        if (lane == 0 && g >= P.nst && !mbar_wait(&s_empty[slot], (uint32_t)((g / P.nst) - 1) & 1u)) {
          dev_fail(a.status, DEV_TIMEOUT, 14, (uint32_t)g);
          atomicExch(&s_err, 1);
          ok = 0;
        }
        if (__shfl_sync(0xffffffffu, ok, 0) == 0) break;
        const int j0 = st * kMmaRows;
        const int cnt = min(kMmaRows, np - j0);
        if (lane == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cnt * tbytes));
        __syncwarp();
        for (int rr = lane; rr < cnt; rr += 32)
          bulk_g2s(s_stage + (size_t)slot * stage_bytes + (size_t)rr * pitch,
                   Wb + (size_t)s_rows[j0 + rr] * row_bytes, (uint32_t)tbytes, &s_full[slot]);
      }
    } else {
      for (int st = 0; st < nstage; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        const bool ready = mbar_wait_backoff(&s_full[slot], (uint32_t)(g / P.nst) & 1u);
        if (!ready) {
          if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 15, (uint32_t)g);
          atomicExch(&s_err, 1);
        }
        const int j0 = st * kMmaRows;
        const int cnt = min(kMmaRows, np - j0);
        unsigned char* sb = s_stage + (size_t)slot * stage_bytes;
        if (cnt < kMmaRows) {
          // rows past the list's end: zero them (a stale NaN times a zero value
          // would still poison the sum); consumer warps sync on a named barrier
          for (int i = tid; i < (kMmaRows - cnt) * tvec; i += NC) {
            const int rr = cnt + i / tvec, vv = i % tvec;
            *reinterpret_cast<uint4*>(sb + (size_t)rr * pitch + (size_t)vv * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          asm volatile("bar.sync 1, %0;" ::"r"(NC) : "memory");
        }
        if (ready) {
          // B: rows bk, bk+1 and bk+8, bk+9 of the stage for token slot bn
          float x0 = 0.f, x1 = 0.f, x8 = 0.f, x9 = 0.f;
          if (bn < TT) {
            const float* vp = s_vals + bn * P.rcap + j0;
            if (bk < cnt) x0 = vp[bk];
            if (bk + 1 < cnt) x1 = vp[bk + 1];
            if (bk + 8 < cnt) x8 = vp[bk + 8];
            if (bk + 9 < cnt) x9 = vp[bk + 9];
          }
          const uint32_t b0 = pack_bf16x2(x0, x1), b1 = pack_bf16x2(x8, x9);
          const uint32_t base = ring_addr + (uint32_t)((size_t)slot * stage_bytes) + lane_off;
#pragma unroll
          for (int b = 0; b < kMmaBPW; ++b) {
            const int blk = warp + b * kMmaWarps;
            if (blk < nblk) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4_trans(base + (uint32_t)(blk * 32), a0, a1, a2, a3);
              mma_bf16_16816(acc[b], a0, a1, a2, a3, b0, b1);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[slot]);
      }
    }
    gst += nstage;
    __syncthreads();
  }
  if (s_err && tid == 0) {
    for (int i = 0; i < P.nst && i < gst; ++i) {
      const int g_last = gst - 1 - i;
      mbar_wait(&s_full[g_last % P.nst], (uint32_t)(g_last / P.nst) & 1u);
    }
  }

  // ---- split sums --------------------------------------------------------------
  // The accumulators of this kernel are column-major, [column][Tp] (tokens
  // contiguous, Tp = T rounded up to 4), so that one lane adds 4 tokens of one
  // column with one vector reduction: lanes 2i and 2i+1 (tokens n..n+1 and
  // n+2..n+3 of columns m and m+8) swap halves, then the even lane adds
  // column m, the odd lane column m+8.  (Scalar adds per element cost ~4x the
  // reduction operations and were the bottleneck.)
  const int Tp = (a.T + 3) & ~3;
  const size_t per_mat = (size_t)d_out * Tp;
  if (!producer) {
    float* base = a.parts + (size_t)(s % P.copies) * P.mats * per_mat + (size_t)mat * per_mat;
    const int cb = (int)(cbyte / 2);
    const int tig = lane & 3;
    const bool even = (tig & 1) == 0;
    const int t = (tig & 2) * 2;                    // first of this lane's 4 tokens
#pragma unroll
    for (int b = 0; b < kMmaBPW; ++b) {
      const int blk = warp + b * kMmaWarps;
      if (blk < nblk) {                            // warp-uniform
        const float r0 = __shfl_xor_sync(0xffffffffu, even ? acc[b][2] : acc[b][0], 1);
        const float r1 = __shfl_xor_sync(0xffffffffu, even ? acc[b][3] : acc[b][1], 1);
        const int col = cb + blk * 16 + (lane >> 2) + (even ? 0 : 8);
        if (t < ntok) {
          float* dst = base + (size_t)col * Tp + tok0 + t;
          if (even) red_add_v4(dst, acc[b][0], acc[b][1], r0, r1);
          else red_add_v4(dst, r0, r1, acc[b][2], acc[b][3]);
        }
      }
    }
  }

  // ---- the last CTA of this column tile: epilogue -----------------------------
  int32_t* ticket = a.tickets + (size_t)grp * P.n_ct + ct;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = (atomicAdd(ticket, 1) == P.mats * S - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0) *ticket = 0;
  const size_t copy_stride = (size_t)P.mats * per_mat;
  // (column vector, token) pairs, tokens fastest: neighbouring threads read
  // neighbouring accumulators
  for (int i = tid; i < tvec * ntok; i += blockDim.x) {
    const int v = i / ntok, tt = i - v * ntok;
    const int col = (ct * P.vec_tile + v) * V;
    const int tok = tok0 + tt;
    const float* pu = a.parts + (size_t)col * Tp + tok;
    float u[V], gv[V];
#pragma unroll
    for (int e = 0; e < V; ++e) { u[e] = 0.0f; gv[e] = 0.0f; }
    for (int c = 0; c < P.copies; ++c) {
#pragma unroll
      for (int e = 0; e < V; ++e) u[e] += __ldcg(pu + c * copy_stride + (size_t)e * Tp);
      if (P.mats == 2) {
#pragma unroll
        for (int e = 0; e < V; ++e) gv[e] += __ldcg(pu + c * copy_stride + per_mat + (size_t)e * Tp);
      }
    }
    const int nz = epilogue<__nv_bfloat16, MODE>(a, tok, col, u, gv);
    if (a.hcount != nullptr && nz != 0) atomicAdd(a.hcount, nz);
  }
}

template <int TT, int MODE, int MINB>
cudaError_t launch_mma(const GemvArgs& a, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(gemv_mma_kernel<TT, MODE, MINB>, 200 * 1024, &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(a.plan.n_ct, a.plan.mats * a.plan.S, a.plan.groups);
  e = launch_pdl(gemv_mma_kernel<TT, MODE, MINB>, grid, dim3(kMmaWarps * 32 + 32), a.plan.smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TT, int MODE>
cudaError_t launch_mma(const GemvArgs& a, cudaStream_t s) {
  return a.plan.cta_sm == 1 ? launch_mma<TT, MODE, 1>(a, s) : launch_mma<TT, MODE, 2>(a, s);
}

template <int TT>
cudaError_t launch_mma_mode(const GemvArgs& a, cudaStream_t s) {
  switch (a.mode) {
    case 0: return launch_mma<TT, 0>(a, s);
    case 1: return launch_mma<TT, 1>(a, s);
    case 2: return launch_mma<TT, 2>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename WT, int TT, int MODE>
cudaError_t launch3(const GemvArgs& a, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(gemv_kernel<WT, TT, MODE>, 200 * 1024, &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(a.plan.n_ct, a.plan.mats * a.plan.S, a.plan.groups);
  e = launch_pdl(gemv_kernel<WT, TT, MODE>, grid, dim3(a.plan.threads), a.plan.smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename WT, int TT>
cudaError_t launch2(const GemvArgs& a, cudaStream_t s) {
  switch (a.mode) {
    case 0: return launch3<WT, TT, 0>(a, s);
    case 1: return launch3<WT, TT, 1>(a, s);
    case 2: return launch3<WT, TT, 2>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename WT>
cudaError_t launch1(const GemvArgs& a_in, cudaStream_t s) {
  GemvArgs a = a_in;
  if (g_fault.mode == QS_FAULT_GATHER_NO_COPIES) {   // failure-detection tests only
    a.no_copies = 1;
    if (g_fault.wait_polls != 0) a.wait_limit = g_fault.wait_polls;
  }
  switch (a.plan.TT) {
    case 1: return launch2<WT, 1>(a, s);
    case 2: return launch2<WT, 2>(a, s);
    case 4: return launch2<WT, 4>(a, s);
    case 8: return launch2<WT, 8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Plan of the tensor-core kernel (bf16, 4 or 8 tokens, d_out % 16 == 0).
GemvPlan plan_gemv_mma(int T, int d_out, int rows_bound, int mats) {
  GemvPlan p{};
  p.mma = 1;
  p.TT = T <= 4 ? 4 : 8;
  p.groups = (T + p.TT - 1) / p.TT;
  p.mats = mats;
  const int blocks = d_out / 16;
  const int max_blk = kMmaWarps * kMmaBPW;
  int nct = (blocks + max_blk - 1) / max_blk;
  for (int c = nct; c <= nct + 8 && c <= blocks; ++c)   // prefer equal tiles
    if (blocks % c == 0) { nct = c; break; }
  const int blk_tile = (blocks + nct - 1) / nct;
  p.n_ct = (blocks + blk_tile - 1) / blk_tile;
  p.vec_tile = blk_tile * 2;
  p.threads = kMmaWarps * 32 + 32;
  p.rps = kMmaRows;
  const long stage = (long)kMmaRows * (p.vec_tile * 16 + 16);
  // Stages of 40 KB or more (tiles of ~2.5 KB) fit only two to a CTA at two
  // CTAs per SM, and a consumed stage leaves one in flight; one CTA per SM
  // with four stages keeps three in flight (8 tokens of 4096 -> 2 x 11008:
  // 51 -> 45 us).  Smaller stages stay at two CTAs per SM, which measured
  // faster for them (4 tokens of 4096 -> 2 x 14336 with 2 KB tiles: 52 us
  // against 62 us at one CTA per SM).
  p.cta_sm = stage >= 40L * 1024 ? 1 : 2;
  long nst = (p.cta_sm == 1 ? 180L * 1024 : 90L * 1024) / stage;
  if (nst < 2) nst = 2;
  if (nst > 4) nst = 4;
  p.nst = (int)nst;
  p.rcap = 512;
  p.smem = (size_t)p.nst * stage + (size_t)p.rcap * 4 * (1 + p.TT);
  const long slots = (long)kNumSMs * p.cta_sm;
  const long units = (long)p.n_ct * mats * p.groups;
  long S = slots / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  const long max_by_rows = rows_bound / 32;      // >= two stages per split
  if (S > max_by_rows) S = max_by_rows > 0 ? max_by_rows : 1;
  if (S > 256) S = 256;
  p.S = (int)S;
  p.copies = (int)(S / 32);
  if (p.copies < 1) p.copies = 1;
  if (p.copies > 4) p.copies = 4;
  p.parts_elems = (size_t)p.copies * mats * d_out * (size_t)((T + 3) & ~3);   // [column][T up to 4]
  p.tickets = p.groups * p.n_ct;
  return p;
}

GemvPlan plan_gemv(int T, int d_out, int rows_bound, int mats, int elem_bytes) {
  if (elem_bytes == 2 && T >= 3 && d_out % 16 == 0 && d_out >= 16)
    return plan_gemv_mma(T, d_out, rows_bound, mats);
  GemvPlan p{};
  p.TT = (T <= 1) ? 1 : (T == 2 ? 2 : (T <= 4 ? 4 : 8));
  p.groups = (T + p.TT - 1) / p.TT;
  p.mats = mats;
  const int vec_row = (int)(((long)d_out * elem_bytes) / 16);
  int nct = (vec_row + kMaxConsumers - 1) / kMaxConsumers;
  for (int c = nct; c <= nct + 8 && c <= vec_row; ++c)    // prefer equal tiles
    if (vec_row % c == 0) { nct = c; break; }
  p.n_ct = nct;
  p.vec_tile = (vec_row + nct - 1) / nct;
  p.threads = ((p.vec_tile + 31) / 32) * 32 + 32;
  const int tile_bytes = p.vec_tile * 16;
  // Stages of ~16 KB in a ring of ~90 KB (two CTAs per SM): measured best on
  // the 2867 x 22 KB gather (a stage handshake per 5.5 KB row costs ~40%).
  p.rps = (16384 + tile_bytes / 2) / tile_bytes;
  if (p.rps < 1) p.rps = 1;
  if (p.rps > 8) p.rps = 8;
  const int per_sm = (p.TT <= 4) ? 2 : 1;
  const long ring_budget = per_sm == 2 ? 90 * 1024 : 176 * 1024;
  long nst = ring_budget / ((long)p.rps * tile_bytes);
  if (nst < 3) nst = 3;
  if (nst > kMaxStages) nst = kMaxStages;
  p.nst = (int)nst;
  p.rcap = (p.TT == 8) ? 512 : 1024;
  p.smem = (size_t)p.nst * p.rps * tile_bytes + (size_t)p.rcap * 4 * (1 + p.TT);
  const long slots = (long)kNumSMs * per_sm;
  const long units = (long)nct * mats * p.groups;
  long S = slots / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  const long max_by_rows = rows_bound / 16;      // keep >= ~16 rows per split
  if (S > max_by_rows) S = max_by_rows > 0 ? max_by_rows : 1;
  if (S > 256) S = 256;
  p.S = (int)S;
  // The L2 applies reductions to one address one after another; with ~150
  // splits per address the sums land late.  Heavily split launches add into
  // up to 4 accumulator copies (~37 per address), which the epilogue sums:
  // measured 0.5 us faster on the down projection of the Llama-7B FFN, while
  // more copies cost more in the epilogue than they save.
  p.copies = (int)(S / 32);
  if (p.copies < 1) p.copies = 1;
  if (p.copies > 4) p.copies = 4;
  p.parts_elems = (size_t)p.copies * mats * T * d_out;   // zeroed by the previous kernel
  p.tickets = p.groups * nct;
  return p;
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.d_out <= 0) return cudaSuccess;
  if (a.plan.mma) {
    if (!a.bf16) return cudaErrorInvalidValue;
    switch (a.plan.TT) {
      case 4: return launch_mma_mode<4>(a, s);
      case 8: return launch_mma_mode<8>(a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  return a.bf16 ? launch1<__nv_bfloat16>(a, s) : launch1<float>(a, s);
}

}  // namespace qs
