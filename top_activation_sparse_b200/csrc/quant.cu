// BitNet b1.58 + Q-Sparse: int8 activations x ternary weights.
//
// Source: Q-Sparse news article (zxwl-tech.com), Top-K section, paragraphs on
// quantized models: the input is quantized before top-K (an epsilon keeps a
// denominator away from zero) and 1-bit weights are scaled by alpha, the mean
// absolute value of W.  The formulas were lost from the page; this library
// reads them as (float32 IEEE steps, in this order, no contraction):
//   gamma_t = amax_t + eps, s_t = 127 / gamma_t, q = clamp(rint(x * s_t), +-127)
//   alpha   = float(sum |W| (fp64) / N),  t = clamp(rint(W / (alpha + eps)), +-1)
//   acc     = sum_{kept i} q_i * t_ij  (exact int32),
//   y       = float(acc) * ((alpha * gamma_t) / 127).
//
// Packed weights: W^T input-major, word [i, j/16] holds t[j, i] at bits
// 2*(j%16) with code 00 = 0, 01 = +1, 10 = -1, so a kept input's ternary row
// is d_out/4 contiguous bytes.  The gather kernel streams only kept rows,
// decodes the 2-bit codes in registers and accumulates in int32; integer sums
// do not depend on the order of the additions, so the result is exact and
// identical however the rows are split.
#include "qs_internal.cuh"

namespace qs {
namespace {

// ---- int8 x ternary gather-GEMV ----------------------------------------------
// Packed rows are streamed like the bf16 gather-GEMV: the producer warp
// issues a cp.async.bulk per kept row (a column tile of it) into a ring of
// ~16 KB shared-memory stages.
//
// Decoding.  Each code c (00 = 0, 01 = +1, 10 = -1) is first mapped to
// u = t + 1 in {0, 1, 2} with four logic operations per word.  Codes j and j+8
// of a word then sit 16 bits apart, so one (shift, and) pulls out the pair as
// two 16-bit lanes and one integer multiply-add accumulates q * u for both:
// two outputs per IMAD.  A lane holds sum q*u with |q| <= 127 and u <= 2, so it
// stays inside int16 for up to 128 rows; every <= 128 rows the lanes are
// unpacked into int32 accumulators and the sum of q over those rows is taken
// off (sum q*t = sum q*u - sum q).  Everything is integer: the result is exact
// and independent of the order of the additions.
//
// Split partials are added with f32 vector reductions: every partial is an
// integer with |value| <= 127 * d_in < 2^24, so the f32 additions are exact and
// the result does not depend on their order.

// One token: 8 lane pairs (one packed word of a row) per thread, so a 3 KB
// tile has ~170 consumer threads; with 32 lane pairs per thread (4 words) the
// tile had 2 consumer warps per CTA, 4 per SM, and the decode of a split's rows
// ran as one dependent chain per scheduler (4096 -> 11008: 18.8 -> 15.1 us).
template <int TT> struct QTune {
  static constexpr int LPT = (TT == 1) ? 8 : (TT == 2 ? 16 : (TT == 4 ? 8 : 4));  // lane pairs per thread
  static constexpr int WPT = LPT >= 8 ? LPT / 8 : 1;   // packed words a thread reads per row
  static constexpr int KPW = LPT >= 8 ? 8 : LPT;       // lane pairs a thread takes from each word
  static constexpr int kMaxConsumers = 192;            // two CTAs per SM
};
constexpr int kLaneRows = 128;                           // rows between lane flushes

__device__ __forceinline__ void red_add_v4_f32(float* dst, float a0, float a1, float a2, float a3) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a0), "f"(a1),
               "f"(a2), "f"(a3)
               : "memory");
}

// The quantized FFN's gating of 4 columns (y is the gate projection g of
// columns col.., u the up projection), see quant_gate_value.
__device__ __forceinline__ float4 quant_gating(const QGemvArgs& a, size_t o, int col, float4 gv) {
  const float4 uv = __ldcg(reinterpret_cast<const float4*>(a.gate_u + o));
  const float us[4] = {uv.x, uv.y, uv.z, uv.w};
  const float gs[4] = {gv.x, gv.y, gv.z, gv.w};
  float hs[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float bu = (a.gating == 2 && a.b_up) ? a.b_up[col + e] : 0.0f;
    const float bg = (a.gating == 2 && a.b_gate) ? a.b_gate[col + e] : 0.0f;
    hs[e] = quant_gate_value(a.gating, us[e], gs[e], bu, bg);
  }
  return make_float4(hs[0], hs[1], hs[2], hs[3]);
}

// codes (00 = 0, 01 = +1, 10 = -1) -> u = t + 1 (00, 01, 10 for -1, 0, +1)
__device__ __forceinline__ uint32_t ternary_to_u(uint32_t w) {
  const uint32_t hi = (w << 1) & 0xAAAAAAAAu;              // +1 -> bit 1 of the field
  const uint32_t zero = ~(w | (w >> 1)) & 0x55555555u;     // 0 -> bit 0 of the field
  return hi | zero;
}

template <int TT>
__global__ void __launch_bounds__(QTune<TT>::kMaxConsumers + 32, 2) qgemv_kernel(QGemvArgs a) {
  using Q = QTune<TT>;
  constexpr int WPT = Q::WPT, KPW = Q::KPW, LPT = Q::LPT;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[32];
  __shared__ __align__(8) uint64_t s_empty[32];
  __shared__ int s_flag;
  __shared__ int s_err;

  const GemvPlan& P = a.plan;
  const int NC = P.threads - 32;
  const int tid = threadIdx.x, lane = tid & 31;
  const bool producer = tid >= NC;
  const int tile_bytes = P.vec_tile * 4;               // vec_tile = packed words per tile
  unsigned char* s_stage = smem;
  int* s_rows = reinterpret_cast<int*>(smem + (size_t)P.nst * P.rps * tile_bytes);
  int8_t* s_q = reinterpret_cast<int8_t*>(s_rows + P.rcap);   // [rcap][TT]

  const int S = P.S;
  const int ct = blockIdx.x;
  const int s = blockIdx.y;
  const int grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const int row_words = d_out / 16;
  const int cword = ct * P.vec_tile;
  const int twords = min(P.vec_tile, row_words - cword);
  const int tbytes = twords * 4;
  const unsigned char* Wb = reinterpret_cast<const unsigned char*>(a.wp) + (size_t)cword * 4;
  const int lp0 = tid * LPT;                             // this thread's first lane pair of the tile
  const int w0 = lp0 >> 3;                               // its first word
  const int k0 = lp0 & 7;                                // its first pair inside that word

  pdl_begin();
  grid_zero(a.zero, a.zero_n);
  const int n = min(max(*a.list_count, 0), d_in);
  const int r0 = (int)(((long long)n * s) / S);
  const int r1 = (int)(((long long)n * (s + 1)) / S);

  if (tid == 0) {
    for (int i = 0; i < P.nst; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], NC / 32);
    }
    mbar_fence_init();
    s_err = 0;
  }
  __syncthreads();

  uint32_t pk[TT][WPT * KPW];      // two 16-bit lanes: outputs (k, k + 8) of a word
  int acc[TT][WPT * KPW * 2];      // int32: [i][kk][lo, hi]
  int qwin[TT];                    // sum of q over the rows since the last flush
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    qwin[t] = 0;
#pragma unroll
    for (int c = 0; c < WPT * KPW; ++c) pk[t][c] = 0u;
#pragma unroll
    for (int c = 0; c < WPT * KPW * 2; ++c) acc[t][c] = 0;
  }
  auto flush = [&]() {
#pragma unroll
    for (int t = 0; t < TT; ++t) {
#pragma unroll
      for (int c = 0; c < WPT * KPW; ++c) {
        const uint32_t v = pk[t][c];
        const int lo = (int)(int16_t)(uint16_t)(v & 0xFFFFu);   // signed low lane
        const int hi = (int)(v - (uint32_t)lo) >> 16;           // signed high lane
        acc[t][2 * c] += lo - qwin[t];
        acc[t][2 * c + 1] += hi - qwin[t];
        pk[t][c] = 0u;
      }
      qwin[t] = 0;
    }
  };
  int since = 0;                                         // rows in the lanes

  int gst = 0;
  for (int pb = r0; pb < r1; pb += P.rcap) {
    const int np = min(P.rcap, r1 - pb);
    for (int j = tid; j < np; j += P.threads) {
      int r = a.list[pb + j];
      const bool ok = (unsigned)r < (unsigned)d_in;
      if (!ok) {
        dev_fail(a.status, DEV_CHECK, 4, (uint32_t)r);
        r = 0;
      }
      s_rows[j] = r;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        int8_t qv = 0;
        if (ok && t < ntok)
          qv = a.list_q ? a.list_q[(size_t)(pb + j) * a.T + tok0 + t]
                        : a.xq[(size_t)(tok0 + t) * d_in + r];
        s_q[j * TT + t] = qv;
      }
    }
    __syncthreads();
    const int nstage = (np + P.rps - 1) / P.rps;
    if (producer) {
      // the producer warp's lanes issue a stage's copies side by side
      for (int st = 0; st < nstage; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        int ok = 1;
        if (lane == 0 && g >= P.nst && !mbar_wait(&s_empty[slot], (uint32_t)((g / P.nst) - 1) & 1u)) {
          dev_fail(a.status, DEV_TIMEOUT, 12, (uint32_t)g);
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
                   Wb + (size_t)s_rows[j0 + rr] * row_words * 4, (uint32_t)tbytes, &s_full[slot]);
      }
    } else {
      for (int st = 0; st < nstage; ++st) {
        const int g = gst + st;
        const int slot = g % P.nst;
        const bool ready = mbar_wait_backoff(&s_full[slot], (uint32_t)(g / P.nst) & 1u);
        if (!ready) {
          if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 13, (uint32_t)g);
          atomicExch(&s_err, 1);
        }
        const int j0 = st * P.rps;
        const int cnt = min(P.rps, np - j0);
        if (ready && w0 < twords) {
          for (int r = 0; r < cnt; ++r) {
            const uint32_t* rw =
                reinterpret_cast<const uint32_t*>(s_stage + ((size_t)slot * P.rps + r) * tile_bytes) + w0;
            int qv[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              qv[t] = s_q[(j0 + r) * TT + t];
              qwin[t] += qv[t];
            }
#pragma unroll
            for (int i = 0; i < WPT; ++i) {
              const uint32_t u = ternary_to_u((w0 + i < twords) ? rw[i] : 0u) >> (2 * k0);
#pragma unroll
              for (int kk = 0; kk < KPW; ++kk) {
                const uint32_t pair = (u >> (2 * kk)) & 0x00030003u;
#pragma unroll
                for (int t = 0; t < TT; ++t) pk[t][i * KPW + kk] += (uint32_t)qv[t] * pair;
              }
            }
          }
          since += cnt;
          if (since + P.rps > kLaneRows) {
            flush();
            since = 0;
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

  // ---- add this split's (integer) partials, exactly, as f32 --------------------
  // lane pair (i, kk) holds output columns 16 (w0 + i) + k0 + kk and that + 8
  const bool mine = !producer && w0 < twords;
  if (mine) {
    flush();
    for (int t = 0; t < ntok; ++t) {
      float* dst = a.parts + (size_t)(s % P.copies) * a.T * d_out + (size_t)(tok0 + t) * d_out +
                   (size_t)(cword + w0) * 16 + k0;
#pragma unroll
      for (int i = 0; i < WPT; ++i) {
        if (w0 + i >= twords) break;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < KPW; kk += 4)
            red_add_v4_f32(dst + i * 16 + h * 8 + kk, (float)acc[t][(i * KPW + kk) * 2 + h],
                           (float)acc[t][(i * KPW + kk + 1) * 2 + h],
                           (float)acc[t][(i * KPW + kk + 2) * 2 + h],
                           (float)acc[t][(i * KPW + kk + 3) * 2 + h]);
      }
    }
  }

  // ---- last CTA of this column tile: rescale ----------------------------------
  int32_t* ticket = a.tickets + grp * P.n_ct + ct;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = (atomicAdd(ticket, 1) == S - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0) *ticket = 0;
  if (mine) {
    for (int t = 0; t < ntok; ++t) {
      const int tok = tok0 + t;
      const float r = __fdiv_rn(__fmul_rn(a.alpha, a.gamma[tok]), 127.0f);
      const size_t o = (size_t)tok * d_out + (size_t)(cword + w0) * 16 + k0;
      float4 v[WPT][2][KPW / 4];
#pragma unroll
      for (int i = 0; i < WPT; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < KPW; kk += 4) v[i][h][kk / 4] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < P.copies; ++c) {
        const float* pc = a.parts + (size_t)c * a.T * d_out + o;
#pragma unroll
        for (int i = 0; i < WPT; ++i) {
          if (w0 + i >= twords) break;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < KPW; kk += 4) {
              const float4 f = __ldcg(reinterpret_cast<const float4*>(pc + i * 16 + h * 8 + kk));
              float4& acc4 = v[i][h][kk / 4];
              acc4.x += f.x; acc4.y += f.y; acc4.z += f.z; acc4.w += f.w;
            }
        }
      }
#pragma unroll
      for (int i = 0; i < WPT; ++i) {
        if (w0 + i >= twords) break;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < KPW; kk += 4) {
            const float4 f = v[i][h][kk / 4];
            const int4 iv = make_int4(__float2int_rn(f.x), __float2int_rn(f.y), __float2int_rn(f.z),
                                      __float2int_rn(f.w));
            const size_t e = o + i * 16 + h * 8 + kk;
            float4 yv = make_float4(__fmul_rn(__int2float_rn(iv.x), r), __fmul_rn(__int2float_rn(iv.y), r),
                                    __fmul_rn(__int2float_rn(iv.z), r), __fmul_rn(__int2float_rn(iv.w), r));
            if (a.gating) yv = quant_gating(a, e, (int)(e - (size_t)tok * d_out), yv);
            reinterpret_cast<float4*>(a.y + e)[0] = yv;
            if (a.acc) reinterpret_cast<int4*>(a.acc + e)[0] = iv;
          }
      }
    }
  }
}

// ---- 8 to 32 tokens: int8 x ternary on the tensor cores ------------------------
// The lane-pair decode spends about one instruction per multiply-add, so with
// many tokens the kernel is integer-issue bound.  Here warp-level
// mma.sync m16n8k32 (s8 x s8 -> s32) does the multiply-adds: A = 16 output
// columns x 32 kept rows of ternary weights, decoded by each lane straight
// from the packed words into its fragment (a shift and mask per row, two byte
// permutes, 0/1/2 -> 0/+1/-1 per byte); B = the 32 rows' int8 codes of 8
// tokens, read as 32-bit groups from a token-major copy in shared memory.
// Integer throughout: exact, and the split sums stay exact in f32.
constexpr int kQmWarps = 8;
constexpr int kQmRows = 32;                        // rows per stage (the MMA's K)

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// codes of 4 rows (packed words w0..w3, already shifted so that column m sits
// in bits 0-1 and column m+8 in bits 16-17) -> int8 weights of column m (lo)
// and of column m+8 (hi), row i in byte i
__device__ __forceinline__ void decode4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                        uint32_t& lo, uint32_t& hi) {
  const uint32_t p01 = (w0 & 0x00030003u) | ((w1 & 0x00030003u) << 8);
  const uint32_t p23 = (w2 & 0x00030003u) | ((w3 & 0x00030003u) << 8);
  const uint32_t clo = __byte_perm(p01, p23, 0x5410);
  const uint32_t chi = __byte_perm(p01, p23, 0x7632);
  // byte code 0 -> 0, 1 -> +1, 2 -> -1 (0xFF)
  lo = clo | (((clo >> 1) & 0x01010101u) * 0xFFu);
  hi = chi | (((chi >> 1) & 0x01010101u) * 0xFFu);
}

template <int NB>
__global__ void __launch_bounds__(kQmWarps * 32 + 32, 2) qgemv_mma_kernel(QGemvArgs a) {
  constexpr int TT = NB * 8;
  constexpr int BPW = 12 / NB;                     // 16-column blocks (packed words) per warp
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[32];
  __shared__ __align__(8) uint64_t s_empty[32];
  __shared__ int s_flag;
  __shared__ int s_err;

  const GemvPlan& P = a.plan;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == kQmWarps;
  const int pitch = P.vec_tile * 4 + 16;           // bytes per staged row (tile + pad)
  const int stage_bytes = kQmRows * pitch;
  unsigned char* s_stage = smem;
  int* s_rows = reinterpret_cast<int*>(smem + (size_t)P.nst * stage_bytes);
  int8_t* s_qT = reinterpret_cast<int8_t*>(s_rows + P.rcap);   // [TT][rcap], token-major

  const int S = P.S;
  const int ct = blockIdx.x;
  const int s = blockIdx.y;
  const int grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const int row_words = d_out / 16;
  const int cword = ct * P.vec_tile;
  const int twords = min(P.vec_tile, row_words - cword);
  const int tbytes = twords * 4;
  const unsigned char* Wb = reinterpret_cast<const unsigned char*>(a.wp) + (size_t)cword * 4;

  pdl_begin();
  grid_zero(a.zero, a.zero_n);
  const int n = min(max(*a.list_count, 0), d_in);
  const int r0 = (int)(((long long)n * s) / S);
  const int r1 = (int)(((long long)n * (s + 1)) / S);

  if (tid == 0) {
    for (int i = 0; i < P.nst; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], kQmWarps);
    }
    mbar_fence_init();
    s_err = 0;
  }
  __syncthreads();

  int acc[BPW][NB][4];
#pragma unroll
  for (int b = 0; b < BPW; ++b)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[b][nb][e] = 0;

  const int g = lane >> 2;                          // A row (column m) / B column (token)
  const int k0 = (lane & 3) * 4;                    // first of this lane's 4 rows
  const int shift = 2 * g;                          // column g of a packed word

  int gst = 0;
  for (int pb = r0; pb < r1; pb += P.rcap) {
    const int np = min(P.rcap, r1 - pb);
    for (int j = tid; j < np; j += blockDim.x) {
      int r = a.list[pb + j];
      const bool ok = (unsigned)r < (unsigned)d_in;
      if (!ok) {
        dev_fail(a.status, DEV_CHECK, 4, (uint32_t)r);
        r = 0;
      }
      s_rows[j] = r;
#pragma unroll
      for (int t = 0; t < TT; ++t)
        s_qT[t * P.rcap + j] = (ok && t < ntok) ? a.xq[(size_t)(tok0 + t) * d_in + r] : (int8_t)0;
    }
    __syncthreads();
    const int nstage = (np + kQmRows - 1) / kQmRows;
    if (producer) {
      // the row segments are short (tens to hundreds of bytes): the warp's 32
      // lanes issue a stage's 32 copies side by side
      for (int st = 0; st < nstage; ++st) {
        const int gg = gst + st;
        const int slot = gg % P.nst;
        int ok = 1;
        if (lane == 0 && gg >= P.nst && !mbar_wait(&s_empty[slot], (uint32_t)((gg / P.nst) - 1) & 1u)) {
          dev_fail(a.status, DEV_TIMEOUT, 16, (uint32_t)gg);
          atomicExch(&s_err, 1);
          ok = 0;
        }
        if (__shfl_sync(0xffffffffu, ok, 0) == 0) break;
        const int j0 = st * kQmRows;
        const int cnt = min(kQmRows, np - j0);
        if (lane == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cnt * tbytes));
        __syncwarp();
        if (lane < cnt)
          bulk_g2s(s_stage + (size_t)slot * stage_bytes + (size_t)lane * pitch,
                   Wb + (size_t)s_rows[j0 + lane] * row_words * 4, (uint32_t)tbytes, &s_full[slot]);
      }
    } else {
      for (int st = 0; st < nstage; ++st) {
        const int gg = gst + st;
        const int slot = gg % P.nst;
        const bool ready = mbar_wait_backoff(&s_full[slot], (uint32_t)(gg / P.nst) & 1u);
        if (!ready) {
          if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 17, (uint32_t)gg);
          atomicExch(&s_err, 1);
        }
        const int j0 = st * kQmRows;
        const int cnt = min(kQmRows, np - j0);
        if (ready) {
          // B: rows k0..k0+3 and k0+16..k0+19 of token nb*8 + g; rows past the
          // stage's end contribute 0 (their staged weights are stale)
          const int v0 = min(max(cnt - k0, 0), 4), v1 = min(max(cnt - k0 - 16, 0), 4);
          const uint32_t m0 = v0 >= 4 ? 0xffffffffu : ((1u << (8 * v0)) - 1u);
          const uint32_t m1 = v1 >= 4 ? 0xffffffffu : ((1u << (8 * v1)) - 1u);
          uint32_t b0[NB], b1[NB];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int8_t* qp = s_qT + (nb * 8 + g) * P.rcap + j0 + k0;
            b0[nb] = *reinterpret_cast<const uint32_t*>(qp) & m0;
            b1[nb] = *reinterpret_cast<const uint32_t*>(qp + 16) & m1;
          }
          const unsigned char* sb = s_stage + (size_t)slot * stage_bytes;
#pragma unroll
          for (int b = 0; b < BPW; ++b) {
            const int blk = warp + b * kQmWarps;
            if (blk < twords) {
              const unsigned char* wp = sb + (size_t)k0 * pitch + (size_t)blk * 4;
              const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wp) >> shift;
              const uint32_t w1 = *reinterpret_cast<const uint32_t*>(wp + pitch) >> shift;
              const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wp + 2 * pitch) >> shift;
              const uint32_t w3 = *reinterpret_cast<const uint32_t*>(wp + 3 * pitch) >> shift;
              const unsigned char* wq = wp + (size_t)16 * pitch;
              const uint32_t x0 = *reinterpret_cast<const uint32_t*>(wq) >> shift;
              const uint32_t x1 = *reinterpret_cast<const uint32_t*>(wq + pitch) >> shift;
              const uint32_t x2 = *reinterpret_cast<const uint32_t*>(wq + 2 * pitch) >> shift;
              const uint32_t x3 = *reinterpret_cast<const uint32_t*>(wq + 3 * pitch) >> shift;
              uint32_t a0, a1, a2, a3;
              decode4(w0, w1, w2, w3, a0, a1);
              decode4(x0, x1, x2, x3, a2, a3);
#pragma unroll
              for (int nb = 0; nb < NB; ++nb) mma_s8_16832(acc[b][nb], a0, a1, a2, a3, b0[nb], b1[nb]);
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

  // ---- split sums (exact integers in f32) ----------------------------------------
  // Column-major accumulators [column][Tp] (Tp = T rounded up to 4): lanes 2i
  // and 2i+1 swap halves so that each adds 4 tokens of one column with one
  // vector reduction (see the bf16 tensor-core gather-GEMV).
  const int Tp = (a.T + 3) & ~3;
  if (!producer) {
    float* base = a.parts + (size_t)(s % P.copies) * d_out * Tp;
    const int tig = lane & 3;
    const bool even = (tig & 1) == 0;
    const int tq = (tig & 2) * 2;
#pragma unroll
    for (int b = 0; b < BPW; ++b) {
      const int blk = warp + b * kQmWarps;
      if (blk < twords) {                          // warp-uniform
        const int col = (cword + blk) * 16 + g + (even ? 0 : 8);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const float c0 = (float)acc[b][nb][0], c1 = (float)acc[b][nb][1];
          const float c2 = (float)acc[b][nb][2], c3 = (float)acc[b][nb][3];
          const float r0 = __shfl_xor_sync(0xffffffffu, even ? c2 : c0, 1);
          const float r1 = __shfl_xor_sync(0xffffffffu, even ? c3 : c1, 1);
          const int t = nb * 8 + tq;
          if (t < ntok) {
            float* dst = base + (size_t)col * Tp + tok0 + t;
            if (even) red_add_v4_f32(dst, c0, c1, r0, r1);
            else red_add_v4_f32(dst, r0, r1, c2, c3);
          }
        }
      }
    }
  }

  // ---- last CTA of this column tile: rescale -----------------------------------
  int32_t* ticket = a.tickets + grp * P.n_ct + ct;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = (atomicAdd(ticket, 1) == S - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();
  if (tid == 0) *ticket = 0;
  // (column, 4 tokens) pairs with four float4 loads in flight per thread:
  // the tokens of a column are contiguous in the split sums (one copy here)
  __shared__ float s_r[TT];
  for (int t = tid; t < ntok; t += blockDim.x)
    s_r[t] = __fdiv_rn(__fmul_rn(a.alpha, a.gamma[tok0 + t]), 127.0f);
  __syncthreads();
  const int ncols = twords * 16;
  const int G = (ntok + 3) / 4;
  const int total = ncols * G;
  for (int i0 = tid; i0 < total; i0 += 4 * (int)blockDim.x) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < total) {
        const int g = i / ncols, cc = i - g * ncols;
        for (int c = 0; c < P.copies; ++c) {
          const float4 f = __ldcg(reinterpret_cast<const float4*>(
              a.parts + (size_t)c * d_out * Tp + (size_t)(cword * 16 + cc) * Tp + tok0) + g);
          v[u].x += f.x; v[u].y += f.y; v[u].z += f.z; v[u].w += f.w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      if (i >= total) break;
      const int g = i / ncols, cc = i - g * ncols;
      const int col = cword * 16 + cc;
      const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 4 * g + e;
        if (t >= ntok) break;
        const int iv = __float2int_rn(vv[e]);
        const size_t o = (size_t)(tok0 + t) * d_out + col;
        float yv = __fmul_rn(__int2float_rn(iv), s_r[t]);
        if (a.gating) {                            // the quantized FFN's gate projection
          const float bu = (a.gating == 2 && a.b_up) ? a.b_up[col] : 0.0f;
          const float bg = (a.gating == 2 && a.b_gate) ? a.b_gate[col] : 0.0f;
          yv = quant_gate_value(a.gating, __ldcg(a.gate_u + o), yv, bu, bg);
        }
        a.y[o] = yv;
        if (a.acc) a.acc[o] = iv;
      }
    }
  }
}

template <int NB>
cudaError_t qlaunch_mma(const QGemvArgs& a, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(qgemv_mma_kernel<NB>, 200 * 1024, &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(a.plan.n_ct, a.plan.S, a.plan.groups);
  e = launch_pdl(qgemv_mma_kernel<NB>, grid, dim3(kQmWarps * 32 + 32), a.plan.smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int TT>
cudaError_t qlaunch(const QGemvArgs& a, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(qgemv_kernel<TT>, 200 * 1024, &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(a.plan.n_ct, a.plan.S, a.plan.groups);
  e = launch_pdl(qgemv_kernel<TT>, grid, dim3(a.plan.threads), a.plan.smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---- ternary quantizer ------------------------------------------------------

constexpr int kPackNT = 256;

__global__ void __launch_bounds__(kPackNT) abs_sum_kernel(PackArgs a) {
  __shared__ double s_w[kPackNT / 32];
  __shared__ int s_last;
  const size_t N = (size_t)a.d_out * (size_t)a.d_in;
  const size_t stride = (size_t)gridDim.x * kPackNT;
  double acc = 0.0;
  for (size_t i = (size_t)blockIdx.x * kPackNT + threadIdx.x; i < N; i += stride)
    acc += fabs((double)__ldg(a.w + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_w[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = 0.0;
    for (int w = 0; w < kPackNT / 32; ++w) b += s_w[w];
    a.alpha_parts[blockIdx.x] = b;
    __threadfence();
    s_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last || threadIdx.x != 0) return;
  __threadfence();
  double tot = 0.0;
  for (int b = 0; b < (int)gridDim.x; ++b) tot += __ldcg(a.alpha_parts + b);
  const float alpha = (float)(tot / (double)N);
  *a.alpha_ws = alpha;
  if (a.alpha_out) *a.alpha_out = alpha;
  *a.ticket = 0;
}

__global__ void __launch_bounds__(kPackNT) pack_kernel(PackArgs a) {
  const int n_words = a.d_out / 16;
  const size_t total = (size_t)n_words * a.d_in;
  const size_t g = (size_t)blockIdx.x * kPackNT + threadIdx.x;
  if (g >= total) return;
  const int i = (int)(g % a.d_in);        // input feature (consecutive threads: coalesced reads)
  const int c = (int)(g / a.d_in);        // output word
  const float denom = __fadd_rn(__ldcg(a.alpha_ws), a.eps);
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float w = __ldg(a.w + (size_t)(c * 16 + j) * a.d_in + i);
    int t = __float2int_rn(__fdiv_rn(w, denom));
    t = min(1, max(-1, t));
    const uint32_t code = (t == 1) ? 1u : (t == -1 ? 2u : 0u);
    word |= code << (2 * j);
  }
  a.packed[(size_t)i * n_words + c] = word;
}

}  // namespace

// Plan of the tensor-core kernel: 8-32 tokens per group (n-blocks of 8).
GemvPlan plan_qgemv_mma(int T, int d_out, int rows_bound) {
  GemvPlan p{};
  p.mma = 1;
  p.TT = T >= 32 ? 32 : ((T + 7) / 8) * 8;
  p.groups = (T + p.TT - 1) / p.TT;
  p.mats = 1;
  const int nb = p.TT / 8;
  const int row_words = d_out / 16;
  const int max_words = kQmWarps * (12 / nb);      // 96, 48, 32, 24: multiples of 4
  int nct = (row_words + max_words - 1) / max_words;
  if (nct < 1) nct = 1;
  int tile = ((row_words + nct - 1) / nct + 3) / 4 * 4;
  if (tile > max_words) tile = max_words;
  p.n_ct = (row_words + tile - 1) / tile;
  p.vec_tile = tile;                               // packed words per tile
  p.threads = kQmWarps * 32 + 32;
  p.rps = kQmRows;
  const long stage = (long)kQmRows * (tile * 4 + 16);
  long nst = (90L * 1024) / stage;
  if (nst < 2) nst = 2;
  if (nst > 16) nst = 16;
  p.nst = (int)nst;
  p.rcap = 512;
  p.smem = (size_t)p.nst * stage + (size_t)p.rcap * (4 + p.TT);
  const long slots = (long)kNumSMs * 2;
  const long units = (long)p.n_ct * p.groups;
  long S = slots / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  const long max_by_rows = rows_bound / kQmRows;
  if (S > max_by_rows) S = max_by_rows > 0 ? max_by_rows : 1;
  if (S > 256) S = 256;
  p.S = (int)S;
  p.copies = 1;
  p.parts_elems = (size_t)d_out * (size_t)((T + 3) & ~3);   // [column][T up to 4]
  p.tickets = p.groups * p.n_ct;
  return p;
}

GemvPlan plan_qgemv(int T, int d_out, int rows_bound) {
  if (T >= 8) return plan_qgemv_mma(T, d_out, rows_bound);
  GemvPlan p{};
  p.TT = (T <= 1) ? 1 : (T == 2 ? 2 : (T <= 4 ? 4 : 8));
  p.groups = (T + p.TT - 1) / p.TT;
  p.mats = 1;
  const int lpt = (p.TT == 1) ? 8 : (p.TT == 2 ? 16 : (p.TT == 4 ? 8 : 4));   // lane pairs / thread (QTune)
  const int max_cons = 192;
  const int row_words = d_out / 16;
  // one token: tiles of <= 192 words (3 KB of packed row), so that the
  // epilogue is spread over several CTAs and fewer splits share an address
  // (measured on 4096 -> 11008: 4 tiles 16.4 us, 1 tile 21.6 us)
  const int max_words = (p.TT == 1) ? 192 : max_cons * lpt / 8;   // a multiple of 4
  // near-equal column tiles of a multiple of 4 words (16-byte bulk copies)
  int nct = (row_words + max_words - 1) / max_words;
  if (nct < 1) nct = 1;
  int tile = ((row_words + nct - 1) / nct + 3) / 4 * 4;
  if (tile > max_words) tile = max_words;
  p.n_ct = (row_words + tile - 1) / tile;
  p.vec_tile = tile;                                          // packed words per tile
  const int cons = (tile * 8 + lpt - 1) / lpt;
  p.threads = ((cons + 31) / 32) * 32 + 32;
  const int tile_bytes = tile * 4;
  p.rps = (16384 + tile_bytes / 2) / tile_bytes;
  if (p.rps < 1) p.rps = 1;
  if (p.rps > 16) p.rps = 16;
  const long ring = 90 * 1024;                               // two CTAs per SM
  long nst = ring / ((long)p.rps * tile_bytes);
  if (nst < 3) nst = 3;
  if (nst > 32) nst = 32;
  p.nst = (int)nst;
  p.rcap = 1024;
  p.smem = (size_t)p.nst * p.rps * tile_bytes + (size_t)p.rcap * (4 + p.TT);
  const long slots = (long)kNumSMs * 2;
  const long units = (long)p.n_ct * p.groups;
  long S = slots / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  const long max_by_rows = rows_bound / 8;       // keep >= ~8 rows per split
  if (S > max_by_rows) S = max_by_rows > 0 ? max_by_rows : 1;
  if (S > 256) S = 256;
  p.S = (int)S;
  // one accumulator copy: summing copies in the epilogue cost more than the
  // contention it removed on these sizes (measured)
  p.copies = 1;
  p.parts_elems = (size_t)p.copies * T * d_out;  // zeroed by the top-K kernel
  p.tickets = p.groups * p.n_ct;
  return p;
}

bool qgemv_supported(int d_out) { return d_out % 64 == 0; }   // 16-byte aligned packed rows

cudaError_t launch_qgemv(const QGemvArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  if (a.plan.mma == 2) return launch_qgemv_tc(a, s);
  if (a.plan.mma) {
    if (a.xq == nullptr) return cudaErrorInvalidValue;   // several tokens: dense codes
    switch (a.plan.TT) {
      case 8: return qlaunch_mma<1>(a, s);
      case 16: return qlaunch_mma<2>(a, s);
      case 24: return qlaunch_mma<3>(a, s);
      case 32: return qlaunch_mma<4>(a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.plan.TT) {
    case 1: return qlaunch<1>(a, s);
    case 2: return qlaunch<2>(a, s);
    case 4: return qlaunch<4>(a, s);
    case 8: return qlaunch<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_ternary_pack(const PackArgs& a, cudaStream_t s) {
  abs_sum_kernel<<<kPackSumBlocks, kPackNT, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t total = (size_t)(a.d_out / 16) * a.d_in;
  if (total == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((total + kPackNT - 1) / kPackNT);
  pack_kernel<<<blocks, kPackNT, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
