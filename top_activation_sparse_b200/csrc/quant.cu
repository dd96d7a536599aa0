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

constexpr int kNT = 256;
constexpr int kNW = kNT / 32;
constexpr int kPiece = 256;
constexpr int kTileWords = 32;          // one 32-bit word (16 columns) per lane

template <int TT>
__global__ void __launch_bounds__(kNT) qgemv_kernel(QGemvArgs a) {
  constexpr int U = (TT <= 2) ? 8 : 4;
  constexpr int TILE = kTileWords * 16;  // 512 columns
  __shared__ int s_rows[kPiece];
  __shared__ int s_q[TT][kPiece];
  __shared__ int s_acc[TT][TILE];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.plan.S;
  const int ct = blockIdx.x;
  const int s = blockIdx.y;
  const int grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const int n_words = d_out / 16;
  const int wcol = ct * kTileWords + lane;
  const bool colok = wcol < n_words;

  pdl_begin();
  for (int q = tid; q < TT * TILE; q += kNT) (&s_acc[0][0])[q] = 0;

  const int n = min(max(*a.list_count, 0), d_in);
  const int r0 = (int)(((long long)n * s) / S);
  const int r1 = (int)(((long long)n * (s + 1)) / S);

  int acc[TT][16];
#pragma unroll
  for (int t = 0; t < TT; ++t)
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[t][c] = 0;

  for (int pb = r0; pb < r1; pb += kPiece) {
    const int np = min(kPiece, r1 - pb);
    __syncthreads();
    for (int j = tid; j < np; j += kNT) {
      int r = a.list[pb + j];
      const bool ok = (unsigned)r < (unsigned)d_in;
      if (!ok) {
        dev_fail(a.status, DEV_CHECK, 4, (uint32_t)r);
        r = 0;
      }
      s_rows[j] = r;
      if (a.list_q) {
        const int8_t* lq = a.list_q + (size_t)(pb + j) * a.T + tok0;
#pragma unroll
        for (int t = 0; t < TT; ++t) s_q[t][j] = (ok && t < ntok) ? (int)lq[t] : 0;
      } else {
#pragma unroll
        for (int t = 0; t < TT; ++t)
          s_q[t][j] = (ok && t < ntok) ? (int)a.xq[(size_t)(tok0 + t) * d_in + r] : 0;
      }
    }
    __syncthreads();
    for (int j0 = warp * U; j0 < np; j0 += kNW * U) {
      uint32_t wv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u;
        wv[u] = (j < np && colok) ? ld_stream_u32(a.wp + (size_t)s_rows[j] * n_words + wcol) : 0u;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u;
        int qv[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) qv[t] = (j < np) ? s_q[t][j] : 0;
        const uint32_t w = wv[u];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int code = (int)((w >> (2 * c)) & 3u);
          const int tv = (code & 1) - (code >> 1);     // 01 -> +1, 10 -> -1, 00 -> 0
#pragma unroll
          for (int t = 0; t < TT; ++t) acc[t][c] += qv[t] * tv;
        }
      }
    }
  }

  // ---- combine warps (integer adds: exact in any order) --------------------
#pragma unroll
  for (int t = 0; t < TT; ++t)
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (acc[t][c] != 0) atomicAdd(&s_acc[t][lane * 16 + c], acc[t][c]);
  __syncthreads();

  const bool direct = (S == 1);
  for (int q = tid; q < TT * TILE; q += kNT) {
    const int t = q / TILE;
    const int gc = ct * TILE + (q - t * TILE);
    if (t >= ntok || gc >= d_out) continue;
    const int tok = tok0 + t;
    const int v = s_acc[t][q - t * TILE];
    if (direct) {
      const float r = __fdiv_rn(__fmul_rn(a.alpha, a.gamma[tok]), 127.0f);
      a.y[(size_t)tok * d_out + gc] = __fmul_rn(__int2float_rn(v), r);
      if (a.acc) a.acc[(size_t)tok * d_out + gc] = v;
    } else {
      a.parts[((size_t)s * a.T + tok) * d_out + gc] = v;
    }
  }
  if (direct) return;

  __threadfence();
  __syncthreads();
  int32_t* ticket = a.tickets + grp * a.plan.n_ct + ct;
  if (tid == 0) s_last = (atomicAdd(ticket, 1) == S - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int q = tid; q < TT * TILE; q += kNT) {
    const int t = q / TILE;
    const int gc = ct * TILE + (q - t * TILE);
    if (t >= ntok || gc >= d_out) continue;
    const int tok = tok0 + t;
    const int32_t* p = a.parts + (size_t)tok * d_out + gc;
    const size_t step = (size_t)a.T * d_out;
    int v = 0;
    for (int s2 = 0; s2 < S; ++s2) v += __ldcg(p + (size_t)s2 * step);
    const float r = __fdiv_rn(__fmul_rn(a.alpha, a.gamma[tok]), 127.0f);
    a.y[(size_t)tok * d_out + gc] = __fmul_rn(__int2float_rn(v), r);
    if (a.acc) a.acc[(size_t)tok * d_out + gc] = v;
  }
  if (tid == 0) *ticket = 0;
}

template <int TT>
cudaError_t qlaunch(const QGemvArgs& a, cudaStream_t s) {
  dim3 grid(a.plan.n_ct, a.plan.S, a.plan.groups);
  cudaError_t e = launch_pdl(qgemv_kernel<TT>, grid, dim3(kNT), 0, s, a);
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

GemvPlan plan_qgemv(int T, int d_out, int rows_bound) {
  GemvPlan p{};
  p.TT = (T <= 1) ? 1 : (T == 2 ? 2 : (T <= 4 ? 4 : 8));
  p.groups = (T + p.TT - 1) / p.TT;
  const int n_words = d_out / 16;
  p.n_ct = (n_words + kTileWords - 1) / kTileWords;
  p.mats = 1;
  const int per_sm = (p.TT <= 2) ? 6 : (p.TT == 4 ? 4 : 2);
  const long slots = (long)kNumSMs * per_sm;
  const long units = (long)p.n_ct * p.groups;
  long S = slots / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  const long max_by_rows = rows_bound / 16;
  if (S > max_by_rows) S = max_by_rows > 0 ? max_by_rows : 1;
  if (S > 256) S = 256;
  p.S = (int)S;
  p.parts_elems = (size_t)p.S * (size_t)T * d_out;
  p.tickets = p.groups * p.n_ct;
  return p;
}

cudaError_t launch_qgemv(const QGemvArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
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
