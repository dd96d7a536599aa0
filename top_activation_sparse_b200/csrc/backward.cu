// Backward of the sparse projection under the straight-through estimator,
// decode-size batches (the tensor-core GEMMs of prefill_gemm.cu take the
// large ones).
//
// Source: Q-Sparse news article (zxwl-tech.com), section "Top-K
// sparsification", paragraphs on the straight-through estimator: top-K has a
// zero gradient almost everywhere, so the gradient with respect to the
// sparsified input is passed unchanged to the input.  For Y = X_sparse . W^T
// (W^T input-major, [d_in, d_out]):
//   dL/dX   = dL/dY . W          (no mask: the estimator copies it through)
//   dL/dW^T = X_sparse^T . dL/dY (row i is nonzero only if some token kept i)
//
// rowdot_kernel: dL/dX[t, i] = sum_j dL/dY[t, j] * W^T[i, j] for every row i.
//   Every weight row is read once (the estimator applies no mask), so the
//   kernel streams W^T like the gather-GEMV streams its kept rows: column
//   tiles of a few KB, a bulk-copy ring of row segments per CTA, rows split
//   over CTAs.  Each consumer thread owns one 16-byte column vector and keeps
//   dL/dY for its columns and up to 8 tokens in registers; per staged row it
//   forms its partial dot products, the warp reduces them with shuffles, and
//   the warps' sums meet in shared memory; the column tiles of a row are added
//   with f32 reductions into dL/dX, which the launch zeroes first.
// rowaxpy_kernel: dL/dW^T[i, :] += sum_t X_sparse[t, i] * dL/dY[t, :] for the
//   rows the top-K listed (the inputs some token kept with a nonzero value);
//   no other row is read or written.  Each thread owns a float4 of a row.
#include <algorithm>

#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr int kBwdMaxConsumers = 384;
constexpr int kBwdMaxStages = 32;
constexpr int kBwdMaxRowsPerStage = 8;

template <typename WT> struct BwdVec;
template <> struct BwdVec<float> { static constexpr int V = 4; };
template <> struct BwdVec<__nv_bfloat16> { static constexpr int V = 8; };

template <typename WT>
__device__ __forceinline__ void bwd_unpack(const uint4& q, float (&w)[BwdVec<WT>::V]) {
  if constexpr (BwdVec<WT>::V == 8) {
    w[0] = bf16lo(q.x); w[1] = bf16hi(q.x);
    w[2] = bf16lo(q.y); w[3] = bf16hi(q.y);
    w[4] = bf16lo(q.z); w[5] = bf16hi(q.z);
    w[6] = bf16lo(q.w); w[7] = bf16hi(q.w);
  } else {
    w[0] = __uint_as_float(q.x); w[1] = __uint_as_float(q.y);
    w[2] = __uint_as_float(q.z); w[3] = __uint_as_float(q.w);
  }
}

__device__ __forceinline__ void red_add_f32(float* dst, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst), "f"(v) : "memory");
}

template <typename WT, int TT>
__global__ void __launch_bounds__(kBwdMaxConsumers + 32, 1) rowdot_kernel(RowDotArgs a) {
  constexpr int V = BwdVec<WT>::V;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t s_full[kBwdMaxStages];
  __shared__ __align__(8) uint64_t s_empty[kBwdMaxStages];
  __shared__ float s_part[kBwdMaxRowsPerStage][TT][kBwdMaxConsumers / 32];
  __shared__ int s_err;

  const RowDotPlan& P = a.plan;
  const int NC = P.threads - 32;                 // consumer threads; the last warp produces
  const int NWC = NC / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = tid >= NC;
  const int tile_bytes = P.vec_tile * 16;
  const int ct = blockIdx.x, s = blockIdx.y, grp = blockIdx.z;
  const int tok0 = grp * TT;
  const int ntok = min(TT, a.T - tok0);
  const int d_in = a.d_in, d_out = a.d_out;
  const size_t row_bytes = (size_t)d_out * sizeof(WT);
  const size_t cbyte = (size_t)ct * tile_bytes;
  const int tbytes = (int)min((size_t)tile_bytes, row_bytes - cbyte);
  const int tvec = tbytes / 16;
  const unsigned char* Wb = reinterpret_cast<const unsigned char*>(a.wt) + cbyte;
  const int col = (ct * P.vec_tile + tid) * V;
  const bool mine = !producer && tid < tvec;
  // rows [r0, r1) of this split
  const int r0 = (int)(((long long)d_in * s) / P.S);
  const int r1 = (int)(((long long)d_in * (s + 1)) / P.S);
  const int nrows = r1 - r0;
  const int nstage = (nrows + P.rps - 1) / P.rps;

  pdl_begin();
  if (tid == 0) {
    for (int i = 0; i < P.nst; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], NWC);
    }
    mbar_fence_init();
    s_err = 0;
  }
  // dL/dY of this thread's columns for the group's tokens (registers)
  float g[TT][V];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    if (mine && t < ntok) {
      const uint4 q = *reinterpret_cast<const uint4*>(
          reinterpret_cast<const unsigned char*>(a.grad_y) + ((size_t)(tok0 + t) * d_out + col) * sizeof(WT));
      bwd_unpack<WT>(q, g[t]);
    } else {
#pragma unroll
      for (int e = 0; e < V; ++e) g[t][e] = 0.0f;
    }
  }
  __syncthreads();

  if (producer) {
    for (int st = 0; st < nstage; ++st) {
      const int slot = st % P.nst;
      int ok = 1;
      if (lane == 0 && st >= P.nst && !mbar_wait(&s_empty[slot], (uint32_t)((st / P.nst) - 1) & 1u)) {
        dev_fail(a.status, DEV_TIMEOUT, 30, (uint32_t)st);
        atomicExch(&s_err, 1);
        ok = 0;
      }
      if (__shfl_sync(0xffffffffu, ok, 0) == 0) break;
      const int j0 = r0 + st * P.rps;
      const int cnt = min(P.rps, r1 - j0);
      if (lane == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)(cnt * tbytes));
      __syncwarp();
      if (lane < cnt)
        bulk_g2s(smem + ((size_t)slot * P.rps + lane) * tile_bytes, Wb + (size_t)(j0 + lane) * row_bytes,
                 (uint32_t)tbytes, &s_full[slot]);
    }
  } else {
    for (int st = 0; st < nstage; ++st) {
      const int slot = st % P.nst;
      const bool ready = !*(volatile int*)&s_err &&
                         mbar_wait_backoff(&s_full[slot], (uint32_t)(st / P.nst) & 1u);
      if (!ready && !*(volatile int*)&s_err) {
        if (lane == 0) dev_fail(a.status, DEV_TIMEOUT, 31, (uint32_t)st);
        atomicExch(&s_err, 1);
      }
      const int j0 = r0 + st * P.rps;
      const int cnt = min(P.rps, r1 - j0);
      // partial dot products of this thread's columns, reduced over the warp
      for (int r = 0; r < cnt; ++r) {
        float p[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) p[t] = 0.0f;
        if (ready && mine) {
          const uint4 q = *reinterpret_cast<const uint4*>(smem + ((size_t)slot * P.rps + r) * tile_bytes +
                                                          (size_t)tid * 16);
          float w[V];
          bwd_unpack<WT>(q, w);
#pragma unroll
          for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int e = 0; e < V; ++e) p[t] = fmaf(w[e], g[t][e], p[t]);
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) p[t] += __shfl_xor_sync(0xffffffffu, p[t], o);
        }
        if (lane == 0) {
#pragma unroll
          for (int t = 0; t < TT; ++t) s_part[r][t][warp] = p[t];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[slot]);   // this warp is done with the stage
      // the warps' sums meet in shared memory (consumer warps sync on a named
      // barrier), then warp 0 adds the rows' tile sums into dL/dX
      asm volatile("bar.sync 1, %0;" ::"r"(NC) : "memory");
      if (warp == 0) {
        for (int i = lane; i < cnt * TT; i += 32) {
          const int r = i / TT, t = i - (i / TT) * TT;
          if (t < ntok) {
            float sum = 0.0f;
            for (int w = 0; w < NWC; ++w) sum += s_part[r][t][w];
            red_add_f32(a.grad_x + (size_t)(tok0 + t) * d_in + j0 + r, sum);
          }
        }
      }
      // s_part is rewritten only after warp 0 has read it
      asm volatile("bar.sync 1, %0;" ::"r"(NC) : "memory");
    }
  }
  if (s_err && tid == 0) {
    for (int i = 0; i < P.nst && i < nstage; ++i) {
      const int g_last = nstage - 1 - i;
      mbar_wait(&s_full[g_last % P.nst], (uint32_t)(g_last / P.nst) & 1u);
    }
  }
}

template <typename WT>
__global__ void __launch_bounds__(256) rowaxpy_kernel(RowAxpyArgs a) {
  const int d_out = a.d_out, T = a.T;
  const int n4 = d_out / 4;                       // float4 groups of a row (d_out % 4 == 0)
  const int v4 = blockIdx.x * 256 + threadIdx.x;  // this thread's float4 of every row
  pdl_begin();
  const int n = min(max(*a.list_count, 0), a.d_in);
  const int rA = (int)(((long long)n * blockIdx.y) / gridDim.y);
  const int rB = (int)(((long long)n * (blockIdx.y + 1)) / gridDim.y);
  if (v4 >= n4) return;
  const int c = v4 * 4;
#pragma unroll 2
  for (int j = rA; j < rB; ++j) {
    const int i = a.list[j];
    if ((unsigned)i >= (unsigned)a.d_in) {         // a corrupted list is reported, never followed
      dev_fail(a.status, DEV_CHECK, 32, (uint32_t)i);
      continue;
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t = 0; t < T; ++t) {
      const float v = a.list_val ? a.list_val[j] : a.xsf[(size_t)t * a.d_in + i];
      if (v == 0.0f) continue;
      float gv[4];
      if constexpr (sizeof(WT) == 2) {
        const uint2 q = *reinterpret_cast<const uint2*>(
            reinterpret_cast<const uint16_t*>(a.grad_y) + (size_t)t * d_out + c);
        gv[0] = bf16lo(q.x); gv[1] = bf16hi(q.x); gv[2] = bf16lo(q.y); gv[3] = bf16hi(q.y);
      } else {
        const float4 q = *reinterpret_cast<const float4*>(
            reinterpret_cast<const float*>(a.grad_y) + (size_t)t * d_out + c);
        gv[0] = q.x; gv[1] = q.y; gv[2] = q.z; gv[3] = q.w;
      }
      acc.x = fmaf(v, gv[0], acc.x);
      acc.y = fmaf(v, gv[1], acc.y);
      acc.z = fmaf(v, gv[2], acc.z);
      acc.w = fmaf(v, gv[3], acc.w);
    }
    // add into the existing gradient; a sum of exactly zero leaves it untouched
    float4* dst = reinterpret_cast<float4*>(a.grad_wt + (size_t)i * d_out + c);
    if (acc.x == 0.0f && acc.y == 0.0f && acc.z == 0.0f && acc.w == 0.0f) continue;
    float4 p = *dst;
    if (acc.x != 0.0f) p.x += acc.x;
    if (acc.y != 0.0f) p.y += acc.y;
    if (acc.z != 0.0f) p.z += acc.z;
    if (acc.w != 0.0f) p.w += acc.w;
    *dst = p;
  }
}

__global__ void __launch_bounds__(256) zero_kernel(float* p, size_t n) {
  pdl_begin();
  const size_t stride = (size_t)gridDim.x * 256;
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += stride) p[i] = 0.0f;
}

template <typename WT, int TT>
cudaError_t rowdot_launch(const RowDotArgs& a, cudaStream_t s) {
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(rowdot_kernel<WT, TT>, 200 * 1024, &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(a.plan.n_ct, a.plan.S, a.plan.groups);
  e = launch_pdl(rowdot_kernel<WT, TT>, grid, dim3(a.plan.threads), a.plan.smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename WT>
cudaError_t rowdot_tt(const RowDotArgs& a, cudaStream_t s) {
  switch (a.plan.TT) {
    case 1: return rowdot_launch<WT, 1>(a, s);
    case 2: return rowdot_launch<WT, 2>(a, s);
    case 4: return rowdot_launch<WT, 4>(a, s);
    case 8: return rowdot_launch<WT, 8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

RowDotPlan plan_rowdot(int T, int d_in, int d_out, int elem_bytes) {
  RowDotPlan p{};
  p.TT = T <= 1 ? 1 : (T == 2 ? 2 : (T <= 4 ? 4 : 8));
  p.groups = (T + p.TT - 1) / p.TT;
  const int vec_row = (int)(((long)d_out * elem_bytes) / 16);
  int nct = (vec_row + kBwdMaxConsumers - 1) / kBwdMaxConsumers;
  for (int c = nct; c <= nct + 8 && c <= vec_row; ++c)   // prefer equal tiles
    if (vec_row % c == 0) { nct = c; break; }
  p.n_ct = nct;
  p.vec_tile = (vec_row + nct - 1) / nct;
  p.threads = ((p.vec_tile + 31) / 32) * 32 + 32;
  const int tile_bytes = p.vec_tile * 16;
  p.rps = (16384 + tile_bytes / 2) / tile_bytes;
  if (p.rps < 1) p.rps = 1;
  if (p.rps > kBwdMaxRowsPerStage) p.rps = kBwdMaxRowsPerStage;
  long nst = (160L * 1024) / ((long)p.rps * tile_bytes);
  if (nst < 2) nst = 2;
  if (nst > kBwdMaxStages) nst = kBwdMaxStages;
  p.nst = (int)nst;
  p.smem = (size_t)p.nst * p.rps * tile_bytes;
  const long units = (long)nct * p.groups;
  long S = (long)kNumSMs / (units > 0 ? units : 1);
  if (S < 1) S = 1;
  if (S > d_in) S = d_in;
  p.S = (int)S;
  return p;
}

cudaError_t launch_rowdot(const RowDotArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.d_in <= 0) return cudaSuccess;
  const size_t n = (size_t)a.T * a.d_in;
  const unsigned zb = (unsigned)std::min<size_t>((n + 255) / 256, (size_t)kNumSMs * 4);
  cudaError_t e = launch_pdl(zero_kernel, dim3(zb), dim3(256), (size_t)0, s, a.grad_x, n);
  if (e != cudaSuccess) return e;
  return a.bf16 ? rowdot_tt<__nv_bfloat16>(a, s) : rowdot_tt<float>(a, s);
}

cudaError_t launch_rowaxpy(const RowAxpyArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.d_out <= 0) return cudaSuccess;
  const int n4 = a.d_out / 4;
  const int cx = (n4 + 255) / 256;
  int ry = (kNumSMs * 4) / cx;
  if (ry < 1) ry = 1;
  if (ry > 1024) ry = 1024;
  cudaError_t e = a.bf16 ? launch_pdl(rowaxpy_kernel<__nv_bfloat16>, dim3(cx, ry), dim3(256), (size_t)0, s, a)
                         : launch_pdl(rowaxpy_kernel<float>, dim3(cx, ry), dim3(256), (size_t)0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qs
