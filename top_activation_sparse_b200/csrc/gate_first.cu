// Gate-first dReLU FFN: the up projection reads only the rows of open gates.
//
// Source: Turbo Sparse summary (blog.csdn.net), Eq. 2: dReLU applies ReLU
// after both the gate and the up projection, h = ReLU(g + b_g) * ReLU(u + b_u).
// Wherever the gate branch is <= 0 the product is 0 whatever u is, so u_j is
// only needed for the columns j where some token's gate is open.  This is an
// exact reordering of the same arithmetic, not an approximation.
//
// Layout.  The gate projection keeps the input-major W_gate^T of the gather
// GEMV (one contiguous row per input), so it is the ordinary decode kernel
// over the listed inputs.  For the up projection the skipped dimension is the
// OUTPUT, so it needs W_up output-major ([d_ff, d_model], nn.Linear's own
// layout): the weights of one output column are then one contiguous 2 d_model
// bytes row, and the kernel below streams exactly the rows of open gates.
//
// Mapping (B200: 148 SMs).  One warp computes one open row at a time: its
// lanes read 16-byte vectors of the row (8 in flight per lane for one token,
// 4 for several; not kept in L1), multiply them with the same vectors of x
// (tiny, L1-resident, shared by every warp) and reduce across the warp.  Open rows are dealt to warps by
// rank: every CTA copies the open-gate bitmask and its prefix counts into
// shared memory, and a warp finds the word of its rank by binary search.
// The grid is 4 CTAs of 8 warps per SM, so about 4.7 K rows are in flight
// (the Mistral shape opens ~3 K of 14336 gates per token).
#include "gate_first.cuh"

#include <mutex>

namespace qs {
namespace {

constexpr int kUpThreads = 256;
constexpr int kUpWarps = kUpThreads / 32;
constexpr int kUpCtasPerSM = 4;
constexpr int kMaxWords = QS_MAX_ROW / 32;

template <typename WT> struct UpVec;
template <> struct UpVec<float> { static constexpr int V = 4; };
template <> struct UpVec<__nv_bfloat16> { static constexpr int V = 8; };

template <typename WT>
__device__ __forceinline__ void to_f32(const uint4& q, float (&w)[UpVec<WT>::V]) {
  if constexpr (UpVec<WT>::V == 8) {
    w[0] = bf16lo(q.x); w[1] = bf16hi(q.x);
    w[2] = bf16lo(q.y); w[3] = bf16hi(q.y);
    w[4] = bf16lo(q.z); w[5] = bf16hi(q.z);
    w[6] = bf16lo(q.w); w[7] = bf16hi(q.w);
  } else {
    w[0] = __uint_as_float(q.x); w[1] = __uint_as_float(q.y);
    w[2] = __uint_as_float(q.z); w[3] = __uint_as_float(q.w);
  }
}

// TT tokens per CTA row (blockIdx.y = token group); U vectors in flight per lane.
template <typename WT, int TT, int U>
__global__ void __launch_bounds__(kUpThreads) up_rows_kernel(UpRowsArgs a) {
  constexpr int V = UpVec<WT>::V;
  __shared__ uint32_t s_bits[kMaxWords];
  __shared__ int s_pre[kMaxWords + 1];     // open gates before word w
  __shared__ int s_wsum[kUpWarps];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d_model = a.d_model, d_ff = a.d_ff;
  const int nwords = (d_ff + 31) >> 5;

  pdl_begin();

  // ---- 1. this CTA's copy of the open-gate bitmask and its prefix counts ----
  const int wpt = (nwords + kUpThreads - 1) / kUpThreads;
  const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
  int mine = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t b = __ldcg(a.gate_bits + w);
    s_bits[w] = b;
    mine += __popc(b);
  }
  int inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) s_wsum[warp] = inc;
  __syncthreads();
  int run = inc - mine;
  for (int q = 0; q < warp; ++q) run += s_wsum[q];
  for (int w = w0; w < w1; ++w) {
    s_pre[w] = run;
    run += __popc(s_bits[w]);
  }
  if (tid == kUpThreads - 1) s_pre[nwords] = run;   // the last thread's run is the total
  __syncthreads();

  // ---- 2. once every CTA holds its copy, the last one clears the mask -------
  if (tid == 0) s_last = (atomicAdd(a.ticket, 1) == (int)(gridDim.x * gridDim.y) - 1);
  __syncthreads();
  if (s_last) {
    for (int w = tid; w < nwords; w += kUpThreads) a.gate_bits[w] = 0u;
    if (tid == 0) *a.ticket = 0;
  }
  const int n_open = s_pre[nwords];
  if (a.n_open != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *a.n_open = n_open;

  // ---- 3. warps take the open rows by rank ----------------------------------
  const int tok0 = blockIdx.y * TT;
  const int ntok = min(TT, a.T - tok0);
  const int nvec = d_model / V;                   // 16-byte vectors per row
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  const int gwarps = gridDim.x * kUpWarps;
  for (int r = blockIdx.x * kUpWarps + warp; r < n_open; r += gwarps) {
    // the word holding the rank-r open gate: the last w with s_pre[w] <= r
    int lo = 0, hi = nwords - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= r) lo = mid; else hi = mid - 1;
    }
    uint32_t bits = s_bits[lo];
    for (int skip = r - s_pre[lo]; skip > 0 && bits != 0u; --skip) bits &= bits - 1u;
    const int j = lo * 32 + __ffs(bits) - 1;        // warp-uniform
    if (bits == 0u || j >= d_ff) {                  // inconsistent mask: report, skip
      if (lane == 0) dev_fail(a.status, DEV_CHECK, 40, (uint32_t)r);
      continue;
    }
    const uint4* row = reinterpret_cast<const uint4*>(a.w_up) + (size_t)j * nvec;
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.0f;
    for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
      uint4 q[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * 32 + lane;
        q[u] = v < nvec ? ld_stream_v4(row + v) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < nvec) {
          float w[V];
          to_f32<WT>(q[u], w);
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            if (t < ntok) {
              float xf[V];
              to_f32<WT>(__ldg(xv + (size_t)(tok0 + t) * nvec + v), xf);
#pragma unroll
              for (int e = 0; e < V; ++e) acc[t] = fmaf(w[e], xf[e], acc[t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane == 0) {
      const float bu = a.b_up != nullptr ? a.b_up[j] : 0.0f;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t < ntok) {
          float* hp = a.h + (size_t)(tok0 + t) * d_ff + j;
          const float hv = *hp * fmaxf(acc[t] + bu, 0.0f);   // ReLU(g + b_g) * ReLU(u + b_u)
          *hp = hv;
          if (a.hbits != nullptr && hv != 0.0f) atomicOr(a.hbits + (j >> 5), 1u << (j & 31));
        }
      }
    }
  }
}

template <typename WT, int TT>
cudaError_t launch_tt(const UpRowsArgs& a, cudaStream_t s) {
  constexpr int U = TT == 1 ? 8 : 4;
  const dim3 grid(kNumSMs * kUpCtasPerSM, (a.T + TT - 1) / TT);
  cudaError_t e = launch_pdl(up_rows_kernel<WT, TT, U>, grid, dim3(kUpThreads), (size_t)0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename WT>
cudaError_t launch_wt(const UpRowsArgs& a, cudaStream_t s) {
  if (a.T == 1) return launch_tt<WT, 1>(a, s);
  if (a.T == 2) return launch_tt<WT, 2>(a, s);
  if (a.T <= 4) return launch_tt<WT, 4>(a, s);
  return launch_tt<WT, 8>(a, s);
}

__global__ void fill_kernel(float* p, int n, float v) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

static __device__ float g_unit[QS_MAX_ROW];
constexpr int kMaxDevices = 64;
std::mutex g_unit_mutex;
float* g_unit_addr[kMaxDevices] = {};

}  // namespace

cudaError_t launch_up_rows(const UpRowsArgs& a, cudaStream_t s) {
  const int V = a.bf16 ? 8 : 4;
  if (a.T <= 0) return cudaSuccess;
  if (a.d_ff < 1 || a.d_ff > QS_MAX_ROW || a.d_model < V || (a.d_model % V) != 0 ||
      a.x == nullptr || a.w_up == nullptr || a.gate_bits == nullptr || a.ticket == nullptr ||
      a.h == nullptr)
    return cudaErrorInvalidValue;
  return a.bf16 ? launch_wt<__nv_bfloat16>(a, s) : launch_wt<float>(a, s);
}

cudaError_t unit_vector_on_current_device(const float** out, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_unit_mutex);
  if (g_unit_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_unit);
    if (e != cudaSuccess) return e;
    fill_kernel<<<(QS_MAX_ROW + 255) / 256, 256, 0, s>>>(reinterpret_cast<float*>(p), QS_MAX_ROW, 1.0f);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);   // visible to every later call
    if (e != cudaSuccess) return e;
    g_unit_addr[dev] = reinterpret_cast<float*>(p);
  }
  *out = g_unit_addr[dev];
  return cudaSuccess;
}

}  // namespace qs
