// Top-K on |x| per token row: radix select of the K-th largest magnitude,
// then an order-preserving compaction of the kept entries.
//
// Source: Q-Sparse news article (zxwl-tech.com), section "Top-K
// sparsification": |X| is ranked, the K largest entries are kept, a 0/1 mask
// M marks them and X_sparse = X (.) M.  The pages only say "sort"; a full
// sort is not needed to find the K largest, so each row is handled by one CTA
// that
//   1. writes one 32-bit entry per element into shared memory (the raw bits
//      of x; for the quantized path the int8 code and its magnitude),
//   2. finds the K-th largest key (key = |x| as bits with the sign cleared,
//      whose unsigned order is the order of |x|) with radix digits of up to
//      11 bits (3 passes for f32, 2 for bf16, 1 for int8 codes): a
//      shared-memory histogram per digit and one block-wide scan to locate
//      the digit that holds the K-th key, stopping early once every element
//      of that digit is needed,
//   3. gives every thread a contiguous chunk of the row, counts the chunk's
//      entries above / at the threshold, and with ONE block scan learns where
//      its kept entries go, so that entries above the threshold and the first
//      `remaining` ties (lowest indices first) land at their final position of
//      the ascending index list without any per-tile synchronisation.
// The quantized path (BitNet b1.58 + Q-Sparse, same article's paragraph on
// quantized inputs) first computes the per-token absmax int8 code
// q = clamp(rint(x * 127 / (amax + eps)), -127, 127) in float32 steps and then
// ranks |q|.
//
// For the projection kernels the row also produces a dense masked copy (f32
// values, or int8 codes) and a list of input rows that carry a kept nonzero
// value; with several token rows the last CTA to finish (an atomic ticket, no
// waiting) merges the rows into the union list.
#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Key layout per input kind and the radix digits used to find the K-th key:
// (shift, width) of each pass, most significant first.
template <int KIND> struct KeyTraits;
template <> struct KeyTraits<TK_F32> {
  static constexpr uint32_t kMask = 0x7fffffffu;  // |x| bits (31)
  static constexpr int kPasses = 3;
  __device__ static constexpr int shift(int p) { return p == 0 ? 20 : (p == 1 ? 9 : 0); }
  __device__ static constexpr int width(int p) { return p == 2 ? 9 : 11; }
};
template <> struct KeyTraits<TK_BF16> {
  static constexpr uint32_t kMask = 0x7fffu;      // |x| bits (15)
  static constexpr int kPasses = 2;
  __device__ static constexpr int shift(int p) { return p == 0 ? 4 : 0; }
  __device__ static constexpr int width(int p) { return p == 0 ? 11 : 4; }
};
struct QuantKeys {
  static constexpr uint32_t kMask = 0xffu;        // |q| in the low byte (<= 127)
  static constexpr int kPasses = 1;
  __device__ static constexpr int shift(int) { return 0; }
  __device__ static constexpr int width(int) { return 8; }
};
template <> struct KeyTraits<TK_QUANT_F32> : QuantKeys {};
template <> struct KeyTraits<TK_QUANT_BF16> : QuantKeys {};

constexpr int kMaxBins = 2048;

template <int KIND>
__device__ __forceinline__ uint32_t load_raw(const void* x, size_t i) {
  if constexpr (KIND == TK_F32 || KIND == TK_QUANT_F32) {
    return __ldg(reinterpret_cast<const uint32_t*>(x) + i);
  } else {
    return (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(x) + i);
  }
}

// raw bits -> float value of the input
template <int KIND>
__device__ __forceinline__ float raw_to_f32(uint32_t raw) {
  if constexpr (KIND == TK_F32 || KIND == TK_QUANT_F32) return __uint_as_float(raw);
  else return __uint_as_float(raw << 16);
}

// raw bits -> |x| as non-negative float bits (monotone in |x|)
template <int KIND>
__device__ __forceinline__ uint32_t raw_abs_f32bits(uint32_t raw) {
  if constexpr (KIND == TK_F32 || KIND == TK_QUANT_F32) return raw & 0x7fffffffu;
  else return (raw & 0x7fffu) << 16;
}

// Block-wide exclusive scan of two 32-bit values per thread.  `sw` holds
// 2 * (NW + 1) words and must not be reused before the next __syncthreads.
template <int NT>
__device__ __forceinline__ void block_scan2(uint32_t a, uint32_t b, uint32_t* sw, uint32_t& ea,
                                            uint32_t& eb, uint32_t& ta, uint32_t& tb) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t xa = __shfl_up_sync(kFull, ia, o);
    const uint32_t xb = __shfl_up_sync(kFull, ib, o);
    if (lane >= o) { ia += xa; ib += xb; }
  }
  if (lane == 31) { sw[warp] = ia; sw[NW + 1 + warp] = ib; }
  __syncthreads();
  if (warp == 0) {
    const uint32_t wa = lane < NW ? sw[lane] : 0u;
    const uint32_t wb = lane < NW ? sw[NW + 1 + lane] : 0u;
    uint32_t sa = wa, sb = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t xa = __shfl_up_sync(kFull, sa, o);
      const uint32_t xb = __shfl_up_sync(kFull, sb, o);
      if (lane >= o) { sa += xa; sb += xb; }
    }
    if (lane < NW) { sw[lane] = sa - wa; sw[NW + 1 + lane] = sb - wb; }
    if (lane == 31) { sw[NW] = sa; sw[2 * NW + 1] = sb; }
  }
  __syncthreads();
  ea = sw[warp] + ia - a;
  eb = sw[NW + 1 + warp] + ib - b;
  ta = sw[NW];
  tb = sw[2 * NW + 1];
}

template <int KIND, int NT>
__global__ void __launch_bounds__(NT) topk_kernel(TopkArgs a) {
  using KT = KeyTraits<KIND>;
  constexpr int NW = NT / 32;
  constexpr uint32_t MASK = KT::kMask;
  constexpr bool QUANT = (KIND == TK_QUANT_F32 || KIND == TK_QUANT_BF16);

  extern __shared__ uint32_t s_ent[];          // [d]
  __shared__ int s_hist[kMaxBins];
  __shared__ uint32_t s_scan[2][2 * (NW + 1)];
  __shared__ uint32_t s_sel[3];
  __shared__ uint32_t s_red[NW];
  __shared__ int s_last;
  __shared__ int s_wnnz[NW];

  const int row = blockIdx.x;
  const int d = a.d;
  const int k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t rbase = (size_t)row * (size_t)d;
  int sbuf = 0;

  pdl_begin();
  grid_zero(a.zero, a.zero_n);
  uint32_t my_nnz = 0;

  // ---- 1. entries --------------------------------------------------------
  if constexpr (QUANT) {
    uint32_t m = 0;
    for (int i = tid; i < d; i += NT) m = max(m, raw_abs_f32bits<KIND>(load_raw<KIND>(a.x, rbase + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    if (warp == 0) {
      uint32_t v = lane < NW ? s_red[lane] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(kFull, v, o));
      if (lane == 0) s_red[0] = v;
    }
    __syncthreads();
    const float amax = __uint_as_float(s_red[0]);
    const float gamma = __fadd_rn(amax, a.eps);
    const float scale = __fdiv_rn(127.0f, gamma);
    if (tid == 0 && a.gamma) a.gamma[row] = gamma;
    for (int i = tid; i < d; i += NT) {
      const float v = raw_to_f32<KIND>(load_raw<KIND>(a.x, rbase + i));
      int qi = __float2int_rn(__fmul_rn(v, scale));
      qi = min(127, max(-127, qi));
      const uint32_t mag = (uint32_t)(qi < 0 ? -qi : qi);
      s_ent[i] = mag | ((uint32_t)(uint8_t)(int8_t)qi << 8);
      my_nnz += (mag != 0u);
      if (a.q_full) a.q_full[rbase + i] = (int8_t)qi;
    }
  } else {
    for (int i = tid; i < d; i += NT) {
      const uint32_t e = load_raw<KIND>(a.x, rbase + i);
      s_ent[i] = e;
      my_nnz += ((e & MASK) != 0u);
    }
  }
  {
    const uint32_t w = __reduce_add_sync(kFull, my_nnz);
    if (lane == 0) s_wnnz[warp] = (int)w;
  }
  __syncthreads();
  int nnz = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) nnz += s_wnnz[w];

  // ---- 2. radix select of the K-th largest key ---------------------------
  // After this block an element is kept iff (key >> shift) > P, or it equals
  // P and fewer than `remaining` equal elements precede it.
  uint32_t P;
  int shift;
  int remaining;
  if (k <= 0) {
    P = 0xffffffffu; shift = 31; remaining = 0;        // nothing is kept
  } else if (k >= d) {
    P = 0u; shift = 31; remaining = d;                 // every key >> 31 == 0: all kept
  } else if (nnz <= k) {
    // At most K nonzero entries: every nonzero beats every zero, so all of
    // them are kept together with the lowest-index zeros (threshold key 0).
    P = 0u; shift = 0; remaining = k - nnz;
  } else {
    uint32_t prefix = 0;
    remaining = k;
    shift = 0;
#pragma unroll 1
    for (int p = 0; p < KT::kPasses; ++p) {
      const int sh = KT::shift(p);
      const int nb = 1 << KT::width(p);
      for (int j = tid; j < nb; j += NT) s_hist[j] = 0;
      __syncthreads();
      const int hi = sh + KT::width(p);
      const uint32_t himask = hi >= 32 ? 0u : (0xffffffffu << hi);
      for (int i = tid; i < d; i += NT) {
        const uint32_t key = s_ent[i] & MASK;
        if (((key ^ prefix) & himask) == 0u) atomicAdd(&s_hist[(key >> sh) & (uint32_t)(nb - 1)], 1);
      }
      __syncthreads();
      // every thread has read the previous pass's s_sel before the barrier above
      if (tid == 0) s_sel[0] = 0xffffffffu;
      // thread j sums bins [nb - (j+1)*bpt, nb - j*bpt): largest digits first
      const int bpt = (nb + NT - 1) / NT;
      const int top = nb - 1 - tid * bpt;
      uint32_t local = 0;
      for (int b = 0; b < bpt; ++b)
        if (top - b >= 0) local += (uint32_t)s_hist[top - b];
      uint32_t excl, unused_e, tot, unused_t;
      block_scan2<NT>(local, 0u, s_scan[sbuf], excl, unused_e, tot, unused_t);
      sbuf ^= 1;
      if ((int)excl < remaining && remaining <= (int)(excl + local)) {
        int run = (int)excl;
        for (int b = 0; b < bpt; ++b) {
          const int c = s_hist[top - b];
          if (run + c >= remaining) {
            s_sel[0] = (uint32_t)(top - b);
            s_sel[1] = (uint32_t)run;
            s_sel[2] = (uint32_t)c;
            break;
          }
          run += c;
        }
      }
      __syncthreads();
      const uint32_t digit = s_sel[0];
      if (digit == 0xffffffffu) {                   // counts inconsistent: report, stop
        if (tid == 0) dev_fail(a.status, DEV_CHECK, 1, (uint32_t)row);
        shift = sh;
        break;
      }
      remaining -= (int)s_sel[1];
      prefix |= digit << sh;
      shift = sh;
      if ((int)s_sel[2] == remaining) break;      // the whole digit is kept
    }
    P = prefix >> shift;
  }

  // ---- 3. compaction in index order (contiguous chunk per thread) --------
  const int chunk = (d + NT - 1) / NT;
  const int i0 = min(tid * chunk, d);
  const int i1 = min(i0 + chunk, d);
  uint32_t n_gt = 0, n_eq = 0, n_eqnz = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = s_ent[i] & MASK;
    const uint32_t c = key >> shift;
    n_gt += (c > P);
    n_eq += (c == P);
    n_eqnz += (c == P && key != 0u);
  }
  // counts fit 16 bits (d <= QS_MAX_ROW < 65536): scan (gt | eq << 16) and eqnz
  uint32_t e_ge, e_eqnz, t_ge, t_eqnz;
  block_scan2<NT>(n_gt | (n_eq << 16), n_eqnz, s_scan[sbuf], e_ge, e_eqnz, t_ge, t_eqnz);
  sbuf ^= 1;
  int gtb = (int)(e_ge & 0xffffu);
  int eqb = (int)(e_ge >> 16);
  // Kept nonzeros before this chunk: every element above P is nonzero; equal
  // elements are nonzero iff P != 0, and when P == 0 with a nonzero key the
  // whole digit is kept (early stop), so its nonzero count is exact.
  int nzb = gtb + (P != 0u ? min(eqb, remaining) : (int)e_eqnz);
  const bool list_direct = (a.list != nullptr) && (a.T == 1);
  for (int i = i0; i < i1; ++i) {
    const uint32_t ent = s_ent[i];
    const uint32_t key = ent & MASK;
    const uint32_t c = key >> shift;
    const bool gt = c > P;
    const bool eq = c == P;
    const bool sel = gt || (eq && eqb < remaining);
    if (sel) {
      const int pos = gtb + min(eqb, remaining);
      if (pos < k) {
        const size_t o = (size_t)row * (size_t)k + (size_t)pos;
        if (a.idx) a.idx[o] = i;
        if (a.val) {
          if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.val)[o] = ent;
          else if constexpr (KIND == TK_BF16) reinterpret_cast<uint16_t*>(a.val)[o] = (uint16_t)ent;
        }
      } else {
        dev_fail(a.status, DEV_CHECK, 2, (uint32_t)row);   // inconsistent select
      }
      if (list_direct && key != 0u) {
        a.list[nzb] = i;
        if constexpr (QUANT) {
          if (a.list_q) a.list_q[nzb] = (int8_t)(ent >> 8);
        } else {
          if (a.list_val) a.list_val[nzb] = raw_to_f32<KIND>(ent);
        }
        ++nzb;
      }
    }
    if (a.mask) a.mask[rbase + i] = sel ? 1 : 0;
    gtb += gt;
    eqb += eq;
    s_ent[i] = sel ? ent : 0u;                  // X_sparse entry (bits) for the dense outputs
  }
  if (list_direct && tid == 0) {
    const int tot_gt = (int)(t_ge & 0xffffu), tot_eq = (int)(t_ge >> 16);
    *a.list_count = tot_gt + (P != 0u ? min(tot_eq, remaining) : (int)t_eqnz);
  }
  __syncthreads();
  // coalesced dense outputs; with several tokens also OR this row's kept
  // nonzeros into the union bitmask (one atomic per 32 inputs)
  const bool want_union = (a.list != nullptr) && (a.T > 1);
  for (int base = 0; base < d; base += NT) {
    const int i = base + tid;
    const bool valid = i < d;
    const uint32_t ent = valid ? s_ent[i] : 0u;
    if (valid) {
      if constexpr (QUANT) {
        if (a.xq) a.xq[rbase + i] = (int8_t)(ent >> 8);
      } else {
        if (a.xsf) a.xsf[rbase + i] = raw_to_f32<KIND>(ent);
        if (a.xs) {
          if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.xs)[rbase + i] = ent;
          else reinterpret_cast<uint16_t*>(a.xs)[rbase + i] = (uint16_t)ent;
        }
      }
    }
    if (want_union) {
      const unsigned b = __ballot_sync(kFull, valid && (ent & MASK) != 0u);
      if (lane == 0 && b != 0u) atomicOr(a.union_bits + (base + warp * 32) / 32, b);
    }
  }

  // ---- 4. union of the rows' kept nonzeros (several tokens) --------------
  if (a.list != nullptr && a.T > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(a.ticket, 1) == a.T - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // list the set bits in index order: a contiguous run of words per thread
    const int nwords = (d + 31) / 32;
    const int wpt = (nwords + NT - 1) / NT;
    const int w0 = min(tid * wpt, nwords);
    const int w1 = min(w0 + wpt, nwords);
    uint32_t n_any = 0;
    for (int w = w0; w < w1; ++w) n_any += __popc(__ldcg(a.union_bits + w));
    uint32_t e_any, e_unused, t_any, t_unused;
    block_scan2<NT>(n_any, 0u, s_scan[sbuf], e_any, e_unused, t_any, t_unused);
    int pos = (int)e_any;
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = __ldcg(a.union_bits + w);
      a.union_bits[w] = 0u;                      // leave the bitmask clean for the next call
      while (bits) {
        const int bpos = __ffs(bits) - 1;
        a.list[pos++] = w * 32 + bpos;
        bits &= bits - 1u;
      }
    }
    if (tid == 0) {
      *a.list_count = (int)t_any;
      *a.ticket = 0;       // leave the counter clean for the next call
    }
  }
}

template <int KIND, int NT>
cudaError_t launch_kind(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)a.d * sizeof(uint32_t);
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(topk_kernel<KIND, NT>, (int)(QS_MAX_ROW * sizeof(uint32_t)),
                                   &configured);
  if (e != cudaSuccess) return e;
  e = launch_pdl(topk_kernel<KIND, NT>, dim3(a.T), dim3(NT), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_nt(const TopkArgs& a, cudaStream_t s) {
  switch (a.kind) {
    case TK_F32: return launch_kind<TK_F32, NT>(a, s);
    case TK_BF16: return launch_kind<TK_BF16, NT>(a, s);
    case TK_QUANT_F32: return launch_kind<TK_QUANT_F32, NT>(a, s);
    case TK_QUANT_BF16: return launch_kind<TK_QUANT_BF16, NT>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.d <= 0) return cudaSuccess;
  // Few rows: a full 1024-thread CTA per row keeps the latency down.  Many
  // rows (prefill): 256-thread CTAs so that several rows share an SM.
  if (a.T >= 2 * kNumSMs) return launch_nt<256>(a, s);
  return launch_nt<1024>(a, s);
}

}  // namespace qs
