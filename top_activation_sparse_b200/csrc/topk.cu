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
#include <algorithm>

#include "qs_internal.cuh"

namespace qs {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Key layout per input kind and the radix digits used to find the K-th key:
// (shift, width) of each pass, most significant first.
// Kernel entry: the programmatic-dependent-launch wait (with the next grid
// released first when it waits for this one itself), then the counter that
// this launch clears for later kernels.
__device__ __forceinline__ void topk_begin(const TopkArgs& a) {
  if (a.early_release) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
  } else {
    pdl_begin();
  }
  if (a.zero_word != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *a.zero_word = 0;
}

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

  extern __shared__ uint32_t s_ent[];          // [d], then the staged list [k], then hist16
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

  topk_begin(a);
  if (row >= a.T) {
    // zeroing CTAs: clear the next kernel's accumulators, nothing else
    if (a.zero != nullptr) {
      const size_t nthr = (size_t)a.zero_ctas * NT;
      const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (size_t i = (size_t)(row - a.T) * NT + tid; i < a.zero_n / 4; i += nthr)
        reinterpret_cast<float4*>(a.zero)[i] = z;
    }
    return;
  }
  // dynamic layout (word offsets rounded to 4 so that hist16 is 16-byte aligned)
  uint32_t* s_stg = s_ent + ((d + 3) & ~3);      // [k] when a.stage
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
  } else if (KIND == TK_BF16 && NT == 1024 && a.hist16) {
    // One pass over the whole 15-bit |x| key: 32768 bins kept as packed
    // 16-bit counters (a bin counts at most d < 65536 entries, so the low
    // half never carries into the high half).
    uint32_t* h16 = s_stg + (a.stage ? ((k + 3) & ~3) : 0);
    for (int j = tid; j < 4096; j += NT) reinterpret_cast<uint4*>(h16)[j] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int i = tid; i < d; i += NT) {
      const uint32_t key = s_ent[i] & 0x7fffu;
      atomicAdd(&h16[key >> 1], 1u << ((key & 1u) * 16u));
    }
    __syncthreads();
    if (tid == 0) s_sel[0] = 0xffffffffu;
    // thread j sums bins [32768 - 32 (j+1), 32768 - 32 j): largest keys first
    uint32_t local = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = reinterpret_cast<const uint4*>(h16)[4095 - 4 * tid - q];
      local += (v.x & 0xffffu) + (v.x >> 16) + (v.y & 0xffffu) + (v.y >> 16) + (v.z & 0xffffu) +
               (v.z >> 16) + (v.w & 0xffffu) + (v.w >> 16);
    }
    uint32_t excl, unused_e, tot, unused_t;
    block_scan2<NT>(local, 0u, s_scan[sbuf], excl, unused_e, tot, unused_t);
    sbuf ^= 1;
    remaining = k;
    if ((int)excl < remaining && remaining <= (int)(excl + local)) {
      int run = (int)excl;
      const int top = 32767 - 32 * tid;
      for (int b = 0; b < 32; ++b) {
        const int bin = top - b;
        const int c = (int)((h16[bin >> 1] >> ((bin & 1) * 16)) & 0xffffu);
        if (run + c >= remaining) {
          s_sel[0] = (uint32_t)bin;
          s_sel[1] = (uint32_t)run;
          s_sel[2] = (uint32_t)c;
          break;
        }
        run += c;
      }
    }
    __syncthreads();
    const uint32_t digit = s_sel[0];
    shift = 0;
    if (digit == 0xffffffffu) {                     // counts inconsistent: report
      if (tid == 0) dev_fail(a.status, DEV_CHECK, 1, (uint32_t)row);
      P = 0xffffffffu;
    } else {
      remaining -= (int)s_sel[1];
      P = digit;
    }
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
  const bool stage_list = list_direct && a.stage;            // list positions < list count <= k
  const bool stage_idx = !list_direct && a.stage && a.idx;   // idx positions < k
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
        if (stage_idx) {
          s_stg[pos] = (uint32_t)i;
        } else {
          const size_t o = (size_t)row * (size_t)k + (size_t)pos;
          if (a.idx) a.idx[o] = i;
          if (a.val) {
            if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.val)[o] = ent;
            else if constexpr (KIND == TK_BF16) reinterpret_cast<uint16_t*>(a.val)[o] = (uint16_t)ent;
          }
        }
      } else {
        dev_fail(a.status, DEV_CHECK, 2, (uint32_t)row);   // inconsistent select
      }
      if (list_direct && key != 0u) {
        if (stage_list) {
          s_stg[nzb] = (uint32_t)i;
        } else {
          a.list[nzb] = i;
          if constexpr (QUANT) {
            if (a.list_q) a.list_q[nzb] = (int8_t)(ent >> 8);
          } else {
            if (a.list_val) a.list_val[nzb] = raw_to_f32<KIND>(ent);
          }
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
  // staged list / idx: coalesced copy-out (kept entries keep their bits in s_ent)
  if (stage_list) {
    const int tot_gt = (int)(t_ge & 0xffffu), tot_eq = (int)(t_ge >> 16);
    const int cnt = min(k, tot_gt + (P != 0u ? min(tot_eq, remaining) : (int)t_eqnz));
    for (int j = tid; j < cnt; j += NT) {
      const int i = (int)s_stg[j];
      const uint32_t ent = s_ent[i];
      a.list[j] = i;
      if constexpr (QUANT) {
        if (a.list_q) a.list_q[j] = (int8_t)(ent >> 8);
      } else {
        if (a.list_val) a.list_val[j] = raw_to_f32<KIND>(ent);
      }
    }
  }
  if (stage_idx) {
    const int tot_gt = (int)(t_ge & 0xffffu), tot_eq = (int)(t_ge >> 16);
    const int nsel = min(k, tot_gt + min(tot_eq, remaining));
    for (int j = tid; j < nsel; j += NT) {
      const int i = (int)s_stg[j];
      const uint32_t ent = s_ent[i];
      const size_t o = (size_t)row * (size_t)k + (size_t)j;
      a.idx[o] = i;
      if (a.val) {
        if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.val)[o] = ent;
        else if constexpr (KIND == TK_BF16) reinterpret_cast<uint16_t*>(a.val)[o] = (uint16_t)ent;
      }
    }
  }
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

// ---- register-resident variant (rows of up to 16 K elements) -------------
// Each thread keeps EPT elements of the row in registers, element j*NT + tid
// in slot j, so loads and stores of a slot are coalesced and ballots over a
// slot follow index order.  Radix digits are 8 bits (256 bins, scanned by one
// warp).  Compaction: one ballot per slot gives each warp its counts of
// entries above / at the threshold; one warp turns the (slot, warp) table into
// exclusive prefixes, and every kept entry then knows its final position from
// the prefix plus its rank in the ballot: no per-element shared-memory traffic
// and three barriers for the whole compaction.
template <int KIND> struct RegKeys;
template <> struct RegKeys<TK_F32> {
  static constexpr int kPasses = 4;
  __device__ static constexpr int shift(int p) { return p == 0 ? 23 : (p == 1 ? 15 : (p == 2 ? 7 : 0)); }
  __device__ static constexpr int width(int p) { return p == 3 ? 7 : 8; }
};
template <> struct RegKeys<TK_BF16> {
  static constexpr int kPasses = 2;
  __device__ static constexpr int shift(int p) { return p == 0 ? 7 : 0; }
  __device__ static constexpr int width(int p) { return p == 0 ? 8 : 7; }
};
struct RegQuantKeys {
  static constexpr int kPasses = 1;
  __device__ static constexpr int shift(int) { return 0; }
  __device__ static constexpr int width(int) { return 8; }
};
template <> struct RegKeys<TK_QUANT_F32> : RegQuantKeys {};
template <> struct RegKeys<TK_QUANT_BF16> : RegQuantKeys {};

// K-th largest key of the row held in registers: after this an entry is kept
// iff (key >> shift) > P, or it equals P and fewer than `remaining` equal
// entries precede it.  Each radix pass: a 256-bin shared-memory histogram,
// one warp scans it (largest digits first) and publishes the digit.  `hist`
// holds NP cleared histograms, `sel` three words.
// Element j of a thread is row entry j*NT + tid (CONTIG false) or tid*EPT + j
// (CONTIG true).  `tied` returns how many entries equal the threshold key
// when that is known to be at most `remaining` (all of them kept), else a
// larger value.
template <int KIND, int NT, int EPT, bool CONTIG = false>
__device__ __forceinline__ void reg_select(const uint32_t (&ent)[EPT], int d, int k, int nnz,
                                           int (*hist)[256], uint32_t* sel, DevStatus* status,
                                           int row, uint32_t& P, int& shift, int& remaining,
                                           int* tied = nullptr) {
  using RK = RegKeys<KIND>;
  constexpr uint32_t MASK = KeyTraits<KIND>::kMask;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tied) *tied = 0x7fffffff;
  if (k <= 0) {
    P = 0xffffffffu; shift = 31; remaining = 0;        // nothing is kept
    if (tied) *tied = 0;
    return;
  }
  if (k >= d) {
    P = 0u; shift = 31; remaining = d;                 // every key >> 31 == 0: all kept
    if (tied) *tied = d;
    return;
  }
  if (nnz <= k) {
    // at most K nonzero entries: all of them, plus the lowest-index zeros
    P = 0u; shift = 0; remaining = k - nnz;
    return;
  }
  uint32_t prefix = 0;
  remaining = k;
  shift = 0;
#pragma unroll 1
  for (int p = 0; p < RK::kPasses; ++p) {
    const int sh = RK::shift(p);
    const int nb = 1 << RK::width(p);
    const int hi = sh + RK::width(p);
    const uint32_t himask = hi >= 32 ? 0u : (0xffffffffu << hi);
    int* h = hist[p];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const uint32_t key = ent[j] & MASK;
      const int e = CONTIG ? tid * EPT + j : j * NT + tid;
      if (e < d && ((key ^ prefix) & himask) == 0u)
        atomicAdd(&h[(key >> sh) & (uint32_t)(nb - 1)], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l: bins [nb - (l+1) bpl, nb - l bpl), largest digits first
      const int bpl = nb / 32;
      const int top = nb - 1 - lane * bpl;
      int cnt[8];
      int local = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        cnt[b] = b < bpl ? h[top - b] : 0;
        local += cnt[b];
      }
      int inc = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += v;
      }
      const int excl = inc - local;
      const bool mine = excl < remaining && remaining <= inc;
      if (__ballot_sync(kFull, mine) == 0u && lane == 0) sel[0] = 0xffffffffu;
      if (mine) {
        int run = excl;
        bool done = false;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (!done && b < bpl) {
            if (run + cnt[b] >= remaining) {
              sel[0] = (uint32_t)(top - b);
              sel[1] = (uint32_t)run;
              sel[2] = (uint32_t)cnt[b];
              done = true;
            } else {
              run += cnt[b];
            }
          }
        }
      }
    }
    __syncthreads();
    const uint32_t digit = sel[0];
    if (digit == 0xffffffffu) {                        // counts inconsistent: report, keep nothing
      if (tid == 0) dev_fail(status, DEV_CHECK, 1, (uint32_t)row);
      P = 0xffffffffu; shift = 0; remaining = 0;
      return;
    }
    remaining -= (int)sel[1];
    prefix |= digit << sh;
    shift = sh;
    if ((int)sel[2] == remaining) {                    // the whole digit is kept
      if (tied) *tied = remaining;
      break;
    }
    if (p == RK::kPasses - 1 && tied) *tied = (int)sel[2];   // entries equal to the full key
    // every thread has read sel before the next pass's first barrier
  }
  P = prefix >> shift;
}

// One token row, list outputs only (the projection path): the kept nonzero
// entries in index order with their values, and their count.  An entry is in
// the list iff it is kept and nonzero, which is
//   key != 0                           when P == 0 (every nonzero is kept), else
//   c > P, or c == P among the first `remaining` such entries (c = key >> shift).
template <int KIND, int NT, int EPT>
__global__ void __launch_bounds__(NT) topk_list_kernel(TopkArgs a) {
  constexpr int NW = NT / 32;
  constexpr int NP = RegKeys<KIND>::kPasses;
  constexpr int E = EPT * NW;
  constexpr uint32_t MASK = KeyTraits<KIND>::kMask;
  constexpr bool QUANT = (KIND == TK_QUANT_F32 || KIND == TK_QUANT_BF16);

  __shared__ int s_hist[NP][256];
  __shared__ uint32_t s_cnt[E];                     // definite | ties << 16 per (slot, warp)
  __shared__ uint32_t s_wred[NW];
  __shared__ uint32_t s_wnnz[NW];
  __shared__ uint32_t s_tot;
  __shared__ uint32_t s_sel[3];

  const int d = a.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;

  topk_begin(a);
  if constexpr (!QUANT) {
    if (a.nz_bits != nullptr) {
      // The producer left a bitmask of the row's nonzero entries (d <= 32 NT,
      // one word per thread).  With at most K nonzeros the list is exactly the
      // nonzeros in index order, and every CTA of the grid writes its NT
      // entries at positions given by a prefix over the bitmask.  Otherwise
      // CTA 0 goes on with the full selection below.
      __shared__ uint32_t s_word[NT];
      __shared__ uint32_t s_wpre[NT];
      __shared__ uint32_t s_scan[2 * (NW + 1)];
      __shared__ int s_last;
      const int nwords = (d + 31) >> 5;
      const uint32_t bits = tid < nwords ? __ldcg(a.nz_bits + tid) : 0u;
      const int e = (int)blockIdx.x * NT + tid;
      const uint32_t raw = e < d ? load_raw<KIND>(a.x, e) : 0u;
      uint32_t excl, unused_e, tot, unused_t;
      block_scan2<NT>((uint32_t)__popc(bits), 0u, s_scan, excl, unused_e, tot, unused_t);
      s_word[tid] = bits;
      s_wpre[tid] = excl;
      __syncthreads();
      if (tid == 0) s_last = (atomicAdd(a.ticket, 1) == (int)gridDim.x - 1);
      __syncthreads();
      if (s_last) {                                  // every CTA has read the bitmask
        if (tid < nwords) a.nz_bits[tid] = 0u;
        if (tid == 0) *a.ticket = 0;
      }
      if ((int)tot <= a.k) {
        if (blockIdx.x == 0 && tid == 0) *a.list_count = (int)tot;
        if (e < d) {
          const uint32_t wb = s_word[e >> 5];
          if ((wb >> lane) & 1u) {
            const int pos = (int)s_wpre[e >> 5] + __popc(wb & lt);
            a.list[pos] = e;
            a.list_val[pos] = raw_to_f32<KIND>(raw);
          }
        }
        return;
      }
      if (blockIdx.x != 0) return;
      __syncthreads();                               // s_scan is reused below
    }
  }
  if (blockIdx.x >= 1) {
    if (a.zero != nullptr) {
      const size_t nthr = (size_t)a.zero_ctas * NT;
      const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (size_t i = (size_t)(blockIdx.x - 1) * NT + tid; i < a.zero_n / 4; i += nthr)
        reinterpret_cast<float4*>(a.zero)[i] = z;
    }
    return;
  }
  for (int j = tid; j < NP * 256; j += NT) (&s_hist[0][0])[j] = 0;

  uint32_t ent[EPT];
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = j * NT + tid;
    ent[j] = e < d ? load_raw<KIND>(a.x, e) : 0u;
  }
  if constexpr (QUANT) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j) m = max(m, raw_abs_f32bits<KIND>(ent[j]));   // padding is 0
    m = __reduce_max_sync(kFull, m);
    if (lane == 0) s_wred[warp] = m;
    __syncthreads();
    const uint32_t amax_bits = __reduce_max_sync(kFull, lane < NW ? s_wred[lane] : 0u);
    const float gamma = __fadd_rn(__uint_as_float(amax_bits), a.eps);
    const float scale = __fdiv_rn(127.0f, gamma);
    if (tid == 0 && a.gamma) a.gamma[0] = gamma;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      int qi = __float2int_rn(__fmul_rn(raw_to_f32<KIND>(ent[j]), scale));
      qi = min(127, max(-127, qi));
      const uint32_t mag = (uint32_t)(qi < 0 ? -qi : qi);
      ent[j] = j * NT + tid < d ? (mag | ((uint32_t)(uint8_t)(int8_t)qi << 8)) : 0u;
    }
  }
  uint32_t my_nnz = 0;
#pragma unroll
  for (int j = 0; j < EPT; ++j) my_nnz += ((ent[j] & MASK) != 0u);   // padding is 0
  my_nnz = __reduce_add_sync(kFull, my_nnz);
  if (lane == 0) s_wnnz[warp] = my_nnz;
  __syncthreads();
  const int nnz = (int)__reduce_add_sync(kFull, lane < NW ? s_wnnz[lane] : 0u);

  uint32_t P;
  int shift, remaining;
  reg_select<KIND, NT, EPT>(ent, d, a.k, nnz, s_hist, s_sel, a.status, 0, P, shift, remaining);
  const bool ties = P != 0u;

#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const uint32_t key = ent[j] & MASK;              // padding: key 0, never listed
    const uint32_t c = key >> shift;
    const uint32_t bd = __ballot_sync(kFull, ties ? c > P : key != 0u);
    const uint32_t bt = __ballot_sync(kFull, ties && c == P);
    if (lane == j) s_cnt[j * NW + warp] = (uint32_t)__popc(bd) | ((uint32_t)__popc(bt) << 16);
  }
  __syncthreads();
  if (warp == 0) {
    constexpr int CH = (E + 31) / 32;
    const int b0 = min(lane * CH, E), b1 = min(b0 + CH, E);
    uint32_t sg = 0;
    for (int i = b0; i < b1; ++i) sg += s_cnt[i];
    uint32_t ig = sg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(kFull, ig, o);
      if (lane >= o) ig += v;
    }
    uint32_t eg = ig - sg;
    for (int i = b0; i < b1; ++i) {
      const uint32_t c = s_cnt[i];
      s_cnt[i] = eg;
      eg += c;
    }
    if (lane == 31) s_tot = ig;
  }
  __syncthreads();
  if (tid == 0) *a.list_count = (int)(s_tot & 0xffffu) + min((int)(s_tot >> 16), remaining);
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const uint32_t key = ent[j] & MASK;
    const uint32_t c = key >> shift;
    const bool def = ties ? c > P : key != 0u;
    const bool tie = ties && c == P;
    const uint32_t bd = __ballot_sync(kFull, def);
    const uint32_t bt = __ballot_sync(kFull, tie);
    const uint32_t pre = s_cnt[j * NW + warp];
    const int def_b = (int)(pre & 0xffffu) + __popc(bd & lt);
    const int tie_b = (int)(pre >> 16) + __popc(bt & lt);
    if (def || (tie && tie_b < remaining)) {
      const int pos = def_b + min(tie_b, remaining);
      a.list[pos] = j * NT + tid;
      if constexpr (QUANT) a.list_q[pos] = (int8_t)(ent[j] >> 8);
      else a.list_val[pos] = raw_to_f32<KIND>(ent[j]);
    }
  }
}

// ---- Block Q-Sparse helpers (a block of rows shares one selection) ------------
constexpr int kMaxBlock = 64;
constexpr int kMaxBlockRow = 1024 * 16;          // features of a block-selected row

// int8 code of one input value (the quantizer of the quant kinds)
template <int KIND>
__device__ __forceinline__ int quant_code(uint32_t raw, float scale) {
  const int qi = __float2int_rn(__fmul_rn(raw_to_f32<KIND>(raw), scale));
  return min(127, max(-127, qi));
}

// Raw element e of a 16-byte vector q (VW elements of the input type).
template <int KIND, int VW>
__device__ __forceinline__ uint32_t vec_elem(const uint4& q, int e) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  if constexpr (KIND == TK_F32 || KIND == TK_QUANT_F32) return w[e];
  else return (w[e >> 1] >> (16 * (e & 1))) & 0xffffu;
}

// Elements per 16-byte vector of the input type.
template <int KIND> constexpr int vec_width() {
  return (KIND == TK_F32 || KIND == TK_QUANT_F32) ? 4 : 8;
}

// Vectors of the row and the vector width the block kernels use: 16-byte
// vectors when the row pitch keeps them aligned, else single elements.
template <int KIND>
__device__ __forceinline__ bool block_vectorized(int d) { return (d % vec_width<KIND>()) == 0; }

// Quant kinds: 127 / gamma_t of every row of the block (one warp per row, its
// lanes reading 16-byte vectors) into s_bscale; gamma of row `own` to a.gamma.
template <int KIND, int NT>
__device__ void block_scales(const TopkArgs& a, int t0, int t1, int own, float* s_bscale) {
  constexpr int V = vec_width<KIND>();
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = a.d;
  const bool vec = block_vectorized<KIND>(d);
  for (int t = t0 + warp; t < t1; t += NW) {
    uint32_t m = 0;
    if (vec) {
      const uint4* row = reinterpret_cast<const uint4*>(
          reinterpret_cast<const unsigned char*>(a.x) + (size_t)t * d * (V == 4 ? 4 : 2));
#pragma unroll 4
      for (int v = lane; v < d / V; v += 32) {
        const uint4 q = __ldg(row + v);
#pragma unroll
        for (int e = 0; e < V; ++e) m = max(m, raw_abs_f32bits<KIND>(vec_elem<KIND, V>(q, e)));
      }
    } else {
      for (int e = lane; e < d; e += 32)
        m = max(m, raw_abs_f32bits<KIND>(load_raw<KIND>(a.x, (size_t)t * d + e)));
    }
    m = __reduce_max_sync(kFull, m);
    if (lane == 0) {
      const float gamma = __fadd_rn(__uint_as_float(m), a.eps);
      if (a.gamma && t == own) a.gamma[t] = gamma;
      s_bscale[t - t0] = __fdiv_rn(127.0f, gamma);
    }
  }
}

// s_key[e] = the block key of feature e: the largest |x| bits (f32 / bf16) or
// the largest |q| (quant kinds) over rows [t0, t1).  Threads take 16-byte
// vectors of the row; when the row has fewer vectors than threads, groups of
// threads take different rows and combine with a shared-memory maximum.
template <int KIND, int NT>
__device__ void block_keys(const TopkArgs& a, int t0, int t1, uint32_t* s_key, const float* s_bscale) {
  constexpr bool QUANT = (KIND == TK_QUANT_F32 || KIND == TK_QUANT_BF16);
  constexpr uint32_t MASK = KeyTraits<KIND>::kMask;
  constexpr int V = vec_width<KIND>();
  const int tid = threadIdx.x;
  const int d = a.d;
  for (int e = tid; e < d; e += NT) s_key[e] = 0u;
  __syncthreads();
  auto key_of = [&](uint32_t raw, int t) -> uint32_t {
    if constexpr (QUANT) {
      const int qi = quant_code<KIND>(raw, s_bscale[t - t0]);
      return (uint32_t)(qi < 0 ? -qi : qi);
    } else {
      return raw & MASK;
    }
  };
  if (block_vectorized<KIND>(d)) {
    const int nvec = d / V;
    const int groups = nvec >= NT ? 1 : min(NT / nvec, t1 - t0);
    const int g = tid / (nvec >= NT ? NT : nvec);
    const int v0 = tid - g * (nvec >= NT ? NT : nvec);
    if (g < groups) {
      for (int v = v0; v < nvec; v += (nvec >= NT ? NT : nvec)) {
        uint32_t k[V];
#pragma unroll
        for (int e = 0; e < V; ++e) k[e] = 0u;
#pragma unroll 4
        for (int t = t0 + g; t < t1; t += groups) {
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(
              reinterpret_cast<const unsigned char*>(a.x) + ((size_t)t * d + (size_t)v * V) * (V == 4 ? 4 : 2)));
#pragma unroll
          for (int e = 0; e < V; ++e) k[e] = max(k[e], key_of(vec_elem<KIND, V>(q, e), t));
        }
#pragma unroll
        for (int e = 0; e < V; ++e)
          if (k[e] != 0u) atomicMax(&s_key[v * V + e], k[e]);
      }
    }
  } else {
    for (int e = tid; e < d; e += NT) {
      uint32_t k = 0;
      for (int t = t0; t < t1; ++t) k = max(k, key_of(load_raw<KIND>(a.x, (size_t)t * d + e), t));
      s_key[e] = k;
    }
  }
  __syncthreads();
}

// The dense outputs of rows [t0, t1) (mask, X_sparse, the masked copies, the
// codes) in one flattened (row, vector) loop, from the selection bitmask s_sel
// (bit e = feature e kept); s_bscale[t - t0] = 127 / gamma_t (quant kinds).
template <int KIND, int NT>
__device__ void block_outputs(const TopkArgs& a, int t0, int t1, const uint32_t* s_sel,
                              const float* s_bscale) {
  constexpr bool QUANT = (KIND == TK_QUANT_F32 || KIND == TK_QUANT_BF16);
  constexpr int V = vec_width<KIND>();
  const int tid = threadIdx.x;
  const int d = a.d;
  const bool dense = a.mask || a.xs || a.xsf || a.xq || a.q_full;
  auto one = [&](int t, int e, uint32_t raw) {
    const size_t o = (size_t)t * d + e;
    const bool sel = (s_sel[e >> 5] >> (e & 31)) & 1u;
    if (a.mask) a.mask[o] = sel ? 1 : 0;
    if constexpr (QUANT) {
      const int qi = quant_code<KIND>(raw, s_bscale[t - t0]);
      if (a.q_full) a.q_full[o] = (int8_t)qi;
      if (a.xq) a.xq[o] = sel ? (int8_t)qi : (int8_t)0;
    } else {
      const uint32_t v = sel ? raw : 0u;
      if (a.xsf) a.xsf[o] = raw_to_f32<KIND>(v);
      if (a.xs) {
        if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.xs)[o] = v;
        else reinterpret_cast<uint16_t*>(a.xs)[o] = (uint16_t)v;
      }
    }
  };
  if (dense) {
    if (block_vectorized<KIND>(d)) {
      const int nvec = d / V;
      const int total = (t1 - t0) * nvec;
#pragma unroll 2
      for (int i = tid; i < total; i += NT) {
        const int t = t0 + i / nvec, v = i - (i / nvec) * nvec;
        const size_t o = (size_t)t * d + (size_t)v * V;
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(
            reinterpret_cast<const unsigned char*>(a.x) + o * (V == 4 ? 4 : 2)));
        const uint32_t bits = (s_sel[(v * V) >> 5] >> ((v * V) & 31)) & ((1u << V) - 1u);
        // V elements at once: vector stores of every output (offsets are
        // multiples of V, so byte outputs are V-byte aligned)
        uint32_t m[V / 4] = {};                       // mask bytes
        uint32_t c8[V / 4] = {}, z8[V / 4] = {};      // codes, masked codes
        uint32_t w[4] = {};                           // masked raw values (input layout)
        float f[V];
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const bool sel = (bits >> e) & 1u;
          const uint32_t raw = vec_elem<KIND, V>(q, e);
          m[e >> 2] |= (sel ? 1u : 0u) << (8 * (e & 3));
          if constexpr (QUANT) {
            const uint32_t qb = (uint32_t)(uint8_t)(int8_t)quant_code<KIND>(raw, s_bscale[t - t0]);
            c8[e >> 2] |= qb << (8 * (e & 3));
            if (sel) z8[e >> 2] |= qb << (8 * (e & 3));
          } else {
            const uint32_t vm = sel ? raw : 0u;
            f[e] = raw_to_f32<KIND>(vm);
            if constexpr (V == 4) w[e] = vm;
            else w[e >> 1] |= vm << (16 * (e & 1));
          }
        }
        if (a.mask) {
          if constexpr (V == 8) *reinterpret_cast<uint2*>(a.mask + o) = make_uint2(m[0], m[1]);
          else *reinterpret_cast<uint32_t*>(a.mask + o) = m[0];
        }
        if constexpr (QUANT) {
          if constexpr (V == 8) {
            if (a.q_full) *reinterpret_cast<uint2*>(a.q_full + o) = make_uint2(c8[0], c8[1]);
            if (a.xq) *reinterpret_cast<uint2*>(a.xq + o) = make_uint2(z8[0], z8[1]);
          } else {
            if (a.q_full) *reinterpret_cast<uint32_t*>(a.q_full + o) = c8[0];
            if (a.xq) *reinterpret_cast<uint32_t*>(a.xq + o) = z8[0];
          }
        } else {
          if (a.xsf) {
#pragma unroll
            for (int c = 0; c < V / 4; ++c)
              reinterpret_cast<float4*>(a.xsf + o)[c] = make_float4(f[4 * c], f[4 * c + 1], f[4 * c + 2], f[4 * c + 3]);
          }
          if (a.xs)
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(a.xs) + o * (V == 4 ? 4 : 2)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    } else {
      const int total = (t1 - t0) * d;
      for (int i = tid; i < total; i += NT) {
        const int t = t0 + i / d, e = i - (i / d) * d;
        one(t, e, load_raw<KIND>(a.x, (size_t)t * d + e));
      }
    }
  }
}

template <int KIND, int NT, int EPT, bool BLOCK>
__global__ void __launch_bounds__(NT) topk_reg_kernel(TopkArgs a) {
  using RK = RegKeys<KIND>;
  constexpr int NW = NT / 32;
  constexpr int NP = RK::kPasses;
  constexpr int E = EPT * NW;                       // (slot, warp) table size
  constexpr uint32_t MASK = KeyTraits<KIND>::kMask;
  constexpr bool QUANT = (KIND == TK_QUANT_F32 || KIND == TK_QUANT_BF16);

  __shared__ int s_hist[NP][256];
  __shared__ uint32_t s_cnt[E];                     // gt | eq << 16 per (slot, warp), then prefixes
  __shared__ uint32_t s_cnz[E];                     // eq with a nonzero key, then prefixes
  __shared__ uint32_t s_wred[NW];
  __shared__ uint32_t s_wnnz[NW];
  __shared__ uint32_t s_tot[2];
  __shared__ uint32_t s_sel[3];
  __shared__ uint32_t s_scan[2 * (NW + 1)];
  __shared__ int s_last;
  __shared__ float s_bscale[BLOCK ? kMaxBlock : 1];           // Block Q-Sparse (quant): 127 / gamma_t
  __shared__ uint32_t s_bsel[BLOCK ? kMaxBlockRow / 32 : 1]; // Block Q-Sparse: kept features
  extern __shared__ uint32_t s_bkey[];                       // Block Q-Sparse: [d] block keys

  // One CTA per token row.  Block Q-Sparse (a.block > 1): the rows of a block
  // of a.block consecutive tokens share one selection, which each of the
  // block's CTAs computes (the same result: the same inputs and order) and
  // uses for its own row's outputs.
  const int row = blockIdx.x;
  const int d = a.d;
  const int k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t rbase = (size_t)row * (size_t)d;
  const uint32_t lt = (1u << lane) - 1u;
  const int blk = BLOCK ? a.block : 1;   // the per-row instantiation keeps no block code
  const int nsel = a.T;                            // row CTAs
  const int t0 = (row / blk) * blk, t1 = min(a.T, t0 + blk);   // this row's block

  topk_begin(a);
  if (row >= nsel) {
    if (a.zero != nullptr) {
      const size_t nthr = (size_t)a.zero_ctas * NT;
      const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (size_t i = (size_t)(row - nsel) * NT + tid; i < a.zero_n / 4; i += nthr)
        reinterpret_cast<float4*>(a.zero)[i] = z;
    }
    return;
  }
  for (int j = tid; j < NP * 256; j += NT) (&s_hist[0][0])[j] = 0;

  // ---- 1. entries in registers ---------------------------------------------
  uint32_t ent[EPT];
  if constexpr (BLOCK) {
    // Block Q-Sparse: the key of feature e is the block magnitude, the
    // largest |x| (or |q|) over the block's rows; values are read again below
    if constexpr (QUANT) {
      block_scales<KIND, NT>(a, t0, t1, row, s_bscale);
      __syncthreads();
    }
    block_keys<KIND, NT>(a, t0, t1, s_bkey, s_bscale);
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * NT + tid;
      ent[j] = e < d ? s_bkey[e] : 0u;
    }
  } else {
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const int e = j * NT + tid;
    ent[j] = e < d ? load_raw<KIND>(a.x, rbase + e) : 0u;
  }
  }
  if (QUANT && !BLOCK) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j)
      if (j * NT + tid < d) m = max(m, raw_abs_f32bits<KIND>(ent[j]));
    m = __reduce_max_sync(kFull, m);
    if (lane == 0) s_wred[warp] = m;
    __syncthreads();
    const uint32_t amax_bits = __reduce_max_sync(kFull, lane < NW ? s_wred[lane] : 0u);
    const float gamma = __fadd_rn(__uint_as_float(amax_bits), a.eps);
    const float scale = __fdiv_rn(127.0f, gamma);
    if (tid == 0 && a.gamma) a.gamma[row] = gamma;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * NT + tid;
      if (e < d) {
        int qi = __float2int_rn(__fmul_rn(raw_to_f32<KIND>(ent[j]), scale));
        qi = min(127, max(-127, qi));
        const uint32_t mag = (uint32_t)(qi < 0 ? -qi : qi);
        ent[j] = mag | ((uint32_t)(uint8_t)(int8_t)qi << 8);
        if (a.q_full) a.q_full[rbase + e] = (int8_t)qi;
      }
    }
  }
  uint32_t my_nnz = 0;
#pragma unroll
  for (int j = 0; j < EPT; ++j) my_nnz += (j * NT + tid < d && (ent[j] & MASK) != 0u);
  my_nnz = __reduce_add_sync(kFull, my_nnz);
  if (lane == 0) s_wnnz[warp] = my_nnz;
  __syncthreads();                                  // also orders the histogram clear
  const int nnz = (int)__reduce_add_sync(kFull, lane < NW ? s_wnnz[lane] : 0u);

  // ---- 2. the K-th largest key ----------------------------------------------
  uint32_t P;
  int shift;
  int remaining;
  reg_select<KIND, NT, EPT>(ent, d, k, nnz, s_hist, s_sel, a.status, row, P, shift, remaining);

  // ---- 3. compaction in index order ------------------------------------------
  const bool list_direct = (a.list != nullptr) && (a.T == 1);
  const bool want_union = (a.list != nullptr) && (a.T > 1);
  // With at most K nonzero entries every nonzero entry is kept; when the only
  // outputs are the dense values and the union of the kept nonzeros (the
  // several-token projection path: h has at most K_h nonzeros per token for
  // the squared-ReLU GLU), nothing needs a position, and the ranked
  // compaction below (ballots, prefix scans and position arithmetic for every
  // entry, on one SM per row) is skipped.  (block-uniform)
  const bool all_nz_kept = !BLOCK && !QUANT && nnz <= k && !list_direct && a.idx == nullptr &&
                           a.val == nullptr && a.mask == nullptr && a.xs == nullptr;
  if (all_nz_kept) {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * NT + tid;
      const bool valid = e < d;
      if (valid && a.xsf) a.xsf[rbase + e] = raw_to_f32<KIND>(ent[j]);
      if (want_union) {
        const uint32_t b = __ballot_sync(kFull, valid && (ent[j] & MASK) != 0u);
        if (lane == 0 && b != 0u) atomicOr(a.union_bits + (j * NT + warp * 32) / 32, b);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const bool valid = j * NT + tid < d;
      const uint32_t key = ent[j] & MASK;
      const uint32_t c = key >> shift;
      const bool eq = valid && c == P;
      const uint32_t bg = __ballot_sync(kFull, valid && c > P);
      const uint32_t be = __ballot_sync(kFull, eq);
      const uint32_t bz = __ballot_sync(kFull, eq && key != 0u);
      if (lane == j) {
        s_cnt[j * NW + warp] = (uint32_t)__popc(bg) | ((uint32_t)__popc(be) << 16);
        s_cnz[j * NW + warp] = (uint32_t)__popc(bz);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // exclusive prefixes over the (slot, warp) table, warps fastest: index order
      constexpr int CH = (E + 31) / 32;
      const int b0 = min(lane * CH, E), b1 = min(b0 + CH, E);
      uint32_t sg = 0, sz = 0;
      for (int i = b0; i < b1; ++i) { sg += s_cnt[i]; sz += s_cnz[i]; }
      uint32_t ig = sg, iz = sz;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t vg = __shfl_up_sync(kFull, ig, o);
        const uint32_t vz = __shfl_up_sync(kFull, iz, o);
        if (lane >= o) { ig += vg; iz += vz; }
      }
      uint32_t eg = ig - sg, ez = iz - sz;
      for (int i = b0; i < b1; ++i) {
        const uint32_t cg = s_cnt[i], cz = s_cnz[i];
        s_cnt[i] = eg; s_cnz[i] = ez;
        eg += cg; ez += cz;
      }
      if (lane == 31) { s_tot[0] = ig; s_tot[1] = iz; }
    }
    __syncthreads();
    const int tot_gt = (int)(s_tot[0] & 0xffffu), tot_eq = (int)(s_tot[0] >> 16);
    const int tot_eqnz = (int)s_tot[1];
    if (list_direct && tid == 0) *a.list_count = tot_gt + (P != 0u ? min(tot_eq, remaining) : tot_eqnz);
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = j * NT + tid;
      const bool valid = e < d;
      const uint32_t key = ent[j] & MASK;
      const uint32_t c = key >> shift;
      const bool gt = valid && c > P;
      const bool eq = valid && c == P;
      const uint32_t bg = __ballot_sync(kFull, gt);
      const uint32_t be = __ballot_sync(kFull, eq);
      const uint32_t bz = __ballot_sync(kFull, eq && key != 0u);
      const uint32_t pre = s_cnt[j * NW + warp];
      const int gt_b = (int)(pre & 0xffffu) + __popc(bg & lt);
      const int eq_b = (int)(pre >> 16) + __popc(be & lt);
      const int eqnz_b = (int)s_cnz[j * NW + warp] + __popc(bz & lt);
      const bool sel = gt || (eq && eq_b < remaining);
      if constexpr (BLOCK) {
        // Block Q-Sparse: this row's idx / val here, its other outputs after
        // the loop from the selection bitmask
        const uint32_t bs = __ballot_sync(kFull, sel);
        if (lane == 0 && j * NT + warp * 32 < d) s_bsel[(j * NT + warp * 32) >> 5] = bs;
        if (sel) {
          const int pos = gt_b + min(eq_b, remaining);
          if (pos < k) {
            const size_t o = (size_t)row * k + pos;
            if (a.idx) a.idx[o] = e;
            if (a.val) {
              const uint32_t raw = load_raw<KIND>(a.x, (size_t)row * d + e);
              if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.val)[o] = raw;
              else if constexpr (KIND == TK_BF16) reinterpret_cast<uint16_t*>(a.val)[o] = (uint16_t)raw;
            }
          } else {
            dev_fail(a.status, DEV_CHECK, 2, (uint32_t)row);
          }
        }
      } else if (sel) {
        const int pos = gt_b + min(eq_b, remaining);
        if (pos < k) {
          const size_t o = (size_t)row * (size_t)k + (size_t)pos;
          if (a.idx) a.idx[o] = e;
          if (a.val) {
            if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.val)[o] = ent[j];
            else if constexpr (KIND == TK_BF16) reinterpret_cast<uint16_t*>(a.val)[o] = (uint16_t)ent[j];
          }
        } else {
          dev_fail(a.status, DEV_CHECK, 2, (uint32_t)row);
        }
        if (list_direct && key != 0u) {
          const int nzp = gt_b + (P != 0u ? min(eq_b, remaining) : eqnz_b);
          a.list[nzp] = e;
          if constexpr (QUANT) {
            if (a.list_q) a.list_q[nzp] = (int8_t)(ent[j] >> 8);
          } else {
            if (a.list_val) a.list_val[nzp] = raw_to_f32<KIND>(ent[j]);
          }
        }
      }
      if (valid && !BLOCK) {
        const uint32_t v = sel ? ent[j] : 0u;
        if (a.mask) a.mask[rbase + e] = sel ? 1 : 0;
        if constexpr (QUANT) {
          if (a.xq) a.xq[rbase + e] = (int8_t)(v >> 8);
        } else {
          if (a.xsf) a.xsf[rbase + e] = raw_to_f32<KIND>(v);
          if (a.xs) {
            if constexpr (KIND == TK_F32) reinterpret_cast<uint32_t*>(a.xs)[rbase + e] = v;
            else reinterpret_cast<uint16_t*>(a.xs)[rbase + e] = (uint16_t)v;
          }
        }
      }
      if (want_union) {
        const uint32_t b = __ballot_sync(kFull, sel && key != 0u);
        if (lane == 0 && b != 0u) atomicOr(a.union_bits + (j * NT + warp * 32) / 32, b);
      }
    }

  }

  if constexpr (BLOCK) {
    __syncthreads();                                 // s_bsel complete
    block_outputs<KIND, NT>(a, row, row + 1, s_bsel, s_bscale + (row - t0));
  }

  // ---- 4. union of the rows' kept nonzeros (several tokens) ------------------
  // The last row CTA lists the set bits: one word per thread for the prefix
  // (d <= 32 NT here), then one word per warp per step with the ballot rank,
  // so that the 32 entries of a word are stored together.
  if (want_union) {
    __shared__ uint32_t s_uword[NT];
    __shared__ uint32_t s_upre[NT];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(a.ticket, 1) == nsel - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int nwords = (d + 31) / 32;
    const uint32_t bits = tid < nwords ? __ldcg(a.union_bits + tid) : 0u;
    uint32_t e_any, e_unused, t_any, t_unused;
    block_scan2<NT>((uint32_t)__popc(bits), 0u, s_scan, e_any, e_unused, t_any, t_unused);
    s_uword[tid] = bits;
    s_upre[tid] = e_any;
    if (tid < nwords) a.union_bits[tid] = 0u;    // leave the bitmask clean for the next call
    __syncthreads();
    for (int w = warp; w < nwords; w += NW) {
      const uint32_t wb = s_uword[w];
      if ((wb >> lane) & 1u) a.list[s_upre[w] + __popc(wb & lt)] = w * 32 + lane;
    }
    if (tid == 0) {
      *a.list_count = (int)t_any;
      *a.ticket = 0;
    }
  }
}

// Many bf16 rows whose only output is X_sparse (the prefill path): each thread
// owns 16 contiguous entries, loaded and stored as two 16-byte vectors.  Zero
// entries are 0 in X_sparse whether kept or not, so ties need ranking only at
// a nonzero threshold that splits them (a block scan of per-thread counts).
template <int NT>
__global__ void __launch_bounds__(NT) topk_dense_bf16_kernel(TopkArgs a) {
  constexpr int EPT = 16;
  constexpr int NW = NT / 32;
  constexpr int NP = RegKeys<TK_BF16>::kPasses;
  constexpr uint32_t MASK = KeyTraits<TK_BF16>::kMask;
  __shared__ int s_hist[NP][256];
  __shared__ uint32_t s_sel[3];
  __shared__ uint32_t s_wnnz[NW];
  __shared__ uint32_t s_scan[2 * (NW + 1)];

  const int row = blockIdx.x;
  const int d = a.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e0 = tid * EPT;
  const uint16_t* xr = reinterpret_cast<const uint16_t*>(a.x) + (size_t)row * d;
  uint16_t* xsr = reinterpret_cast<uint16_t*>(a.xs) + (size_t)row * d;

  topk_begin(a);
  for (int j = tid; j < NP * 256; j += NT) (&s_hist[0][0])[j] = 0;
  uint32_t ent[EPT];
  if (e0 + EPT <= d) {                               // d % 8 == 0: rows are 16-byte aligned
    const uint4 v0 = ld_stream_v4(xr + e0);
    const uint4 v1 = ld_stream_v4(xr + e0 + 8);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) { ent[2 * q] = w[q] & 0xffffu; ent[2 * q + 1] = w[q] >> 16; }
  } else {
#pragma unroll
    for (int j = 0; j < EPT; ++j) ent[j] = e0 + j < d ? (uint32_t)xr[e0 + j] : 0u;
  }
  uint32_t my_nnz = 0;
#pragma unroll
  for (int j = 0; j < EPT; ++j) my_nnz += ((ent[j] & MASK) != 0u);
  my_nnz = __reduce_add_sync(kFull, my_nnz);
  if (lane == 0) s_wnnz[warp] = my_nnz;
  __syncthreads();
  const int nnz = (int)__reduce_add_sync(kFull, lane < NW ? s_wnnz[lane] : 0u);

  uint32_t P;
  int shift, remaining, tied;
  reg_select<TK_BF16, NT, EPT, true>(ent, d, a.k, nnz, s_hist, s_sel, a.status, row, P, shift,
                                     remaining, &tied);
  // ties at a nonzero threshold that are not all kept: rank them by index
  int eq_b = 0;
  if (P != 0u && remaining < tied) {
    uint32_t my_eq = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j) my_eq += (e0 + j < d && ((ent[j] & MASK) >> shift) == P);
    uint32_t excl, unused_e, tot, unused_t;
    block_scan2<NT>(my_eq, 0u, s_scan, excl, unused_e, tot, unused_t);
    eq_b = (int)excl;
  } else {
    eq_b = -0x40000000;                              // every tie is below `remaining`
  }
  uint32_t out[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) out[q] = 0u;
#pragma unroll
  for (int j = 0; j < EPT; ++j) {
    const uint32_t c = (ent[j] & MASK) >> shift;
    const bool eq = c == P;
    const bool keep = c > P || (eq && eq_b < remaining);
    eq_b += eq;
    if (keep) out[j >> 1] |= ent[j] << (16 * (j & 1));
  }
  if (e0 + EPT <= d) {
    reinterpret_cast<uint4*>(xsr + e0)[0] = make_uint4(out[0], out[1], out[2], out[3]);
    reinterpret_cast<uint4*>(xsr + e0)[1] = make_uint4(out[4], out[5], out[6], out[7]);
  } else {
#pragma unroll
    for (int j = 0; j < EPT; ++j)
      if (e0 + j < d) xsr[e0 + j] = (uint16_t)(out[j >> 1] >> (16 * (j & 1)));
  }
}

// Row CTAs of a launch (Block Q-Sparse included: one CTA per token row).
int selections(const TopkArgs& a) { return a.T; }

bool dense_only_bf16(const TopkArgs& a) {
  return a.block <= 1 && a.kind == TK_BF16 && a.xs != nullptr && a.idx == nullptr && a.val == nullptr &&
         a.mask == nullptr && a.xsf == nullptr && a.xq == nullptr && a.list == nullptr &&
         a.zero == nullptr && a.d <= 256 * 16 && (a.d % 8) == 0 &&
         ((uintptr_t)a.x & 15u) == 0 && ((uintptr_t)a.xs & 15u) == 0;
}

// The list-only kernel serves one token row whose only outputs are the list,
// its values and count (and gamma): the projection path's decode step.
bool list_only(const TopkArgs& a) {
  const bool quant = a.kind == TK_QUANT_F32 || a.kind == TK_QUANT_BF16;
  return a.T == 1 && a.block <= 1 && a.list != nullptr && a.list_count != nullptr && a.idx == nullptr &&
         a.val == nullptr && a.mask == nullptr && a.xs == nullptr && a.xsf == nullptr &&
         a.xq == nullptr && a.q_full == nullptr &&
         (quant ? a.list_q != nullptr : a.list_val != nullptr);
}

template <int KIND, int NT, int EPT>
cudaError_t launch_reg(const TopkArgs& a_in, cudaStream_t s) {
  TopkArgs a = a_in;
  a.stage = 0;
  a.hist16 = 0;
  a.zero_ctas = 0;
  if (a.zero != nullptr && a.zero_n >= 4)
    a.zero_ctas = (int)std::min<size_t>((a.zero_n / 4 + NT - 1) / NT, 32);
  cudaError_t e;
  if (list_only(a) && a.nz_bits != nullptr) {
    if (a.zero != nullptr || NT != 1024 || a.kind == TK_QUANT_F32 || a.kind == TK_QUANT_BF16)
      return cudaErrorInvalidValue;                 // not a configuration the API builds
    a.zero_ctas = 0;
    e = launch_pdl(topk_list_kernel<KIND, NT, EPT>, dim3((a.d + NT - 1) / NT), dim3(NT), (size_t)0, s, a);
  } else if (list_only(a))
    e = launch_pdl(topk_list_kernel<KIND, NT, EPT>, dim3(1 + a.zero_ctas), dim3(NT), (size_t)0, s, a);
  else if (a.block > 1) {
    // block keys in dynamic shared memory: 4 bytes per feature
    static unsigned configured = 0;
    e = ensure_smem_attr(topk_reg_kernel<KIND, NT, EPT, true>, kMaxBlockRow * 4, &configured);
    if (e != cudaSuccess) return e;
    e = launch_pdl(topk_reg_kernel<KIND, NT, EPT, true>, dim3(selections(a) + a.zero_ctas),
                   dim3(NT), (size_t)a.d * 4, s, a);
  }
  else
    e = launch_pdl(topk_reg_kernel<KIND, NT, EPT, false>, dim3(selections(a) + a.zero_ctas),
                   dim3(NT), (size_t)0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Register-resident launch when the row fits (EPT <= 16); false otherwise.
template <int KIND>
bool try_launch_reg(const TopkArgs& a, cudaStream_t s, cudaError_t* err) {
  if (selections(a) >= 2 * kNumSMs) {            // many rows: 256-thread CTAs
    if (KIND == TK_BF16 && dense_only_bf16(a)) {
      *err = launch_pdl(topk_dense_bf16_kernel<256>, dim3(a.T), dim3(256), (size_t)0, s, a);
      if (*err == cudaSuccess) *err = cudaGetLastError();
      return true;
    }
    if (a.d <= 256 * 4) { *err = launch_reg<KIND, 256, 4>(a, s); return true; }
    if (a.d <= 256 * 8) { *err = launch_reg<KIND, 256, 8>(a, s); return true; }
    if (a.d <= 256 * 16) { *err = launch_reg<KIND, 256, 16>(a, s); return true; }
    return false;
  }
  if (a.d <= 1024 * 1) { *err = launch_reg<KIND, 1024, 1>(a, s); return true; }
  if (a.d <= 1024 * 2) { *err = launch_reg<KIND, 1024, 2>(a, s); return true; }
  if (a.d <= 1024 * 4) { *err = launch_reg<KIND, 1024, 4>(a, s); return true; }
  if (a.d <= 1024 * 8) { *err = launch_reg<KIND, 1024, 8>(a, s); return true; }
  if (a.d <= 1024 * 12) { *err = launch_reg<KIND, 1024, 12>(a, s); return true; }
  if (a.d <= 1024 * 16) { *err = launch_reg<KIND, 1024, 16>(a, s); return true; }
  return false;
}

constexpr size_t kTopkSmemMax = 216 * 1024;   // dynamic; the static arrays take ~9 KB
static_assert((size_t)QS_MAX_ROW * 4 <= kTopkSmemMax, "a full row must fit");

template <int KIND, int NT>
cudaError_t launch_kind(const TopkArgs& a_in, cudaStream_t s) {
  TopkArgs a = a_in;
  const bool list_direct = a.list != nullptr && a.T == 1;
  const bool want_stage = list_direct || a.idx != nullptr;
  const size_t d4 = ((size_t)a.d + 3) / 4 * 4, k4 = ((size_t)a.k + 3) / 4 * 4;
  a.stage = (want_stage && (d4 + k4) * 4 <= kTopkSmemMax) ? 1 : 0;
  const size_t words = d4 + (a.stage ? k4 : 0);
  a.hist16 = (KIND == TK_BF16 && NT == 1024 && (words + 16384) * 4 <= kTopkSmemMax) ? 1 : 0;
  const size_t smem = (words + (a.hist16 ? 16384 : 0)) * sizeof(uint32_t);
  a.zero_ctas = 0;
  if (a.zero != nullptr && a.zero_n >= 4) {
    const size_t v = a.zero_n / 4;
    a.zero_ctas = (int)std::min<size_t>((v + NT - 1) / NT, 32);
  }
  static unsigned configured = 0;
  cudaError_t e = ensure_smem_attr(topk_kernel<KIND, NT>, (int)kTopkSmemMax, &configured);
  if (e != cudaSuccess) return e;
  e = launch_pdl(topk_kernel<KIND, NT>, dim3(a.T + a.zero_ctas), dim3(NT), smem, s, a);
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

bool topk_block_supported(int d) { return d >= 1 && d <= kMaxBlockRow; }

bool topk_bitmask_supported(int T, int d, int kind) {
  return T == 1 && d >= 1 && d <= 1024 * 16 && (kind == TK_F32 || kind == TK_BF16);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.T <= 0 || a.d <= 0) return cudaSuccess;
  cudaError_t err = cudaSuccess;
  bool done = false;
  switch (a.kind) {
    case TK_F32: done = try_launch_reg<TK_F32>(a, s, &err); break;
    case TK_BF16: done = try_launch_reg<TK_BF16>(a, s, &err); break;
    case TK_QUANT_F32: done = try_launch_reg<TK_QUANT_F32>(a, s, &err); break;
    case TK_QUANT_BF16: done = try_launch_reg<TK_QUANT_BF16>(a, s, &err); break;
    default: return cudaErrorInvalidValue;
  }
  if (done) return err;
  if (a.block > 1) return cudaErrorInvalidValue;   // block selections: rows of up to 16 K only
  // longer rows: the shared-memory kernel
  // Few rows: a full 1024-thread CTA per row keeps the latency down.  Many
  // rows (prefill): 256-thread CTAs so that several rows share an SM.
  if (a.T >= 2 * kNumSMs) return launch_nt<256>(a, s);
  return launch_nt<1024>(a, s);
}

}  // namespace qs
