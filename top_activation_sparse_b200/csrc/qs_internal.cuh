// Internal declarations shared by the library's translation units.
// Nothing here is part of the C ABI (see include/qs.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "qs.h"

namespace qs {

// ---------------------------------------------------------------------------
// device status word (first bytes of every workspace)
// ---------------------------------------------------------------------------
enum DevCode : uint32_t {
  DEV_OK = 0,
  DEV_TIMEOUT = 1,      // a bounded wait ran out
  DEV_CHECK = 2,        // an internal consistency check failed
};

struct DevStatus {
  uint32_t code;        // first error wins (atomicCAS from 0)
  uint32_t where;       // which check / wait
  uint32_t detail;      // free-form (an index, an iteration count)
  uint32_t pad;
};

__device__ __forceinline__ void dev_fail(DevStatus* st, uint32_t code, uint32_t where,
                                         uint32_t detail) {
  if (st == nullptr) return;
  if (atomicCAS(&st->code, 0u, code) == 0u) {
    st->where = where;
    st->detail = detail;
  }
}

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  // weights are read exactly once per call: do not keep them in L1
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// ---- mbarrier / bulk-copy (TMA) helpers ------------------------------------
// Every wait is bounded: after kWaitLimit polls it gives up and returns false,
// and the caller records DEV_TIMEOUT instead of hanging the GPU.
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity,
                                          uint32_t limit = kWaitLimit) {
  for (uint32_t it = 0; it < limit; ++it)
    if (mbar_try_wait(b, parity)) return true;
  return false;
}
// Consumer-side wait: poll with a short sleep so that waiting warps leave the
// issue slots to the producer and to the warps that have data.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* b, uint32_t parity,
                                                  uint32_t limit = kWaitLimit) {
  for (uint32_t it = 0; it < limit; ++it) {
    if (mbar_try_wait(b, parity)) return true;
    __nanosleep(64);
  }
  return false;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory (this CTA only); completion
// is signalled on `bar` as transaction bytes.  16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---- programmatic dependent launch ----------------------------------------
// Kernels of one call are launched with programmatic stream serialization:
// the next kernel's CTAs may be scheduled while this one runs, which hides the
// launch latency.  Every kernel first waits for the previous grid to finish
// (griddepcontrol.wait, a no-op when not launched that way) and only then
// touches memory, so the stream order of the results is unchanged.  The next
// grid is released only once every CTA of this one has executed
// launch_dependents (or exited), so it never takes resources this grid's
// later waves need.
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename F>
cudaError_t ensure_smem_attr(F* kernel, int bytes, unsigned* done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned bit = 1u << (dev & 31);
  if (*done_mask & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) *done_mask |= bit;
  return e;
}

// ---------------------------------------------------------------------------
// workspace layout (host side; one function sizes and places every buffer)
// ---------------------------------------------------------------------------
constexpr int kNumSMs = 148;          // B200; split counts are a pure function of sizes
constexpr size_t kWsAlign = 256;

struct GemvPlan {
  int TT;          // tokens per pass (1, 2, 4, 8)
  int groups;      // ceil(T / TT)
  int n_ct;        // column tiles
  int S;           // splits of the row list
  int mats;        // weight matrices sharing the row list (2 for up/gate)
  size_t parts_elems;  // partial-sum buffer, f32 elements (all copies)
  int tickets;     // ticket counters the launch uses
  // gather-GEMV pipeline (bulk-copy ring), unused by the int8 path
  int vec_tile;    // 16-byte vectors of one row segment (= consumer threads used)
  int threads;     // consumer threads (multiple of 32) + one producer warp
  int rps;         // rows per pipeline stage
  int nst;         // pipeline stages
  int copies;      // accumulator copies: split s adds into copy s % copies (fewer adds per address)
  int mma;         // bf16, 4-8 tokens: the tensor-core (mma.sync) kernel
  int cta_sm;      // tensor-core kernel: CTAs per SM the plan is sized for (1 or 2)
  int rcap;        // rows staged in shared memory per piece
  size_t smem;     // dynamic shared memory bytes
};

GemvPlan plan_gemv(int T, int d_out, int rows_bound, int mats, int elem_bytes);
GemvPlan plan_qgemv(int T, int d_out, int rows_bound);
bool qgemv_supported(int d_out);

struct WsLayout {
  size_t status = 0;          // DevStatus
  size_t tickets = 0;         // int32 counters, zero between calls
  int n_tickets = 0;
  // stage 1: top-K on the projection input
  size_t xsf_x = 0;           // [T, d_in] f32 dense masked values
  size_t xq = 0;              // [T, d_in] int8 dense masked q (quant path)
  size_t gamma = 0;           // [T] f32 (quant path)
  size_t list_x = 0;          // [d_in] int32
  size_t lval_x = 0;          // [d_in][T] f32 (or int8 for the quant path)
  size_t cnt = 0;             // int32[4]: rows of list_x, rows of list_h, ...
  // stage 2: projection(s)
  size_t parts1 = 0;          // gemv partial sums
  size_t h = 0;               // [T, d_ff] f32 (ffn)
  size_t xsf_h = 0;           // [T, d_ff] f32 (ffn)
  size_t list_h = 0;          // [d_ff] int32 (ffn)
  size_t lval_h = 0;          // [d_ff][T] f32 (ffn)
  size_t parts2 = 0;          // down-projection partials (ffn)
  size_t parts1b = 0;         // gate-projection partials (quantized ffn)
  size_t u = 0;               // [T, d_ff] f32 up projection (quantized ffn)
  size_t xq_h = 0;            // [T, d_ff] int8 dense masked codes of h (quantized ffn)
  size_t gamma_h = 0;         // [T] f32 (quantized ffn)
  size_t xs_bf16 = 0;         // [T, d_in] bf16 (prefill)
  size_t alpha_parts = 0;     // f64 partial sums (ternary pack)
  size_t alpha = 0;           // f32 (ternary pack)
  size_t fpug = 0;            // one-kernel FFN: per-split up/gate partial sums
  size_t fpug_elems = 0;
  size_t fhnz = 0;            // one-kernel FFN: nonzero h per index range (int32)
  size_t total = 0;
  size_t parts1_elems = 0, parts2_elems = 0;
  int ticket_topk_x = 0, ticket_topk_h = 0, ticket_g1 = 0, ticket_g2 = 0, ticket_alpha = 0;
};

// Returns false if the sizes are invalid for `op`.
bool ws_layout(int op, int T, int d_in, int d_out, int k, WsLayout* L);

// Every host-side check of qs_sparse_linear's arguments (nothing is enqueued).
qs_status check_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                              const void* wt, const void* y, const void* ws, size_t ws_bytes,
                              WsLayout* L);

// ---------------------------------------------------------------------------
// kernel launchers (host functions, defined next to their kernels)
// ---------------------------------------------------------------------------
enum TopkKind { TK_F32 = 0, TK_BF16 = 1, TK_QUANT_F32 = 2, TK_QUANT_BF16 = 3 };

struct TopkArgs {
  const void* x = nullptr;   // [T, d] input (f32 / bf16)
  int T = 0, d = 0, k = 0;
  int kind = TK_F32;
  // optional outputs
  int32_t* idx = nullptr;    // [T, k]
  void* val = nullptr;       // [T, k] in the input dtype
  uint8_t* mask = nullptr;   // [T, d]
  void* xs = nullptr;        // [T, d] input dtype, masked
  float* xsf = nullptr;      // [T, d] f32, masked (gemv input)
  int8_t* xq = nullptr;      // [T, d] int8, masked q (quant gemv input)
  int8_t* q_full = nullptr;  // [T, d] int8, all q (quant path debug output)
  float* gamma = nullptr;    // [T] (quant path)
  float eps = 0.f;           // (quant path)
  int32_t* list = nullptr;   // [d] union of rows with a kept nonzero
  float* list_val = nullptr; // [d][T] f32 values of the listed rows (projection input)
  int8_t* list_q = nullptr;  // [d][T] int8 codes of the listed rows (quant path)
  int32_t* list_count = nullptr;
  int32_t* ticket = nullptr;
  int block = 1;             // Block Q-Sparse: rows per shared selection (1 = per row)
  uint32_t* union_bits = nullptr;  // [ceil(d/32)] zero between calls (several tokens)
  uint32_t* nz_bits = nullptr;     // one token: bitmask of the row's nonzero entries, written by
                                   // the kernel that produced the row; read, then zeroed, here
  float* zero = nullptr;     // accumulators of the next kernel: set to 0 here
  size_t zero_n = 0;         // floats, multiple of 4
  int32_t* zero_word = nullptr;    // a counter of later kernels: set to 0 here (after the wait)
  int early_release = 0;     // release the next grid before waiting (it waits for this one)
  DevStatus* status = nullptr;
  // set by launch_topk from the sizes
  int stage = 0;             // the row's list (or idx) is staged in shared memory
  int hist16 = 0;            // bf16: one 15-bit radix pass (packed 16-bit counters)
  int zero_ctas = 0;         // CTAs after the T row CTAs that only zero `zero`
};

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);
// True when launch_topk takes a one-token row of this size through the list
// kernel, which can consume (and then clears) a producer's nonzero bitmask.
bool topk_bitmask_supported(int T, int d, int kind);
// Rows this long can take block selections (a.block > 1).
bool topk_block_supported(int d);

// Zero `n` floats (n % 4 == 0) cooperatively across the whole grid.
__device__ __forceinline__ void grid_zero(float* p, size_t n) {
  if (p == nullptr) return;
  const size_t nthr = (size_t)gridDim.x * gridDim.y * gridDim.z * blockDim.x;
  const size_t cta = ((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  const float4 z = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (size_t i = cta * blockDim.x + threadIdx.x; i < n / 4; i += nthr)
    reinterpret_cast<float4*>(p)[i] = z;
}

struct GemvArgs {
  const void* w[2] = {nullptr, nullptr};  // W^T [d_in, d_out]
  int d_in = 0, d_out = 0, T = 0;
  int bf16 = 1;               // weight / output element type
  int mode = 0;               // 0 plain, 1 relu2-glu, 2 drelu
  const int32_t* list = nullptr;      // rows to stream
  const float* list_val = nullptr;    // [n][T] their per-token values (one token), or
  const float* xsf = nullptr;         // [T][d_in] dense masked values (several tokens)
  const int32_t* list_count = nullptr;
  float* parts = nullptr;
  int32_t* tickets = nullptr;
  void* y = nullptr;          // mode 0: [T, d_out] in the weight dtype
  float* h = nullptr;         // mode 1/2: [T, d_out] f32
  const float* b_up = nullptr;
  const float* b_gate = nullptr;
  float* zero = nullptr;       // accumulators of the next kernel: set to 0 here
  size_t zero_n = 0;
  uint32_t* hbits = nullptr;   // mode 1/2, one token: OR the bitmask of nonzero h in here
  // One-token FFN, counter of the nonzero h (zero between calls):
  //   mode 1/2 add their nonzero h to it;
  //   mode 0 (the down projection) reads it: with at most k_sel nonzero h the
  //   kept rows are exactly the nonzero h, so each CTA takes them from its own
  //   index range of hsrc instead of the top-K's list.  The first kernel of
  //   the next FFN call (the top-K on x, TopkArgs::zero_word) clears it.
  int32_t* hcount = nullptr;
  const float* hsrc = nullptr;
  int k_sel = 0;
  int32_t* rows_out = nullptr;   // mode 0 from h: the number of rows streamed (workspace stats)
  DevStatus* status = nullptr;
  // failure-detection testing only (qs_debug_inject): the producer issues no
  // copies, and every wait of the launch gives up after wait_limit polls
  int no_copies = 0;
  uint32_t wait_limit = kWaitLimit;
  GemvPlan plan{};
};

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t s);

// Host-side fault injection state set by qs_debug_inject (tests only).
struct FaultState {
  int mode = QS_FAULT_NONE;
  uint32_t wait_polls = 0;
};
extern FaultState g_fault;

struct QGemvArgs {
  const uint32_t* wp = nullptr;  // [d_in, d_out/16]
  int d_in = 0, d_out = 0, T = 0;
  const float* gamma = nullptr;  // [T]
  float alpha = 0.f;
  const int32_t* list = nullptr;
  const int8_t* list_q = nullptr;  // [n][T] int8 codes of the listed rows (one token), or
  const int8_t* xq = nullptr;      // [T][d_in] dense masked codes (several tokens)
  const int32_t* list_count = nullptr;
  float* parts = nullptr;          // [T][d_out] f32 accumulators (exact integers), zeroed before
  int32_t* tickets = nullptr;
  float* y = nullptr;
  int32_t* acc = nullptr;
  // the quantized FFN's gate projection: y receives h = act(u, this
  // projection) in float32 steps instead of the projection itself
  int gating = 0;                  // 0: plain, 1: ReLU(u)^2 * g, 2: ReLU(g + b_gate) * ReLU(u + b_up)
  const float* gate_u = nullptr;   // [T, d_out] the up projection, read by the gating epilogue
  const float* b_up = nullptr;
  const float* b_gate = nullptr;
  float* zero = nullptr;           // accumulators of the next launch: set to 0 here
  size_t zero_n = 0;
  DevStatus* status = nullptr;
  GemvPlan plan{};
};

cudaError_t launch_qgemv(const QGemvArgs& a, cudaStream_t s);

// ---- one-token FFN as one persistent kernel (ffn_fused.cu) -------------------
struct FfnFusedPlan {
  int G = 0;                   // CTAs (the occupancy-sized grid: all resident)
  int n_ct_ug = 0, vt_ug = 0;  // up/gate column tiles, 16-byte vectors per tile
  int n_ct_dn = 0, vt_dn = 0;  // down column tiles
  int rps_ug = 0, rps_dn = 0;  // row tiles per ring stage
  int S_ug = 0, S_dn = 0;      // index ranges (splits) of x and of h
};
struct FfnFusedArgs {
  const void* x = nullptr;     // [d_model] bf16
  const void* w_up = nullptr;  // W^T [d_model, d_ff] bf16
  const void* w_gate = nullptr;
  const void* w_down = nullptr;  // W^T [d_ff, d_model] bf16
  int d_model = 0, d_ff = 0, k_in = 0, k_h = 0;
  int act = 1;                 // 1: ReLU(u)^2 * g, 2: ReLU(g + b_gate) * ReLU(u + b_up)
  const float* b_up = nullptr;
  const float* b_gate = nullptr;
  void* y = nullptr;           // [d_model] bf16
  float* h = nullptr;          // [d_ff] f32
  float* pug = nullptr;        // [S_ug][2][d_ff] per-split partial sums
  float* pdn = nullptr;        // [d_model] down accumulator (cleared in the kernel)
  int32_t* hnz = nullptr;      // [S_dn] nonzero h per index range
  int32_t* bar = nullptr;      // [5] grid-barrier counters, zero between calls
  int32_t* list_x = nullptr;
  float* lval_x = nullptr;
  int32_t* list_h = nullptr;
  float* lval_h = nullptr;
  int32_t* cnt = nullptr;      // [0] listed x rows, [1] listed h rows
  DevStatus* status = nullptr;
  // failure-detection testing only (qs_debug_inject): no weight copies, and
  // the stage waits give up after wait_limit polls
  int no_copies = 0;
  uint32_t wait_limit = 0;
  FfnFusedPlan plan{};
};
size_t ffn_fused_smem();
bool plan_ffn_fused(int d_model, int d_ff, int G, FfnFusedPlan* p);
size_t ffn_fused_pug_elems(int d_model, int d_ff);   // 0: the sizes are not supported
int ffn_fused_grid();                                  // resident CTAs (0: unavailable)
cudaError_t launch_ffn_fused(const FfnFusedArgs& a, bool cooperative, cudaStream_t s);


// The quantized FFN's gating of one column, float32 steps in a fixed order
// (g: this projection, u: the up projection):
//   1: r = max(u, 0); h = (r * r) * g       2: h = max(g + b_gate, 0) * max(u + b_up, 0)
__device__ __forceinline__ float quant_gate_value(int gating, float u, float g, float bu, float bg) {
  if (gating == 1) {
    const float r = fmaxf(u, 0.0f);
    return __fmul_rn(__fmul_rn(r, r), g);
  }
  return __fmul_rn(fmaxf(__fadd_rn(g, bg), 0.0f), fmaxf(__fadd_rn(u, bu), 0.0f));
}

// The tensor-core (tcgen05 kind::i8) int8 x ternary kernel for 8 to 64 tokens,
// streaming every packed row (qgemv_tc.cu); plan.mma == 2 marks its plans.
bool qgemv_tc_supported(int T, int d_in, int d_out);
GemvPlan plan_qgemv_tc(int T, int d_in, int d_out);
cudaError_t launch_qgemv_tc(const QGemvArgs& a, cudaStream_t s);

struct PackArgs {
  const float* w = nullptr;  // [d_out, d_in]
  int d_out = 0, d_in = 0;
  float eps = 0.f;
  uint32_t* packed = nullptr;
  float* alpha_out = nullptr;
  double* alpha_parts = nullptr;
  float* alpha_ws = nullptr;
  int32_t* ticket = nullptr;
  DevStatus* status = nullptr;
};

constexpr int kPackSumBlocks = 592;   // fixed: the fp64 sum order does not depend on the GPU

cudaError_t launch_ternary_pack(const PackArgs& a, cudaStream_t s);

struct PrefillArgs {
  const __nv_bfloat16* xs = nullptr;  // [M, K] masked activations (row-major)
  const __nv_bfloat16* wt = nullptr;  // [K, N] W^T (row-major)
  __nv_bfloat16* y = nullptr;         // [M, N]
  int M = 0, N = 0, K = 0;
  DevStatus* status = nullptr;
};

cudaError_t launch_prefill_gemm(const PrefillArgs& a, cudaStream_t s);
bool prefill_supported(int M, int N, int K);

// Backward of the projection under the straight-through estimator, on the
// tensor cores (bf16 operands, f32 results).
struct BackwardGemmArgs {
  const __nv_bfloat16* grad_y = nullptr;  // [T, d_out]
  const __nv_bfloat16* wt = nullptr;      // [d_in, d_out] (W^T)
  const __nv_bfloat16* xs = nullptr;      // [T, d_in] X_sparse
  float* grad_x = nullptr;                // [T, d_in] out
  float* grad_wt = nullptr;               // [d_in, d_out] accumulated into
  int T = 0, d_in = 0, d_out = 0;
  DevStatus* status = nullptr;
};
bool backward_gemm_supported(int T, int d_in, int d_out);

// Decode-size backward kernels (backward.cu).
struct RowDotPlan {
  int TT;          // tokens per pass (1, 2, 4, 8)
  int groups;      // ceil(T / TT)
  int n_ct;        // column tiles of W^T
  int S;           // row splits
  int vec_tile;    // 16-byte vectors per row segment
  int threads;     // consumers (multiple of 32) + one producer warp
  int rps;         // rows per ring stage
  int nst;         // ring stages
  size_t smem;
};
RowDotPlan plan_rowdot(int T, int d_in, int d_out, int elem_bytes);

struct RowDotArgs {            // grad_x [T, d_in] = grad_y [T, d_out] . (W^T)^T
  const void* wt = nullptr;    // [d_in, d_out]
  const void* grad_y = nullptr;
  float* grad_x = nullptr;     // zeroed, then added into, by launch_rowdot
  int T = 0, d_in = 0, d_out = 0;
  int bf16 = 1;
  DevStatus* status = nullptr;
  RowDotPlan plan{};
};
cudaError_t launch_rowdot(const RowDotArgs& a, cudaStream_t s);

struct RowAxpyArgs {           // grad_wt[i, :] += sum_t xs[t, i] grad_y[t, :] for listed rows i
  const void* grad_y = nullptr;
  float* grad_wt = nullptr;
  const int32_t* list = nullptr;
  const int32_t* list_count = nullptr;
  const float* list_val = nullptr;   // one token: the listed rows' values
  const float* xsf = nullptr;        // several tokens: [T, d_in] dense masked values
  int T = 0, d_in = 0, d_out = 0;
  int bf16 = 1;
  DevStatus* status = nullptr;
};
cudaError_t launch_rowaxpy(const RowAxpyArgs& a, cudaStream_t s);
cudaError_t launch_grad_x_gemm(const BackwardGemmArgs& a, cudaStream_t s);
cudaError_t launch_grad_wt_gemm(const BackwardGemmArgs& a, cudaStream_t s);

}  // namespace qs
