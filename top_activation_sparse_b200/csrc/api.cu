// extern "C" entry points of include/qs.h: argument checks, the workspace
// layout, and the order in which the kernels are enqueued.  Every step of the
// computation runs in this library's CUDA kernels; there is no host fallback.
#include <atomic>
#include <cstring>

#include "gate_first.cuh"
#include "qs_internal.cuh"

namespace qs {

FaultState g_fault;

namespace {

// Token rows are processed in chunks of at most this many (decode kernels
// keep one accumulator per token in registers; see plan_gemv).
constexpr int kChunkT = QS_PREFILL_MIN_T;
constexpr size_t kTicketBytes = 64 * 1024;       // fixed ticket region
constexpr int kTicketCap = (int)(kTicketBytes / sizeof(int32_t));
// fixed ticket slots
constexpr int kTkTopkX = 0, kTkTopkH = 1, kTkAlpha = 2, kTkUpRows = 3, kTkHCount = 4,
              kTkGemv = 8;                        // (slots 5-7 unused)
// union bitmasks of the several-token path, and the open gates of the
// gate-first FFN (zero between calls)
constexpr int kTkGemvEnd = 4096;
constexpr int kUnionX = 4096, kUnionH = 4096 + QS_MAX_ROW / 32;
constexpr int kGateBits = kUnionH + QS_MAX_ROW / 32;
// grid-barrier counters of the one-kernel FFN (zero between calls)
constexpr int kTkFusedBar = kGateBits + QS_MAX_ROW / 32;
static_assert(kTkFusedBar + 5 <= (int)(64 * 1024 / 4), "ticket region too small");

size_t align_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }

bool aligned16(const void* p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

int elem_bytes(int dtype) { return dtype == QS_F32 ? 4 : 2; }

long rows_bound(int T, int d, int k) {
  const long tk = (long)T * (long)k;
  return tk < d ? tk : d;
}

// Tokens per chunk: at most kChunkT, a whole number of Block Q-Sparse blocks.
int chunk_tokens(int block) { return block <= 1 ? kChunkT : (kChunkT / block) * block; }

// Distinct rows a chunk of Tc tokens can keep: k per selection.
long rows_bound_blocks(int Tc, int d, int k, int block) {
  const int b = block < 1 ? 1 : block;
  return rows_bound((Tc + b - 1) / b, d, k);
}

}  // namespace

// Same layout for every dtype: each buffer is sized for the larger of the
// f32 and bf16 plans.  The status word and the ticket counters sit at fixed
// offsets, so a zeroed workspace stays valid across ops and sizes.
bool ws_layout(int op, int T, int d_in, int d_out, int k, WsLayout* L) {
  *L = WsLayout{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + (bytes ? bytes : 1));
    return o;
  };
  L->status = take(sizeof(DevStatus));
  L->tickets = take(kTicketBytes);
  L->n_tickets = kTicketCap;
  L->cnt = take(4 * sizeof(int32_t));
  L->ticket_topk_x = kTkTopkX;
  L->ticket_topk_h = kTkTopkH;
  L->ticket_alpha = kTkAlpha;
  const int Tc = T < kChunkT ? T : kChunkT;
  // Partial-sum buffers are sized for the largest plan any chunk (1..Tc
  // tokens) of either dtype can pick: a short last chunk may split more.
  // The number of accumulator copies grows with the splits, i.e. with K, so
  // the buffers are sized for every K up to the row length: a workspace stays
  // valid for calls of the same sizes with any K.
  (void)k;
  auto max_parts = [&](int d_out_, int d_rows, int /*kk*/, int mats) {
    size_t m = 0;
    for (int t = 1; t <= Tc; ++t) {
      for (int rb : {(int)rows_bound(t, d_rows, 1), (int)rows_bound(t, d_rows, d_rows)}) {
        for (int eb = 2; eb <= 4; eb += 2) {
          const GemvPlan p = plan_gemv(t, d_out_, rb, mats, eb);
          if (p.parts_elems > m) m = p.parts_elems;
        }
      }
    }
    return m;
  };
  auto max_qparts = [&](int d_out_, int d_rows, int /*kk*/) {
    size_t m = 0;
    for (int t = 1; t <= Tc; ++t) {
      for (int rb : {(int)rows_bound(t, d_rows, 1), (int)rows_bound(t, d_rows, d_rows)}) {
        const GemvPlan p = plan_qgemv(t, d_out_, rb);
        if (p.parts_elems > m) m = p.parts_elems;
      }
    }
    return m;
  };
  switch (op) {
    case QS_OP_TOPK_MASK:
      if (T < 1 || d_in < 1 || d_in > QS_MAX_ROW || k < 0 || k > d_in) return false;
      break;
    case QS_OP_SPARSE_LINEAR: {
      if (T < 1 || d_in < 1 || d_out < 1 || d_in > QS_MAX_ROW || d_out > QS_MAX_ROW || k < 0 ||
          k > d_in)
        return false;
      L->xsf_x = take((size_t)Tc * d_in * sizeof(float));
      L->list_x = take((size_t)d_in * sizeof(int32_t));
      L->lval_x = take((size_t)d_in * Tc * sizeof(float));
      L->parts1_elems = max_parts(d_out, d_in, k, 1);
      L->parts1 = take(L->parts1_elems * sizeof(float));
      if (T >= kChunkT) L->xs_bf16 = take((size_t)T * d_in * sizeof(uint16_t));
      break;
    }
    case QS_OP_SPARSE_FFN:
    case QS_OP_SPARSE_FFN_GATE_FIRST: {
      if (T < 1 || d_in < 1 || d_out < 1 || d_in > QS_MAX_ROW || d_out > QS_MAX_ROW || k < 0 ||
          k > d_out)
        return false;
      L->xsf_x = take((size_t)Tc * d_in * sizeof(float));
      L->list_x = take((size_t)d_in * sizeof(int32_t));
      L->lval_x = take((size_t)d_in * Tc * sizeof(float));
      // up and gate together, or (gate first) the gate alone
      L->parts1_elems = max_parts(d_out, d_in, d_in, op == QS_OP_SPARSE_FFN ? 2 : 1);
      L->parts1 = take(L->parts1_elems * sizeof(float));
      L->h = take((size_t)Tc * d_out * sizeof(float));
      L->xsf_h = take((size_t)Tc * d_out * sizeof(float));
      L->list_h = take((size_t)d_out * sizeof(int32_t));
      L->lval_h = take((size_t)d_out * Tc * sizeof(float));
      L->parts2_elems = max_parts(d_in, d_out, k, 1);
      L->parts2 = take(L->parts2_elems * sizeof(float));
      if (op == QS_OP_SPARSE_FFN) {
        // the one-kernel path of one-token bf16 calls (ffn_fused.cu); its down
        // accumulator is parts2 (>= d_model floats)
        L->fpug_elems = ffn_fused_pug_elems(d_in, d_out);
        if (L->fpug_elems != 0) {
          L->fpug = take(L->fpug_elems * sizeof(float));
          L->fhnz = take((size_t)2 * kNumSMs * sizeof(int32_t));
        }
      }
      break;
    }
    case QS_OP_QUANT_SPARSE_LINEAR: {
      if (T < 1 || d_in < 1 || d_out < 64 || d_in > QS_MAX_ROW || d_out > QS_MAX_ROW || k < 0 ||
          k > d_in || (d_out % 64) != 0)
        return false;
      L->xq = take((size_t)Tc * d_in);
      L->gamma = take((size_t)Tc * sizeof(float));
      L->list_x = take((size_t)d_in * sizeof(int32_t));
      L->lval_x = take((size_t)d_in * Tc);
      L->parts1_elems = max_qparts(d_out, d_in, k);
      L->parts1 = take(L->parts1_elems * sizeof(float));
      break;
    }
    case QS_OP_QUANT_SPARSE_FFN: {
      if (T < 1 || d_in < 64 || d_out < 64 || d_in > QS_MAX_ROW || d_out > QS_MAX_ROW || k < 0 ||
          k > d_out || (d_in % 64) != 0 || (d_out % 64) != 0)
        return false;
      L->xq = take((size_t)Tc * d_in);
      L->gamma = take((size_t)Tc * sizeof(float));
      L->list_x = take((size_t)d_in * sizeof(int32_t));
      L->lval_x = take((size_t)d_in * Tc);
      L->parts1_elems = max_qparts(d_out, d_in, d_in);
      L->parts1 = take(L->parts1_elems * sizeof(float));
      L->parts1b = take(L->parts1_elems * sizeof(float));
      L->u = take((size_t)Tc * d_out * sizeof(float));
      L->h = take((size_t)Tc * d_out * sizeof(float));
      L->xq_h = take((size_t)Tc * d_out);
      L->gamma_h = take((size_t)Tc * sizeof(float));
      L->list_h = take((size_t)d_out * sizeof(int32_t));
      L->lval_h = take((size_t)d_out * Tc);
      L->parts2_elems = max_qparts(d_in, d_out, d_out);
      L->parts2 = take(L->parts2_elems * sizeof(float));
      break;
    }
    case QS_OP_TERNARY_PACK:
      if (d_in < 1 || d_out < 16 || (d_out % 16) != 0) return false;
      L->alpha_parts = take(kPackSumBlocks * sizeof(double));
      L->alpha = take(sizeof(float));
      break;
    default:
      return false;
  }
  L->total = off;
  return true;
}

qs_status check_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                              const void* wt, const void* y, const void* ws, size_t ws_bytes,
                              WsLayout* L) {
  if ((dtype != QS_F32 && dtype != QS_BF16) || x == nullptr || wt == nullptr || y == nullptr ||
      T < 1 || d_in < 1 || d_out < 1 || k < 0 || k > d_in)
    return QS_ERR_INVALID_ARG;
  if (d_in > QS_MAX_ROW || d_out > QS_MAX_ROW) return QS_ERR_UNSUPPORTED;
  const int V = 16 / elem_bytes(dtype);
  if ((d_out % V) != 0 || !aligned16(x) || !aligned16(wt) || !aligned16(y)) return QS_ERR_ALIGNMENT;
  if (!ws_layout(QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, L)) return QS_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < L->total) return QS_ERR_WORKSPACE;
  if (!aligned16(ws)) return QS_ERR_ALIGNMENT;
  return QS_OK;
}

}  // namespace qs

using namespace qs;

namespace {

struct WsView {
  unsigned char* base;
  DevStatus* status() const { return reinterpret_cast<DevStatus*>(base); }
  int32_t* ticket(const WsLayout& L, int slot) const {
    return reinterpret_cast<int32_t*>(base + L.tickets) + slot;
  }
  template <typename T> T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
};

qs_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QS_OK : QS_ERR_CUDA; }

#define QS_TRY_CUDA(expr)                         \
  do {                                            \
    cudaError_t _e = (expr);                      \
    if (_e != cudaSuccess) return QS_ERR_CUDA;    \
  } while (0)

qs_status check_ws(int op, int T, int d_in, int d_out, int k, void* ws, size_t ws_bytes,
                   WsLayout* L) {
  if (!ws_layout(op, T, d_in, d_out, k, L)) return QS_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < L->total) return QS_ERR_WORKSPACE;
  if (!aligned16(ws)) return QS_ERR_ALIGNMENT;
  return QS_OK;
}

bool valid_dtype(int dt) { return dt == QS_F32 || dt == QS_BF16; }

// A launch plan must fit the buffers the layout reserved for it.
bool plan_fits(const GemvPlan& p, size_t parts_cap, int ticket_offset) {
  return p.parts_elems <= parts_cap && kTkGemv + ticket_offset + p.tickets <= kTkGemvEnd;
}

// Split the gemv ticket slots of one layout: first projection, then second.
int32_t* gemv_tickets(const WsView& w, const WsLayout& L, int which, const GemvPlan& first) {
  return w.ticket(L, kTkGemv + (which == 0 ? 0 : first.tickets));
}

}  // namespace

extern "C" {

const char* qs_status_string(int status) {
  switch (status) {
    case QS_OK: return "QS_OK";
    case QS_ERR_INVALID_ARG: return "QS_ERR_INVALID_ARG: invalid size, k, enum or NULL pointer";
    case QS_ERR_ALIGNMENT: return "QS_ERR_ALIGNMENT: pointer or row length not 16-byte aligned";
    case QS_ERR_WORKSPACE: return "QS_ERR_WORKSPACE: workspace missing or too small";
    case QS_ERR_CUDA: return "QS_ERR_CUDA: a CUDA call or kernel launch failed";
    case QS_ERR_TIMEOUT: return "QS_ERR_TIMEOUT: a bounded device wait ran out";
    case QS_ERR_DEVICE_CHECK: return "QS_ERR_DEVICE_CHECK: a device-side consistency check failed";
    case QS_ERR_UNSUPPORTED: return "QS_ERR_UNSUPPORTED: sizes outside what this build handles";
    default: return "unknown qs_status";
  }
}

size_t qs_workspace_size(int op, int T, int d_in, int d_out, int k) {
  WsLayout L;
  if (!ws_layout(op, T, d_in, d_out, k, &L)) return 0;
  return L.total;
}

qs_status qs_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr) return QS_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

qs_status qs_device_status(void* ws, void* stream) {
  if (ws == nullptr) return QS_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  DevStatus st;
  QS_TRY_CUDA(cudaStreamSynchronize(s));
  QS_TRY_CUDA(cudaMemcpyAsync(&st, ws, sizeof(st), cudaMemcpyDeviceToHost, s));
  QS_TRY_CUDA(cudaStreamSynchronize(s));
  if (st.code == DEV_OK) return QS_OK;
  QS_TRY_CUDA(cudaMemsetAsync(ws, 0, sizeof(st), s));
  QS_TRY_CUDA(cudaStreamSynchronize(s));
  return st.code == DEV_TIMEOUT ? QS_ERR_TIMEOUT : QS_ERR_DEVICE_CHECK;
}

qs_status qs_workspace_stats(const void* ws, int op, int T, int d_in, int d_out, int k,
                             int32_t* rows, void* stream) {
  if (ws == nullptr || rows == nullptr) return QS_ERR_INVALID_ARG;
  WsLayout L;
  if (!ws_layout(op, T, d_in, d_out, k, &L)) return QS_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t c[4] = {0, 0, 0, 0};
  QS_TRY_CUDA(cudaMemcpyAsync(c, (const unsigned char*)ws + L.cnt, sizeof(c),
                              cudaMemcpyDeviceToHost, s));
  QS_TRY_CUDA(cudaStreamSynchronize(s));
  const bool ffn = op == QS_OP_SPARSE_FFN || op == QS_OP_SPARSE_FFN_GATE_FIRST ||
                   op == QS_OP_QUANT_SPARSE_FFN;
  rows[0] = c[0];
  rows[1] = ffn ? c[1] : 0;
  if (op == QS_OP_SPARSE_FFN_GATE_FIRST) rows[2] = c[2];
  return QS_OK;
}

qs_status qs_workspace_list(const void* ws, int op, int T, int d_in, int d_out, int k, int which,
                            int32_t* rows, int cap, void* vals, int32_t* count, void* stream) {
  if (ws == nullptr || rows == nullptr || count == nullptr || cap < 0) return QS_ERR_INVALID_ARG;
  const bool ffn = op == QS_OP_SPARSE_FFN || op == QS_OP_SPARSE_FFN_GATE_FIRST ||
                   op == QS_OP_QUANT_SPARSE_FFN;
  if (!(op == QS_OP_SPARSE_LINEAR || op == QS_OP_QUANT_SPARSE_LINEAR || ffn)) return QS_ERR_INVALID_ARG;
  if (which != 0 && !(which == 1 && ffn)) return QS_ERR_INVALID_ARG;
  if (vals != nullptr && T != 1) return QS_ERR_INVALID_ARG;
  WsLayout L;
  if (!ws_layout(op, T, d_in, d_out, k, &L)) return QS_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const unsigned char* base = (const unsigned char*)ws;
  int32_t c[4] = {0, 0, 0, 0};
  QS_TRY_CUDA(cudaMemcpyAsync(c, base + L.cnt, sizeof(c), cudaMemcpyDeviceToHost, s));
  QS_TRY_CUDA(cudaStreamSynchronize(s));
  const int n = c[which];
  const int d_rows = which == 0 ? d_in : d_out;
  *count = n;
  if (n < 0 || n > d_rows) return QS_OK;           // reported as is; nothing to copy
  const int m = n < cap ? n : cap;
  if (m > 0) {
    QS_TRY_CUDA(cudaMemcpyAsync(rows, base + (which == 0 ? L.list_x : L.list_h),
                                (size_t)m * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    if (vals != nullptr) {
      const bool codes = op == QS_OP_QUANT_SPARSE_LINEAR || op == QS_OP_QUANT_SPARSE_FFN;
      const size_t vb = codes ? 1 : sizeof(float);
      QS_TRY_CUDA(cudaMemcpyAsync(vals, base + (which == 0 ? L.lval_x : L.lval_h), (size_t)m * vb,
                                  cudaMemcpyDeviceToHost, s));
    }
    QS_TRY_CUDA(cudaStreamSynchronize(s));
  }
  return QS_OK;
}

namespace {
std::atomic<int> g_ffn_fused{1};

// A one-token bf16 FFN call (list outputs only) runs as one persistent kernel
// when the device can hold its grid and the sizes fit its staging.
bool use_ffn_fused(int op, int dtype, int T, int d_model, int d_ff, const int32_t* idx_h_out,
                   const WsLayout& L, FfnFusedPlan* fp) {
  if (!g_ffn_fused.load() || op != QS_OP_SPARSE_FFN || dtype != QS_BF16 || T != 1 ||
      idx_h_out != nullptr || L.fpug == 0)
    return false;
  const int G = ffn_fused_grid();
  if (G <= 0 || !plan_ffn_fused(d_model, d_ff, G, fp)) return false;
  return (size_t)fp->S_ug * 2 * (size_t)d_ff <= L.fpug_elems && fp->S_dn <= 2 * kNumSMs &&
         (size_t)d_model <= L.parts2_elems;
}
}  // namespace

qs_status qs_set_ffn_fused(int mode) {
  if (mode < 0 || mode > 2) return QS_ERR_INVALID_ARG;
  g_ffn_fused.store(mode);
  return QS_OK;
}

int qs_sparse_ffn_fused(int dtype, int T, int d_model, int d_ff, int with_idx_h) {
  if (!valid_dtype(dtype) || T < 1 || d_model < 1 || d_ff < 1 || d_model > QS_MAX_ROW ||
      d_ff > QS_MAX_ROW)
    return 0;
  WsLayout L;
  if (!ws_layout(QS_OP_SPARSE_FFN, T, d_model, d_ff, 0, &L)) return 0;
  FfnFusedPlan fp;
  int32_t dummy = 0;
  return use_ffn_fused(QS_OP_SPARSE_FFN, dtype, T, d_model, d_ff, with_idx_h ? &dummy : nullptr, L,
                       &fp)
             ? 1
             : 0;
}

qs_status qs_debug_inject(int mode, unsigned wait_polls) {
  if (mode != QS_FAULT_NONE && mode != QS_FAULT_GATHER_NO_COPIES) return QS_ERR_INVALID_ARG;
  g_fault.mode = mode;
  g_fault.wait_polls = mode == QS_FAULT_NONE ? 0u : wait_polls;
  return QS_OK;
}

qs_status qs_topk_mask(const void* x, int dtype, int T, int d, int k, int32_t* idx, void* val,
                       uint8_t* mask, void* xs, void* ws, size_t ws_bytes, void* stream) {
  if (!valid_dtype(dtype) || x == nullptr || T < 1 || d < 1 || k < 0 || k > d)
    return QS_ERR_INVALID_ARG;
  if (k > 0 && idx == nullptr) return QS_ERR_INVALID_ARG;
  if (d > QS_MAX_ROW) return QS_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(idx) || !aligned16(val) || !aligned16(mask) || !aligned16(xs))
    return QS_ERR_ALIGNMENT;
  WsLayout L;
  qs_status st = check_ws(QS_OP_TOPK_MASK, T, d, 0, k, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  WsView w{(unsigned char*)ws};
  TopkArgs a;
  a.x = x; a.T = T; a.d = d; a.k = k;
  a.kind = dtype == QS_F32 ? TK_F32 : TK_BF16;
  a.idx = k > 0 ? idx : nullptr;
  a.val = k > 0 ? val : nullptr;
  a.mask = mask; a.xs = xs;
  a.status = w.status();
  return from_cuda(launch_topk(a, (cudaStream_t)stream));
}

static qs_status linear_impl(const void* x, int dtype, int T, int d_in, int d_out, int k, int block,
                             const void* wt, void* y, void* const* phase_events, void* ws,
                             size_t ws_bytes, void* stream) {
  WsLayout L;
  const qs_status st = qs::check_sparse_linear(x, dtype, T, d_in, d_out, k, wt, y, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  if (block < 1 || block > QS_MAX_BLOCK) return QS_ERR_INVALID_ARG;
  if (block > 1 && !topk_block_supported(d_in)) return QS_ERR_UNSUPPORTED;
  WsView w{(unsigned char*)ws};
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = elem_bytes(dtype);
  auto mark = [&](int i) -> cudaError_t {
    if (phase_events == nullptr) return cudaSuccess;
    return cudaEventRecord((cudaEvent_t)phase_events[i], s);
  };

  // Prefill: many tokens make this a dense contraction over X_sparse.
  if (dtype == QS_BF16 && T >= QS_PREFILL_MIN_T && prefill_supported(T, d_out, d_in)) {
    QS_TRY_CUDA(mark(0));
    TopkArgs a;
    a.x = x; a.T = T; a.d = d_in; a.k = k; a.kind = TK_BF16;
    a.block = block;
    a.xs = w.at<void>(L.xs_bf16);
    a.status = w.status();
    QS_TRY_CUDA(launch_topk(a, s));
    QS_TRY_CUDA(mark(1));
    PrefillArgs p;
    p.xs = w.at<__nv_bfloat16>(L.xs_bf16);
    p.wt = reinterpret_cast<const __nv_bfloat16*>(wt);
    p.y = reinterpret_cast<__nv_bfloat16*>(y);
    p.M = T; p.N = d_out; p.K = d_in;
    p.status = w.status();
    QS_TRY_CUDA(launch_prefill_gemm(p, s));
    QS_TRY_CUDA(mark(2));
    return QS_OK;
  }

  const int chunk = chunk_tokens(block);
  for (int t0 = 0; t0 < T; t0 += chunk) {
    const bool timed = (t0 == 0);
    if (timed) QS_TRY_CUDA(mark(0));
    const int Tc = (T - t0) < chunk ? (T - t0) : chunk;
    TopkArgs a;
    a.x = (const unsigned char*)x + (size_t)t0 * d_in * eb;
    a.T = Tc; a.d = d_in; a.k = k;
    a.block = Tc > 1 ? block : 1;
    a.kind = dtype == QS_F32 ? TK_F32 : TK_BF16;
    a.xsf = Tc > 1 ? w.at<float>(L.xsf_x) : nullptr;   // only the union pass reads it
    a.list = w.at<int32_t>(L.list_x);
    a.list_val = Tc == 1 ? w.at<float>(L.lval_x) : nullptr;
    a.list_count = w.at<int32_t>(L.cnt) + 0;
    a.ticket = w.ticket(L, kTkTopkX);
    a.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionX));
    a.status = w.status();
    const GemvPlan gp = plan_gemv(Tc, d_out, (int)rows_bound_blocks(Tc, d_in, k, a.block), 1, eb);
    if (!plan_fits(gp, L.parts1_elems, 0)) return QS_ERR_UNSUPPORTED;
    a.zero = w.at<float>(L.parts1);
    a.zero_n = gp.parts_elems;
    QS_TRY_CUDA(launch_topk(a, s));
    if (timed) QS_TRY_CUDA(mark(1));

    GemvArgs g;
    g.w[0] = wt;
    g.d_in = d_in; g.d_out = d_out; g.T = Tc;
    g.bf16 = dtype == QS_BF16;
    g.mode = 0;
    g.list = a.list; g.list_val = a.list_val; g.xsf = a.xsf; g.list_count = a.list_count;
    g.parts = w.at<float>(L.parts1);
    g.plan = gp;
    g.tickets = gemv_tickets(w, L, 0, g.plan);
    if (!plan_fits(g.plan, L.parts1_elems, 0)) return QS_ERR_UNSUPPORTED;
    g.y = (unsigned char*)y + (size_t)t0 * d_out * eb;
    g.status = w.status();
    QS_TRY_CUDA(launch_gemv(g, s));
    if (timed) QS_TRY_CUDA(mark(2));
  }
  return QS_OK;
}

// One sparse gated FFN layer.  With w_up_rows (W_up output-major, [d_ff,
// d_model]) instead of wt_up it is the gate-first dReLU form: the gate
// projection runs alone, and the up projection reads only the rows of open
// gates (exact: the dReLU product is 0 wherever the gate branch is).
static qs_status ffn_impl(int op, const void* x, int dtype, int T, int d_model, int d_ff, int act,
                          int k_in, int k_h, int block, const void* wt_up, const void* w_up_rows,
                          const void* wt_gate, const float* b_up, const float* b_gate,
                          const void* wt_down, void* y, float* h_out, int32_t* idx_h_out,
                          void* const* phase_events, void* ws, size_t ws_bytes, void* stream) {
  const bool gate_first = op == QS_OP_SPARSE_FFN_GATE_FIRST;
  const void* up = gate_first ? w_up_rows : wt_up;
  if (!valid_dtype(dtype) || x == nullptr || up == nullptr || wt_gate == nullptr ||
      wt_down == nullptr || y == nullptr || T < 1 || d_model < 1 || d_ff < 1 || k_in < 0 ||
      k_in > d_model || k_h < 0 || k_h > d_ff ||
      (act != QS_ACT_RELU2_GLU && act != QS_ACT_DRELU) || (gate_first && act != QS_ACT_DRELU))
    return QS_ERR_INVALID_ARG;
  if (block < 1 || block > QS_MAX_BLOCK) return QS_ERR_INVALID_ARG;
  if (d_model > QS_MAX_ROW || d_ff > QS_MAX_ROW) return QS_ERR_UNSUPPORTED;
  if (block > 1 && (!topk_block_supported(d_model) || !topk_block_supported(d_ff)))
    return QS_ERR_UNSUPPORTED;
  const int eb = elem_bytes(dtype);
  const int V = 16 / eb;
  if ((d_model % V) != 0 || (d_ff % V) != 0) return QS_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(up) || !aligned16(wt_gate) || !aligned16(wt_down) ||
      !aligned16(y) || !aligned16(h_out) || !aligned16(idx_h_out) || !aligned16(b_up) ||
      !aligned16(b_gate))
    return QS_ERR_ALIGNMENT;
  WsLayout L;
  qs_status st = check_ws(op, T, d_model, d_ff, k_h, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  WsView w{(unsigned char*)ws};
  cudaStream_t s = (cudaStream_t)stream;
  auto mark = [&](int i) -> cudaError_t {
    if (phase_events == nullptr) return cudaSuccess;
    return cudaEventRecord((cudaEvent_t)phase_events[i], s);
  };
  FfnFusedPlan fp;
  if (use_ffn_fused(op, dtype, T, d_model, d_ff, idx_h_out, L, &fp)) {
    // one token, bf16: every step in one persistent kernel (ffn_fused.cu);
    // phase events 1-4 are all recorded after it
    FfnFusedArgs f;
    f.x = x; f.w_up = wt_up; f.w_gate = wt_gate; f.w_down = wt_down;
    f.d_model = d_model; f.d_ff = d_ff; f.k_in = k_in; f.k_h = k_h;
    f.act = act == QS_ACT_RELU2_GLU ? 1 : 2;
    f.b_up = b_up; f.b_gate = b_gate;
    f.y = y;
    f.h = h_out ? h_out : w.at<float>(L.h);
    f.pug = w.at<float>(L.fpug);
    f.pdn = w.at<float>(L.parts2);
    f.hnz = w.at<int32_t>(L.fhnz);
    f.bar = w.ticket(L, kTkFusedBar);
    f.list_x = w.at<int32_t>(L.list_x); f.lval_x = w.at<float>(L.lval_x);
    f.list_h = w.at<int32_t>(L.list_h); f.lval_h = w.at<float>(L.lval_h);
    f.cnt = w.at<int32_t>(L.cnt);
    f.status = w.status();
    f.plan = fp;
    QS_TRY_CUDA(mark(0));
    QS_TRY_CUDA(launch_ffn_fused(f, g_ffn_fused.load() == 2, s));
    for (int i = 1; i < QS_FFN_PHASE_EVENTS; ++i) QS_TRY_CUDA(mark(i));
    return QS_OK;
  }
  const float* unit = nullptr;                   // gate first: a vector of 1.0 (see step 2)
  if (gate_first) QS_TRY_CUDA(unit_vector_on_current_device(&unit, s));

  const int chunk = chunk_tokens(block);
  for (int t0 = 0; t0 < T; t0 += chunk) {
    const int Tc = (T - t0) < chunk ? (T - t0) : chunk;
    const bool timed = (t0 == 0);
    if (timed) QS_TRY_CUDA(mark(0));
    const int blk = Tc > 1 ? block : 1;

    // 1. top-K on |x|
    TopkArgs a;
    a.x = (const unsigned char*)x + (size_t)t0 * d_model * eb;
    a.T = Tc; a.d = d_model; a.k = k_in;
    a.block = blk;
    a.kind = dtype == QS_F32 ? TK_F32 : TK_BF16;
    a.xsf = Tc > 1 ? w.at<float>(L.xsf_x) : nullptr;
    a.list = w.at<int32_t>(L.list_x);
    a.list_val = Tc == 1 ? w.at<float>(L.lval_x) : nullptr;
    a.list_count = w.at<int32_t>(L.cnt) + 0;
    a.ticket = w.ticket(L, kTkTopkX);
    a.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionX));
    a.status = w.status();
    const GemvPlan p_ug =
        plan_gemv(Tc, d_ff, (int)rows_bound(Tc, d_model, d_model), gate_first ? 1 : 2, eb);
    const GemvPlan p_dn = plan_gemv(Tc, d_model, (int)rows_bound_blocks(Tc, d_ff, k_h, blk), 1, eb);
    if (!plan_fits(p_ug, L.parts1_elems, 0) || !plan_fits(p_dn, L.parts2_elems, p_ug.tickets))
      return QS_ERR_UNSUPPORTED;
    a.zero = w.at<float>(L.parts1);
    a.zero_n = p_ug.parts_elems;
    // the nonzero-h counter of step 2 starts at zero (see GemvArgs::hcount)
    const bool h_range_call = Tc == 1 && idx_h_out == nullptr && !gate_first;
    a.zero_word = h_range_call ? w.ticket(L, kTkHCount) : nullptr;
    QS_TRY_CUDA(launch_topk(a, s));
    if (timed) QS_TRY_CUDA(mark(1));

    // 2. up and gate projections over the kept rows, gating epilogue -> h
    float* h = h_out ? h_out + (size_t)t0 * d_ff : w.at<float>(L.h);
    GemvArgs g;
    g.w[0] = wt_up; g.w[1] = wt_gate;
    g.d_in = d_model; g.d_out = d_ff; g.T = Tc;
    g.bf16 = dtype == QS_BF16;
    g.mode = act == QS_ACT_RELU2_GLU ? 1 : 2;
    g.list = a.list; g.list_val = a.list_val; g.xsf = a.xsf; g.list_count = a.list_count;
    g.parts = w.at<float>(L.parts1);
    g.plan = p_ug;
    g.tickets = gemv_tickets(w, L, 0, g.plan);
    g.h = h; g.b_up = b_up; g.b_gate = b_gate;
    g.zero = w.at<float>(L.parts2);
    g.zero_n = p_dn.parts_elems;
    g.status = w.status();
    // one token, list outputs only: the epilogue marks the nonzero h, and the
    // top-K on h starts from that bitmask (it clears it again)
    const bool h_bits = Tc == 1 && idx_h_out == nullptr && topk_bitmask_supported(Tc, d_ff, TK_F32);
    uint32_t* hbits = h_bits ? reinterpret_cast<uint32_t*>(w.ticket(L, kUnionH)) : nullptr;
    // one token: the down projection may take its rows straight from h (see
    // GemvArgs::hcount) when a split's index range fits its row staging
    const bool h_range = h_bits && !gate_first && !p_dn.mma && p_dn.TT == 1 &&
                         (d_ff + p_dn.S - 1) / p_dn.S <= p_dn.rcap;
    int32_t* hcount = h_range ? w.ticket(L, kTkHCount) : nullptr;
    if (!gate_first) {
      g.hbits = hbits;
      g.hcount = hcount;
      QS_TRY_CUDA(launch_gemv(g, s));
    } else {
      // 2a. the gate alone, through the dReLU epilogue: the gate sums sit in
      // the first slot with b_gate, the empty second slot gets a bias of 1,
      // so the epilogue writes ReLU(1) * ReLU(g + b_gate) = ReLU(g + b_gate)
      // to h (exactly) and marks the open gates, over all tokens, in a bitmask
      g.w[0] = wt_gate; g.w[1] = nullptr;
      g.mode = 2;
      g.b_up = b_gate; g.b_gate = unit;
      uint32_t* gate_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kGateBits));
      g.hbits = gate_bits;
      QS_TRY_CUDA(launch_gemv(g, s));
      // 2b. up projection over the open gates' rows of W_up; finishes h
      UpRowsArgs u;
      u.x = a.x; u.T = Tc; u.d_model = d_model; u.d_ff = d_ff;
      u.bf16 = dtype == QS_BF16;
      u.w_up = w_up_rows; u.b_up = b_up;
      u.gate_bits = gate_bits;
      u.ticket = w.ticket(L, kTkUpRows);
      u.h = h;
      u.hbits = hbits;
      u.n_open = w.at<int32_t>(L.cnt) + 2;
      u.status = w.status();
      QS_TRY_CUDA(launch_up_rows(u, s));
    }
    if (timed) QS_TRY_CUDA(mark(2));

    // 3. top-K on |h|
    TopkArgs b;
    b.x = h; b.T = Tc; b.d = d_ff; b.k = k_h; b.kind = TK_F32;
    b.block = blk;
    b.idx = (idx_h_out && k_h > 0) ? idx_h_out + (size_t)t0 * k_h : nullptr;
    b.xsf = Tc > 1 ? w.at<float>(L.xsf_h) : nullptr;
    b.list = w.at<int32_t>(L.list_h);
    b.list_val = Tc == 1 ? w.at<float>(L.lval_h) : nullptr;
    b.list_count = w.at<int32_t>(L.cnt) + 1;
    b.ticket = w.ticket(L, kTkTopkH);
    b.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionH));
    if (h_bits) b.nz_bits = b.union_bits;
    b.early_release = h_range ? 1 : 0;             // the down projection waits for this grid
    b.status = w.status();
    QS_TRY_CUDA(launch_topk(b, s));
    if (timed) QS_TRY_CUDA(mark(3));

    // 4. down projection over the kept nonzero h
    GemvArgs dn;
    dn.w[0] = wt_down;
    dn.d_in = d_ff; dn.d_out = d_model; dn.T = Tc;
    dn.bf16 = dtype == QS_BF16;
    dn.mode = 0;
    dn.list = b.list; dn.list_val = b.list_val; dn.xsf = b.xsf; dn.list_count = b.list_count;
    dn.parts = w.at<float>(L.parts2);
    dn.plan = p_dn;
    dn.tickets = gemv_tickets(w, L, 1, g.plan);
    dn.y = (unsigned char*)y + (size_t)t0 * d_model * eb;
    if (h_range) {
      dn.hcount = hcount;
      dn.hsrc = h;
      dn.k_sel = k_h;
      dn.rows_out = w.at<int32_t>(L.cnt) + 1;
    }
    dn.status = w.status();
    QS_TRY_CUDA(launch_gemv(dn, s));
    if (timed) QS_TRY_CUDA(mark(4));
  }
  return QS_OK;
}

qs_status qs_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                        int k_in, int k_h, const void* wt_up, const void* wt_gate,
                        const float* b_up, const float* b_gate, const void* wt_down, void* y,
                        float* h_out, int32_t* idx_h_out, void* const* phase_events, void* ws,
                        size_t ws_bytes, void* stream) {
  return ffn_impl(QS_OP_SPARSE_FFN, x, dtype, T, d_model, d_ff, act, k_in, k_h, 1, wt_up, nullptr,
                  wt_gate, b_up, b_gate, wt_down, y, h_out, idx_h_out, phase_events, ws, ws_bytes,
                  stream);
}

qs_status qs_sparse_ffn_gate_first(const void* x, int dtype, int T, int d_model, int d_ff,
                                   int k_h, const void* wt_gate, const void* w_up,
                                   const float* b_up, const float* b_gate, const void* wt_down,
                                   void* y, float* h_out, int32_t* idx_h_out,
                                   void* const* phase_events, void* ws, size_t ws_bytes,
                                   void* stream) {
  return ffn_impl(QS_OP_SPARSE_FFN_GATE_FIRST, x, dtype, T, d_model, d_ff, QS_ACT_DRELU, d_model,
                  k_h, 1, nullptr, w_up, wt_gate, b_up, b_gate, wt_down, y, h_out, idx_h_out,
                  phase_events, ws, ws_bytes, stream);
}

static qs_status quant_impl(const void* x, int dtype, int T, int d_in, int d_out, int k, int block,
                            const uint32_t* wt_packed, float alpha, float eps, float* y,
                            int32_t* acc, int8_t* q, int32_t* idx, void* const* phase_events,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!valid_dtype(dtype) || x == nullptr || wt_packed == nullptr || y == nullptr || T < 1 ||
      d_in < 1 || d_out < 1 || k < 0 || k > d_in || !(eps >= 0.0f) || !(alpha == alpha) ||
      block < 1 || block > QS_MAX_BLOCK)
    return QS_ERR_INVALID_ARG;
  if (d_in > QS_MAX_ROW || d_out > QS_MAX_ROW) return QS_ERR_UNSUPPORTED;
  if (block > 1 && !topk_block_supported(d_in)) return QS_ERR_UNSUPPORTED;
  if (!qgemv_supported(d_out) || !aligned16(x) || !aligned16(wt_packed) || !aligned16(y) ||
      !aligned16(acc) || !aligned16(q) || !aligned16(idx))
    return QS_ERR_ALIGNMENT;
  WsLayout L;
  qs_status st = check_ws(QS_OP_QUANT_SPARSE_LINEAR, T, d_in, d_out, k, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  WsView w{(unsigned char*)ws};
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = elem_bytes(dtype);
  auto mark = [&](int i) -> cudaError_t {
    if (phase_events == nullptr) return cudaSuccess;
    return cudaEventRecord((cudaEvent_t)phase_events[i], s);
  };
  const int chunk = chunk_tokens(block);
  for (int t0 = 0; t0 < T; t0 += chunk) {
    const int Tc = (T - t0) < chunk ? (T - t0) : chunk;
    const bool timed = (t0 == 0);
    if (timed) QS_TRY_CUDA(mark(0));
    TopkArgs a;
    a.x = (const unsigned char*)x + (size_t)t0 * d_in * eb;
    a.T = Tc; a.d = d_in; a.k = k;
    a.block = Tc > 1 ? block : 1;
    a.kind = dtype == QS_F32 ? TK_QUANT_F32 : TK_QUANT_BF16;
    a.eps = eps;
    a.idx = (idx && k > 0) ? idx + (size_t)t0 * k : nullptr;
    a.q_full = q ? q + (size_t)t0 * d_in : nullptr;
    a.xq = Tc > 1 ? w.at<int8_t>(L.xq) : nullptr;     // only the union pass reads it
    a.gamma = w.at<float>(L.gamma);
    a.list = w.at<int32_t>(L.list_x);
    a.list_q = Tc == 1 ? w.at<int8_t>(L.lval_x) : nullptr;
    a.list_count = w.at<int32_t>(L.cnt) + 0;
    a.ticket = w.ticket(L, kTkTopkX);
    a.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionX));
    a.status = w.status();
    // 8 or more tokens with per-token selections: their union covers about
    // every input, so the tensor-core kernel streams every packed row
    const GemvPlan qp = (a.block == 1 && qgemv_tc_supported(Tc, d_in, d_out))
                            ? plan_qgemv_tc(Tc, d_in, d_out)
                            : plan_qgemv(Tc, d_out, (int)rows_bound_blocks(Tc, d_in, k, a.block));
    if (!plan_fits(qp, L.parts1_elems, 0)) return QS_ERR_UNSUPPORTED;
    a.zero = w.at<float>(L.parts1);
    a.zero_n = qp.parts_elems;
    QS_TRY_CUDA(launch_topk(a, s));
    if (timed) QS_TRY_CUDA(mark(1));

    QGemvArgs g;
    g.wp = wt_packed; g.d_in = d_in; g.d_out = d_out; g.T = Tc;
    g.gamma = a.gamma; g.alpha = alpha;
    g.list = a.list; g.list_q = a.list_q; g.xq = a.xq; g.list_count = a.list_count;
    g.parts = w.at<float>(L.parts1);
    g.plan = qp;
    g.tickets = w.ticket(L, kTkGemv);
    g.y = y + (size_t)t0 * d_out;
    g.acc = acc ? acc + (size_t)t0 * d_out : nullptr;
    g.status = w.status();
    QS_TRY_CUDA(launch_qgemv(g, s));
    if (timed) QS_TRY_CUDA(mark(2));
  }
  return QS_OK;
}

qs_status qs_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                           const void* wt, void* y, void* const* phase_events, void* ws,
                           size_t ws_bytes, void* stream) {
  return linear_impl(x, dtype, T, d_in, d_out, k, 1, wt, y, phase_events, ws, ws_bytes, stream);
}

qs_status qs_block_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                 int block, const void* wt, void* y, void* const* phase_events,
                                 void* ws, size_t ws_bytes, void* stream) {
  return linear_impl(x, dtype, T, d_in, d_out, k, block, wt, y, phase_events, ws, ws_bytes, stream);
}

qs_status qs_block_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                              int k_in, int k_h, int block, const void* wt_up, const void* wt_gate,
                              const float* b_up, const float* b_gate, const void* wt_down, void* y,
                              float* h_out, int32_t* idx_h_out, void* const* phase_events,
                              void* ws, size_t ws_bytes, void* stream) {
  return ffn_impl(QS_OP_SPARSE_FFN, x, dtype, T, d_model, d_ff, act, k_in, k_h, block, wt_up,
                  nullptr, wt_gate, b_up, b_gate, wt_down, y, h_out, idx_h_out, phase_events, ws,
                  ws_bytes, stream);
}

qs_status qs_quant_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                 const uint32_t* wt_packed, float alpha, float eps, float* y,
                                 int32_t* acc, int8_t* q, int32_t* idx,
                                 void* const* phase_events, void* ws, size_t ws_bytes,
                                 void* stream) {
  return quant_impl(x, dtype, T, d_in, d_out, k, 1, wt_packed, alpha, eps, y, acc, q, idx,
                    phase_events, ws, ws_bytes, stream);
}

qs_status qs_block_quant_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                       int block, const uint32_t* wt_packed, float alpha, float eps,
                                       float* y, int32_t* acc, int8_t* q, int32_t* idx,
                                       void* const* phase_events, void* ws, size_t ws_bytes,
                                       void* stream) {
  return quant_impl(x, dtype, T, d_in, d_out, k, block, wt_packed, alpha, eps, y, acc, q, idx,
                    phase_events, ws, ws_bytes, stream);
}

qs_status qs_sparse_linear_backward(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                    int block, const void* wt, const void* grad_y, float* grad_x,
                                    float* grad_wt, void* ws, size_t ws_bytes, void* stream) {
  WsLayout L;
  qs_status st = qs::check_sparse_linear(x, dtype, T, d_in, d_out, k, wt, grad_y, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  if (block < 1 || block > QS_MAX_BLOCK || (grad_x == nullptr && grad_wt == nullptr))
    return QS_ERR_INVALID_ARG;
  if (block > 1 && !topk_block_supported(d_in)) return QS_ERR_UNSUPPORTED;
  if (!aligned16(grad_x) || !aligned16(grad_wt)) return QS_ERR_ALIGNMENT;
  WsView w{(unsigned char*)ws};
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = elem_bytes(dtype);
  const bool bf16 = dtype == QS_BF16;

  // Many tokens: both gradients are dense contractions on the tensor cores.
  if (bf16 && T >= QS_PREFILL_MIN_T && backward_gemm_supported(T, d_in, d_out) &&
      prefill_supported(T, d_out, d_in)) {
    BackwardGemmArgs g;
    g.grad_y = reinterpret_cast<const __nv_bfloat16*>(grad_y);
    g.wt = reinterpret_cast<const __nv_bfloat16*>(wt);
    g.xs = w.at<__nv_bfloat16>(L.xs_bf16);
    g.grad_x = grad_x; g.grad_wt = grad_wt;
    g.T = T; g.d_in = d_in; g.d_out = d_out;
    g.status = w.status();
    if (grad_wt != nullptr) {
      TopkArgs a;
      a.x = x; a.T = T; a.d = d_in; a.k = k; a.kind = TK_BF16;
      a.block = block;
      a.xs = w.at<void>(L.xs_bf16);
      a.status = w.status();
      QS_TRY_CUDA(launch_topk(a, s));
      QS_TRY_CUDA(launch_grad_wt_gemm(g, s));
    }
    if (grad_x != nullptr) QS_TRY_CUDA(launch_grad_x_gemm(g, s));
    return QS_OK;
  }

  // Decode-size batches: dL/dX by streaming every row of W^T once; dL/dW^T
  // by adding into the rows the top-K listed, chunk by chunk.
  if (grad_wt != nullptr) {
    const int chunk = chunk_tokens(block);
    for (int t0 = 0; t0 < T; t0 += chunk) {
      const int Tc = (T - t0) < chunk ? (T - t0) : chunk;
      TopkArgs a;
      a.x = (const unsigned char*)x + (size_t)t0 * d_in * eb;
      a.T = Tc; a.d = d_in; a.k = k;
      a.block = Tc > 1 ? block : 1;
      a.kind = bf16 ? TK_BF16 : TK_F32;
      a.xsf = Tc > 1 ? w.at<float>(L.xsf_x) : nullptr;
      a.list = w.at<int32_t>(L.list_x);
      a.list_val = Tc == 1 ? w.at<float>(L.lval_x) : nullptr;
      a.list_count = w.at<int32_t>(L.cnt) + 0;
      a.ticket = w.ticket(L, kTkTopkX);
      a.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionX));
      a.status = w.status();
      QS_TRY_CUDA(launch_topk(a, s));
      RowAxpyArgs r;
      r.grad_y = (const unsigned char*)grad_y + (size_t)t0 * d_out * eb;
      r.grad_wt = grad_wt;
      r.list = a.list; r.list_count = a.list_count;
      r.list_val = a.list_val; r.xsf = a.xsf;
      r.T = Tc; r.d_in = d_in; r.d_out = d_out;
      r.bf16 = bf16;
      r.status = w.status();
      QS_TRY_CUDA(launch_rowaxpy(r, s));
    }
  }
  if (grad_x != nullptr) {
    RowDotArgs r;
    r.wt = wt; r.grad_y = grad_y; r.grad_x = grad_x;
    r.T = T; r.d_in = d_in; r.d_out = d_out;
    r.bf16 = bf16;
    r.status = w.status();
    r.plan = plan_rowdot(T, d_in, d_out, eb);
    QS_TRY_CUDA(launch_rowdot(r, s));
  }
  return QS_OK;
}

qs_status qs_quant_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                              int k_in, int k_h, int block, const uint32_t* wp_up, float alpha_up,
                              const uint32_t* wp_gate, float alpha_gate, const uint32_t* wp_down,
                              float alpha_down, float eps, const float* b_up, const float* b_gate,
                              float* y, float* h_out, void* const* phase_events, void* ws,
                              size_t ws_bytes, void* stream) {
  if (!valid_dtype(dtype) || x == nullptr || wp_up == nullptr || wp_gate == nullptr ||
      wp_down == nullptr || y == nullptr || T < 1 || d_model < 1 || d_ff < 1 || k_in < 0 ||
      k_in > d_model || k_h < 0 || k_h > d_ff || !(eps >= 0.0f) || !(alpha_up == alpha_up) ||
      !(alpha_gate == alpha_gate) || !(alpha_down == alpha_down) ||
      (act != QS_ACT_RELU2_GLU && act != QS_ACT_DRELU) || block < 1 || block > QS_MAX_BLOCK)
    return QS_ERR_INVALID_ARG;
  if (d_model > QS_MAX_ROW || d_ff > QS_MAX_ROW) return QS_ERR_UNSUPPORTED;
  if (block > 1 && (!topk_block_supported(d_model) || !topk_block_supported(d_ff)))
    return QS_ERR_UNSUPPORTED;
  if (!qgemv_supported(d_model) || !qgemv_supported(d_ff) || !aligned16(x) || !aligned16(wp_up) ||
      !aligned16(wp_gate) || !aligned16(wp_down) || !aligned16(y) || !aligned16(h_out) ||
      !aligned16(b_up) || !aligned16(b_gate))
    return QS_ERR_ALIGNMENT;
  WsLayout L;
  qs_status st = check_ws(QS_OP_QUANT_SPARSE_FFN, T, d_model, d_ff, k_h, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  WsView w{(unsigned char*)ws};
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = elem_bytes(dtype);
  auto mark = [&](int i) -> cudaError_t {
    if (phase_events == nullptr) return cudaSuccess;
    return cudaEventRecord((cudaEvent_t)phase_events[i], s);
  };
  const int chunk = chunk_tokens(block);
  for (int t0 = 0; t0 < T; t0 += chunk) {
    const int Tc = (T - t0) < chunk ? (T - t0) : chunk;
    const bool timed = (t0 == 0);
    const int blk = Tc > 1 ? block : 1;
    if (timed) QS_TRY_CUDA(mark(0));
    const bool tc_up = blk == 1 && qgemv_tc_supported(Tc, d_model, d_ff);
    const bool tc_dn = blk == 1 && qgemv_tc_supported(Tc, d_ff, d_model);
    const GemvPlan p_up = tc_up ? plan_qgemv_tc(Tc, d_model, d_ff)
                                : plan_qgemv(Tc, d_ff, (int)rows_bound_blocks(Tc, d_model, k_in, blk));
    const GemvPlan p_dn = tc_dn ? plan_qgemv_tc(Tc, d_ff, d_model)
                                : plan_qgemv(Tc, d_model, (int)rows_bound_blocks(Tc, d_ff, k_h, blk));
    if (!plan_fits(p_up, L.parts1_elems, 0) || !plan_fits(p_up, L.parts1_elems, p_up.tickets) ||
        !plan_fits(p_dn, L.parts2_elems, 2 * p_up.tickets))
      return QS_ERR_UNSUPPORTED;

    // 1. quantize x, top-K on |q|
    TopkArgs a;
    a.x = (const unsigned char*)x + (size_t)t0 * d_model * eb;
    a.T = Tc; a.d = d_model; a.k = k_in;
    a.block = blk;
    a.kind = dtype == QS_F32 ? TK_QUANT_F32 : TK_QUANT_BF16;
    a.eps = eps;
    a.xq = Tc > 1 ? w.at<int8_t>(L.xq) : nullptr;
    a.gamma = w.at<float>(L.gamma);
    a.list = w.at<int32_t>(L.list_x);
    a.list_q = Tc == 1 ? w.at<int8_t>(L.lval_x) : nullptr;
    a.list_count = w.at<int32_t>(L.cnt) + 0;
    a.ticket = w.ticket(L, kTkTopkX);
    a.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionX));
    a.zero = w.at<float>(L.parts1);
    a.zero_n = p_up.parts_elems;
    a.status = w.status();
    QS_TRY_CUDA(launch_topk(a, s));
    if (timed) QS_TRY_CUDA(mark(1));

    // 2. up projection -> u; 3. gate projection, its epilogue forms h from u
    float* h = h_out ? h_out + (size_t)t0 * d_ff : w.at<float>(L.h);
    QGemvArgs g;
    g.wp = wp_up; g.d_in = d_model; g.d_out = d_ff; g.T = Tc;
    g.gamma = a.gamma; g.alpha = alpha_up;
    g.list = a.list; g.list_q = a.list_q; g.xq = a.xq; g.list_count = a.list_count;
    g.parts = w.at<float>(L.parts1);
    g.plan = p_up;
    g.tickets = w.ticket(L, kTkGemv);
    g.y = w.at<float>(L.u);
    g.zero = w.at<float>(L.parts1b);
    g.zero_n = p_up.parts_elems;
    g.status = w.status();
    QS_TRY_CUDA(launch_qgemv(g, s));
    g.wp = wp_gate; g.alpha = alpha_gate;
    g.parts = w.at<float>(L.parts1b);
    g.tickets = w.ticket(L, kTkGemv + p_up.tickets);
    g.gating = act == QS_ACT_RELU2_GLU ? 1 : 2;
    g.gate_u = w.at<float>(L.u);
    g.b_up = b_up; g.b_gate = b_gate;
    g.y = h;
    g.zero = nullptr; g.zero_n = 0;
    QS_TRY_CUDA(launch_qgemv(g, s));
    if (timed) QS_TRY_CUDA(mark(2));

    // 4. quantize h, top-K on |q_h|
    TopkArgs b;
    b.x = h; b.T = Tc; b.d = d_ff; b.k = k_h;
    b.block = blk;
    b.kind = TK_QUANT_F32;
    b.eps = eps;
    b.xq = Tc > 1 ? w.at<int8_t>(L.xq_h) : nullptr;
    b.gamma = w.at<float>(L.gamma_h);
    b.list = w.at<int32_t>(L.list_h);
    b.list_q = Tc == 1 ? w.at<int8_t>(L.lval_h) : nullptr;
    b.list_count = w.at<int32_t>(L.cnt) + 1;
    b.ticket = w.ticket(L, kTkTopkH);
    b.union_bits = reinterpret_cast<uint32_t*>(w.ticket(L, kUnionH));
    b.zero = w.at<float>(L.parts2);
    b.zero_n = p_dn.parts_elems;
    b.status = w.status();
    QS_TRY_CUDA(launch_topk(b, s));
    if (timed) QS_TRY_CUDA(mark(3));

    // 5. down projection
    QGemvArgs dn;
    dn.wp = wp_down; dn.d_in = d_ff; dn.d_out = d_model; dn.T = Tc;
    dn.gamma = b.gamma; dn.alpha = alpha_down;
    dn.list = b.list; dn.list_q = b.list_q; dn.xq = b.xq; dn.list_count = b.list_count;
    dn.parts = w.at<float>(L.parts2);
    dn.plan = p_dn;
    dn.tickets = w.ticket(L, kTkGemv + 2 * p_up.tickets);
    dn.y = y + (size_t)t0 * d_model;
    dn.status = w.status();
    QS_TRY_CUDA(launch_qgemv(dn, s));
    if (timed) QS_TRY_CUDA(mark(4));
  }
  return QS_OK;
}

qs_status qs_ternary_pack(const float* wmat, int d_out, int d_in, float eps, uint32_t* wt_packed,
                          float* alpha_out, void* ws, size_t ws_bytes, void* stream) {
  if (wmat == nullptr || wt_packed == nullptr || d_out < 16 || d_in < 1 || !(eps >= 0.0f))
    return QS_ERR_INVALID_ARG;
  if ((d_out % 16) != 0 || !aligned16(wmat) || !aligned16(wt_packed) || !aligned16(alpha_out))
    return QS_ERR_ALIGNMENT;
  WsLayout L;
  qs_status st = check_ws(QS_OP_TERNARY_PACK, 0, d_in, d_out, 0, ws, ws_bytes, &L);
  if (st != QS_OK) return st;
  WsView w{(unsigned char*)ws};
  PackArgs a;
  a.w = wmat; a.d_out = d_out; a.d_in = d_in; a.eps = eps;
  a.packed = wt_packed; a.alpha_out = alpha_out;
  a.alpha_parts = w.at<double>(L.alpha_parts);
  a.alpha_ws = w.at<float>(L.alpha);
  a.ticket = w.ticket(L, kTkAlpha);
  a.status = w.status();
  return from_cuda(launch_ternary_pack(a, (cudaStream_t)stream));
}

}  // extern "C"
