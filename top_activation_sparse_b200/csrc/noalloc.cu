// qs_sparse_linear_noalloc: qs_sparse_linear for callers that cannot allocate.
//
// Some callers are not allowed to allocate device memory at all: code that
// runs inside a framework which owns every allocation (a custom-op slot with
// no allocator handle), long-lived services that forbid allocation after
// start-up so that memory use stays fixed, or plugins loaded into a process
// whose allocator they cannot reach.  For them the scratch space the
// projection needs lives in a fixed array that is part of this library's own
// device image.  The caller still owns x, W^T and y.
//
// The array is QS_NOALLOC_SCRATCH_BYTES on every GPU that loads the library
// and stays there until the process exits.  All calls share it, and it keeps
// whatever the last call left in it: the counters that must start at zero are
// cleared at the start of every call (a memset on the caller's stream, after
// every argument check has passed), the rest is overwritten before it is read.
// The status word is not cleared by a call: like a workspace's, it keeps the
// first device-side failure until qs_sparse_linear_noalloc_status reads it.
// Two calls whose kernels overlap on the GPU (different streams, no ordering)
// race on it.
#include <mutex>

#include "qs_internal.cuh"

namespace {

constexpr size_t kScratchBytes = QS_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the name
// g_scratch only stands for the symbol; the address has to be looked up once
// per device, with that device current.
qs_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return QS_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return QS_OK;
}

}  // namespace

extern "C" qs_status qs_sparse_linear_noalloc(const void* x, int dtype, int T, int d_in, int d_out,
                                              int k, const void* wt, void* y, void* stream) {
  if (x == nullptr || wt == nullptr || y == nullptr) return QS_ERR_INVALID_ARG;
  const size_t need = qs_workspace_size(QS_OP_SPARSE_LINEAR, T, d_in, d_out, k);
  if (need == 0) return QS_ERR_INVALID_ARG;
  if (need > kScratchBytes) return QS_ERR_UNSUPPORTED;   // sizes beyond the fixed scratch
  // every argument check of qs_sparse_linear first (with no workspace yet, so
  // only the missing workspace may be reported): an invalid call enqueues nothing
  qs::WsLayout L;
  qs_status st = qs::check_sparse_linear(x, dtype, T, d_in, d_out, k, wt, y, nullptr, 0, &L);
  if (st != QS_ERR_WORKSPACE) return st == QS_OK ? QS_ERR_CUDA : st;
  void* ws = nullptr;
  st = scratch_on_current_device(&ws);
  if (st != QS_OK) return st;
  // the counters (between the status word and the per-call buffers) start at zero
  if (cudaMemsetAsync((unsigned char*)ws + L.tickets, 0, L.cnt - L.tickets, (cudaStream_t)stream) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  return qs_sparse_linear(x, dtype, T, d_in, d_out, k, wt, y, nullptr, ws, kScratchBytes, stream);
}

extern "C" qs_status qs_sparse_linear_noalloc_status(void* stream) {
  void* ws = nullptr;
  const qs_status st = scratch_on_current_device(&ws);
  if (st != QS_OK) return st;
  return qs_device_status(ws, stream);
}
