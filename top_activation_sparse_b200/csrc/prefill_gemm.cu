// Prefill masked-dense GEMM: Y = X_sparse . W^T on the tensor cores.
// (Placeholder until the tcgen05 kernel lands: reports "unsupported" so that
// qs_sparse_linear keeps prefill sizes on the gather-GEMV path.)
#include "qs_internal.cuh"

namespace qs {

bool prefill_supported(int, int, int) { return false; }

cudaError_t launch_prefill_gemm(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace qs
