// Gate-first dReLU FFN: the kernels behind qs_sparse_ffn_gate_first.
#pragma once

#include "qs_internal.cuh"

namespace qs {

// Up projection restricted to the open gates.  Row j of the output-major W_up
// ([d_ff, d_model]) is read only where some token has ReLU(g_j + b_gate_j) > 0,
// and h_tj = ReLU(g_tj + b_gate_j) * ReLU(u_tj + b_up_j) is finished in place.
struct UpRowsArgs {
  const void* x = nullptr;         // [T, d_model] f32 / bf16 (dense)
  int T = 0, d_model = 0, d_ff = 0;
  int bf16 = 0;
  const void* w_up = nullptr;      // [d_ff, d_model], same dtype as x
  const float* b_up = nullptr;     // [d_ff] or NULL
  uint32_t* gate_bits = nullptr;   // [ceil(d_ff/32)] open gates (union over the tokens);
                                   // read, then zeroed by the grid's last CTA
  int32_t* ticket = nullptr;       // zero between calls
  float* h = nullptr;              // [T, d_ff] in: ReLU(g + b_gate); out: h
  uint32_t* hbits = nullptr;       // one token: OR the bitmask of nonzero h in here (or NULL)
  int32_t* n_open = nullptr;       // out: number of open gates (W_up rows read), or NULL
  DevStatus* status = nullptr;
};

cudaError_t launch_up_rows(const UpRowsArgs& a, cudaStream_t s);

// Device address of a [QS_MAX_ROW] f32 array of 1.0 on the current device.
// The first call on a device fills it on `s` and waits for `s`.
cudaError_t unit_vector_on_current_device(const float** out, cudaStream_t s);

}  // namespace qs
