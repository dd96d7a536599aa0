/*
 * qs.h -- C ABI of the B200 (sm_100a) Q-Sparse top-K sparse projection library.
 *
 * What the library computes (sources are the pages this project follows):
 *
 *   Q-Sparse news article (zxwl-tech.com), section "Top-K sparsification"
 *   (用Top-K函數實現稀疏化): every linear projection Y = X.W^T takes a
 *   sparsified input.  For each token row x, |x| is ranked, the K largest
 *   entries are kept (K preset), a 0/1 mask M of x's shape marks them, and
 *   X_sparse = X (.) M replaces X in the matmul.  Because most of X_sparse is
 *   zero, only the weight rows of the kept inputs have to be read.
 *
 * Conventions shared by every entry point
 *
 *   Layout.   Activations are row-major [T, d] (T token rows).  Weights are
 *             given INPUT-MAJOR: wt = W^T, row-major [d_in, d_out], so that the
 *             weights of one input feature i are the contiguous row wt[i, :].
 *   Pointers. Every tensor pointer is a CUDA DEVICE pointer owned by the
 *             caller, 16-byte aligned.  The library never allocates or frees
 *             memory and keeps no state between calls; all scratch lives in
 *             the caller's workspace `ws`.
 *   Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *             default stream).  Every call only enqueues work on that stream
 *             and returns; nothing synchronises the host except
 *             qs_device_status() and qs_workspace_stats().
 *   Workspace. `ws` must hold at least qs_workspace_size(op, ...) bytes, be
 *             16-byte aligned and be ZERO-FILLED before its first use
 *             (qs_workspace_init does this).  Each call leaves its internal
 *             counters at zero again when its kernels finish, so a workspace is
 *             reused without clearing.  Calls that share one workspace must be
 *             ordered (same stream, or event-ordered): overlapping them races.
 *   Errors.   Argument errors are detected on the host, before anything is
 *             enqueued, and returned as a qs_status; a failed launch returns
 *             QS_ERR_CUDA.  Conditions only the device can see (a bounded wait
 *             that gave up, an internal check) are recorded in the workspace's
 *             status word and reported by qs_device_status().  No kernel traps.
 *   Ties.     "The K largest |x|" is a total order: larger |x| first, equal |x|
 *             -> lower index first; -0.0 and +0.0 are the same magnitude.  The
 *             mask always has exactly K ones per row, even when fewer than K
 *             entries are nonzero.  Inputs must be finite (NaN ranks above inf).
 *   Numerics. Products accumulate in fp32 (int32 for the int8 x ternary path);
 *             a bf16 output is rounded once, to nearest-even, at the end.  With
 *             bf16 weights and 3 to 64 tokens the projections run on the tensor
 *             cores and the token values enter them rounded to bf16 (the
 *             inputs are bf16 already; the FFN's f32 h is rounded for the
 *             down projection).  Split-K partial sums are added in an order
 *             that is not fixed, so float results may differ in their last
 *             bits between runs; integer results never do.
 */
#ifndef QS_H
#define QS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qs_status {
  QS_OK = 0,
  QS_ERR_INVALID_ARG = 1,   /* bad size, k, enum value, or a required pointer is NULL */
  QS_ERR_ALIGNMENT = 2,     /* pointer not 16-byte aligned, or d_out not a multiple of the
                               16-byte vector width (4 for f32, 8 for bf16; 64 for the
                               packed int8 x ternary projection) */
  QS_ERR_WORKSPACE = 3,     /* ws NULL or smaller than qs_workspace_size() */
  QS_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  QS_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (see qs_device_status) */
  QS_ERR_DEVICE_CHECK = 6,  /* device: an internal consistency check failed */
  QS_ERR_UNSUPPORTED = 7    /* arguments valid but outside what this build handles
                               (e.g. d above QS_MAX_ROW) */
} qs_status;

typedef enum qs_dtype { QS_F32 = 0, QS_BF16 = 1 } qs_dtype;

typedef enum qs_act {
  QS_ACT_RELU2_GLU = 0,   /* h = ReLU(u)^2 * g           (Q-Sparse squared-ReLU FFN) */
  QS_ACT_DRELU = 1        /* h = ReLU(g + b_gate) * ReLU(u + b_up)   (Turbo Sparse dReLU) */
} qs_act;

typedef enum qs_op {
  QS_OP_TOPK_MASK = 0,
  QS_OP_SPARSE_LINEAR = 1,
  QS_OP_SPARSE_FFN = 2,
  QS_OP_QUANT_SPARSE_LINEAR = 3,
  QS_OP_TERNARY_PACK = 4,
  QS_OP_SPARSE_FFN_GATE_FIRST = 5,
  QS_OP_QUANT_SPARSE_FFN = 6
} qs_op;

/* Largest row length (d, d_in, d_ff) a top-K row may have: one CTA holds a
 * row's keys in shared memory. */
#define QS_MAX_ROW 49152
/* From this many tokens on, qs_sparse_linear on bf16 runs the masked-dense
 * tensor-core GEMM instead of the gather-GEMV. */
#define QS_PREFILL_MIN_T 64
/* Largest Block Q-Sparse block (tokens sharing one selection). */
#define QS_MAX_BLOCK 64
/* Number of cudaEvent_t handles qs_sparse_ffn records when given phase events. */
#define QS_FFN_PHASE_EVENTS 5
/* ... and qs_sparse_linear / qs_quant_sparse_linear (before the top-K, after
 * the top-K, after the projection; first chunk of QS_PREFILL_MIN_T tokens). */
#define QS_LINEAR_PHASE_EVENTS 3

/*
 * qs_topk_mask -- top-K on |x| per row, with the mask and the sparsified input.
 *   Source: Q-Sparse news article, section "Top-K sparsification" (rank |X|,
 *   keep the K largest, binary mask M, X_sparse = X (.) M).
 *
 *   x     [T, d] in `dtype` (QS_F32 or QS_BF16), device.
 *   k     0 <= k <= d.  k = d keeps every entry, k = 0 none.
 *   idx   [T, k] int32 out: kept indices of each row, ascending.  Required if k > 0.
 *   val   [T, k] `dtype` out or NULL: x at idx (the compacted value list).
 *   mask  [T, d] uint8 out or NULL: 1 at kept positions, 0 elsewhere.
 *   xs    [T, d] `dtype` out or NULL: X_sparse = x * mask (+0.0 where dropped).
 *   ws    workspace of qs_workspace_size(QS_OP_TOPK_MASK, T, d, 0, k) bytes.
 *   Errors: INVALID_ARG (T < 1, d < 1, k outside [0, d], NULL x/idx, bad dtype),
 *   ALIGNMENT, WORKSPACE, UNSUPPORTED (d > QS_MAX_ROW), CUDA.
 */
qs_status qs_topk_mask(const void* x, int dtype, int T, int d, int k,
                       int32_t* idx, void* val, uint8_t* mask, void* xs,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * qs_sparse_linear -- Y = (X (.) M) . W^T with M the top-K mask of |X|.
 *   Source: Q-Sparse news article, section "Top-K sparsification" (X_sparse
 *   replaces X in the projection; zeros cut compute and memory traffic), and
 *   the aibase.com summary, "Vantagens da ativacao esparsa" (I/O is the
 *   bottleneck of inference, so only the kept inputs' weights are read).
 *
 *   x     [T, d_in] `dtype`.       wt  [d_in, d_out] `dtype` (= W^T).
 *   y     [T, d_out] `dtype` out.  k   0 <= k <= d_in (k = d_in: dense layer).
 *   Decode (T < QS_PREFILL_MIN_T, or f32): a gather-GEMV streams only the rows
 *   wt[i, :] of inputs kept by some token.  Prefill (bf16, T >= QS_PREFILL_MIN_T):
 *   X_sparse is materialised and multiplied on the tensor cores (tcgen05).
 *   d_out must be a multiple of 8 (bf16) or 4 (f32).
 *   phase_events  NULL, or QS_LINEAR_PHASE_EVENTS cudaEvent_t handles (as void*)
 *             recorded on `stream` before the top-K, after it, and after the
 *             projection (timing hook; recording them costs a little).
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                           const void* wt, void* y, void* const* phase_events,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * qs_sparse_ffn -- one sparse gated FFN layer.
 *   x_s = topK(x, k_in);  u = x_s.W_up^T;  g = x_s.W_gate^T;
 *   h   = act(u, g);      h_s = topK(h, k_h);   y = h_s.W_down^T.
 *   Sources: Q-Sparse news article, Top-K section, feed-forward paragraph
 *   (squared ReLU combined by a Hadamard product); aibase.com summary (top-K
 *   on every linear projection); Turbo Sparse summary (blog.csdn.net), Eq. 2
 *   (dReLU) and Eq. 3-4 (top k% of |h| by absolute value before W_down).
 *
 *   x         [T, d_model] `dtype` (bf16 or f32).
 *   act       QS_ACT_RELU2_GLU or QS_ACT_DRELU.
 *   k_in      0..d_model  (d_model = dense input).   k_h  0..d_ff.
 *   wt_up, wt_gate  [d_model, d_ff] `dtype`.   wt_down [d_ff, d_model] `dtype`.
 *   b_up, b_gate    [d_ff] f32 or NULL (= 0); added to u and g before the ReLUs
 *                   of QS_ACT_DRELU; ignored by QS_ACT_RELU2_GLU.
 *   y         [T, d_model] `dtype` out.
 *   h_out     [T, d_ff] f32 out or NULL: h before its top-K.
 *   idx_h_out [T, k_h] int32 out or NULL: indices kept by the top-K on |h|.
 *   phase_events  NULL, or QS_FFN_PHASE_EVENTS cudaEvent_t handles (as void*)
 *             recorded on `stream` before the first kernel and after the input
 *             top-K, the up/gate projection, the top-K on |h| and the down
 *             projection (for per-phase timing; recording them costs a little).
 *             A call that runs as one kernel (qs_sparse_ffn_fused) records the
 *             first event before it and all the others after it.
 *   ws        qs_workspace_size(QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h) bytes.
 *   d_model and d_ff must be multiples of 8 (bf16) or 4 (f32).
 *   One token, bf16, idx_h_out NULL, d_model <= 8192: the whole layer runs as
 *   ONE persistent kernel (every CTA resident, phases separated by grid
 *   barriers) instead of four; same results up to float32 summation order,
 *   same lists and statistics.  qs_set_ffn_fused selects how it is launched
 *   or turns it off.
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                        int k_in, int k_h, const void* wt_up, const void* wt_gate,
                        const float* b_up, const float* b_gate, const void* wt_down,
                        void* y, float* h_out, int32_t* idx_h_out,
                        void* const* phase_events,
                        void* ws, size_t ws_bytes, void* stream);

/* 1 if a qs_sparse_ffn call with these sizes (and idx_h_out given or not)
 * runs as one persistent kernel on the current device, else 0 (also without
 * a device).  Host-only: nothing is enqueued. */
int qs_sparse_ffn_fused(int dtype, int T, int d_model, int d_ff, int with_idx_h);

/* Process-wide switch for the one-kernel path of qs_sparse_ffn:
 *   1 (default) an ordinary launch with programmatic dependent launch: the
 *     next launch's set-up overlaps this one's exit.  Its grid barriers need
 *     every CTA resident, which holds on a device that runs these layers alone
 *     on their stream; another kernel running concurrently on the device can
 *     hold SMs that its CTAs wait for, and a barrier wait that runs out ends in
 *     QS_ERR_TIMEOUT (qs_device_status), never a hang;
 *   2 a cooperative launch, which the driver admits only when the whole grid
 *     can be resident (for callers that overlap other kernels; ~1.7 us more a
 *     launch, launches do not overlap);
 *   0 every call uses the separate kernels (for comparison and testing).
 * Returns QS_ERR_INVALID_ARG for any other value, else QS_OK. */
qs_status qs_set_ffn_fused(int mode);

/*
 * qs_sparse_ffn_gate_first -- the dReLU layer of qs_sparse_ffn (QS_ACT_DRELU,
 *   dense x, k_in = d_model), with the up projection restricted to open gates.
 *   Source: Turbo Sparse summary (blog.csdn.net), Eq. 2: h = ReLU(g + b_gate)
 *   * ReLU(u + b_up) is 0 wherever g + b_gate <= 0, whatever u is.  So the
 *   gate projection runs first (all of W_gate), and row j of W_up is read only
 *   if some token's gate j is open.  Same result as qs_sparse_ffn with
 *   QS_ACT_DRELU and k_in = d_model, up to float32 summation order: an exact
 *   reordering, not an approximation.
 *
 *   x         [T, d_model] `dtype` (bf16 or f32), used dense.
 *   k_h       0..d_ff: top-K on |h| before the down projection.
 *   wt_gate   [d_model, d_ff] `dtype` (= W_gate^T, input-major as in qs_sparse_ffn).
 *   w_up      [d_ff, d_model] `dtype` (= W_up, OUTPUT-major: the nn.Linear layout),
 *             so that the weights of one output column are one contiguous row.
 *   wt_down   [d_ff, d_model] `dtype` (= W_down^T).
 *   b_up, b_gate, y, h_out, idx_h_out, phase_events: as qs_sparse_ffn (the
 *             "up/gate" phase event follows both the gate and the up kernel).
 *   ws        qs_workspace_size(QS_OP_SPARSE_FFN_GATE_FIRST, T, d_model, d_ff, k_h)
 *             bytes.  qs_workspace_stats also reports rows[2] = rows of w_up read.
 *   The first call on a device fills a constant array (a vector of 1.0 used by
 *   the gate's epilogue) and synchronises `stream`: make it before any stream
 *   capture.
 *   d_model and d_ff must be multiples of 8 (bf16) or 4 (f32).
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_sparse_ffn_gate_first(const void* x, int dtype, int T, int d_model, int d_ff,
                                   int k_h, const void* wt_gate, const void* w_up,
                                   const float* b_up, const float* b_gate, const void* wt_down,
                                   void* y, float* h_out, int32_t* idx_h_out,
                                   void* const* phase_events,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * qs_quant_sparse_linear -- BitNet b1.58 + Q-Sparse projection.
 *   Source: Q-Sparse news article, Top-K section, quantized-model paragraphs
 *   (inputs are quantized before top-K, with an epsilon guarding a division;
 *   1-bit weights scaled by alpha = mean|W|).  The lost formulas are read as:
 *     gamma_t = max_j |x_tj| + eps;  s_t = 127 / gamma_t;
 *     q_tj    = clamp(rint(x_tj * s_t), -127, 127)          (float32 steps)
 *     keep    = topK(|q_t|, k)  (ties -> lower index)
 *     acc_tj  = sum_{i in keep} q_ti * t_ij                  (exact int32)
 *     y_tj    = float(acc_tj) * ((alpha * gamma_t) / 127)    (float32 steps)
 *
 *   x          [T, d_in] `dtype` (bf16 or f32).
 *   wt_packed  [d_in, d_out/16] uint32: ternary W^T from qs_ternary_pack.
 *   alpha      the weight scale qs_ternary_pack returned.   eps  e.g. 1e-5.
 *   y          [T, d_out] f32 out.
 *   acc        [T, d_out] int32 out or NULL.   q  [T, d_in] int8 out or NULL.
 *   idx        [T, k] int32 out or NULL: kept indices, ascending.
 *   phase_events  NULL or QS_LINEAR_PHASE_EVENTS events (as qs_sparse_linear).
 *   d_out must be a multiple of 64 (whole packed rows move in 16-byte bulk
 *   copies); 127 * d_in < 2^24 keeps float(acc) exact.
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_quant_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                 const uint32_t* wt_packed, float alpha, float eps,
                                 float* y, int32_t* acc, int8_t* q, int32_t* idx,
                                 void* const* phase_events,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * qs_ternary_pack -- ternary weight quantizer and 2-bit packing (offline step).
 *   Source: Q-Sparse news article, quantized-model paragraph (alpha is the
 *   mean absolute value of W).  Read as:
 *     alpha = float(sum |W| in fp64 / (d_out * d_in));
 *     t     = clamp(rint(W / (alpha + eps)), -1, 1)   (float32 division)
 *   Packing: word [i, j/16] of the output holds t[j, i] at bits 2*(j%16),
 *   code 00 = 0, 01 = +1, 10 = -1.
 *
 *   w          [d_out, d_in] f32 (output-major, as nn.Linear stores it).
 *   wt_packed  [d_in, d_out/16] uint32 out.    alpha_out  1 f32 out (device).
 *   d_out must be a multiple of 16.
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, CUDA.
 */
qs_status qs_ternary_pack(const float* w, int d_out, int d_in, float eps,
                          uint32_t* wt_packed, float* alpha_out,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * Block Q-Sparse: the three projections above with one selection per block of
 * tokens instead of one per token.
 *   Source: Q-Sparse paper summary (shd-paper.top), abstract ("Block Q-Sparse
 *   for batch training and inference") and method section, key design 3
 *   (splitting the activations into blocks uses the hardware better in
 *   batches).  The pages give no mechanism; this library reads it as:
 *     the T token rows are cut into blocks of `block` consecutive rows (the
 *     last may be shorter); a block ranks feature i by its block magnitude
 *     s_i = max over the block's rows of |x_ti| (ties -> lower index, -0 == +0)
 *     and keeps the k largest; every row of the block keeps those k features.
 *   So a block's projection reads at most k weight rows however many tokens
 *   it holds, where per-token selections read the union of theirs.  block = 1
 *   is the per-token entry point exactly.
 *
 *   block  1..QS_MAX_BLOCK.  Rows (d_in; d_model and d_ff) of more than 16384
 *          features with block > 1 return QS_ERR_UNSUPPORTED.
 *   Every other argument, output and error is that of the per-token entry
 *   point; idx / idx_h_out rows of one block are equal.  For the FFN the same
 *   block size applies to the top-K on |x| and to the top-K on |h|.  Tokens
 *   run in chunks of whole blocks (at most QS_PREFILL_MIN_T tokens), and
 *   qs_sparse_linear's prefill path (bf16, T >= QS_PREFILL_MIN_T) multiplies
 *   the block-masked X_sparse on the tensor cores.
 *   Workspace: qs_workspace_size of the per-token op with the same sizes.
 */
qs_status qs_block_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                 int block, const void* wt, void* y, void* const* phase_events,
                                 void* ws, size_t ws_bytes, void* stream);
qs_status qs_block_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                              int k_in, int k_h, int block, const void* wt_up, const void* wt_gate,
                              const float* b_up, const float* b_gate, const void* wt_down, void* y,
                              float* h_out, int32_t* idx_h_out, void* const* phase_events,
                              void* ws, size_t ws_bytes, void* stream);
qs_status qs_block_quant_sparse_linear(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                       int block, const uint32_t* wt_packed, float alpha, float eps,
                                       float* y, int32_t* acc, int8_t* q, int32_t* idx,
                                       void* const* phase_events, void* ws, size_t ws_bytes,
                                       void* stream);

/*
 * qs_sparse_linear_backward -- gradients of Y = X_sparse . W^T under the
 *   straight-through estimator.
 *   Source: Q-Sparse news article, section "Top-K sparsification", the
 *   straight-through-estimator paragraphs: top-K has a zero gradient almost
 *   everywhere, so the gradient with respect to the sparsified input is used
 *   unchanged as the gradient with respect to the input:
 *     grad_x  = grad_y . W               [T, d_in]   (no mask applied)
 *     grad_wt += X_sparse^T . grad_y     [d_in, d_out]
 *   X_sparse is the forward's: top-K on |x| per token (block = 1) or per
 *   block of tokens (Block Q-Sparse, block > 1), k kept.
 *
 *   x, dtype, T, d_in, d_out, k, block, wt: as qs_block_sparse_linear.
 *   grad_y   [T, d_out] `dtype`: dL/dY.
 *   grad_x   [T, d_in] f32 out, or NULL: overwritten.
 *   grad_wt  [d_in, d_out] f32, or NULL: ACCUMULATED into.  Only rows of
 *            inputs that some token kept with a nonzero value are read and
 *            written; within them an element whose added sum is exactly zero
 *            is left as it was.  Rows no token kept are never touched.
 *   At least one of grad_x, grad_wt.  With bf16, T >= QS_PREFILL_MIN_T and
 *   d_in, d_out multiples of 8, both run as tcgen05 GEMMs (bf16 operands, f32
 *   accumulation); otherwise grad_x streams W^T once per 8 tokens and grad_wt
 *   adds into the kept rows only.
 *   ws       qs_workspace_size(QS_OP_SPARSE_LINEAR, T, d_in, d_out, k) bytes.
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_sparse_linear_backward(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                    int block, const void* wt, const void* grad_y, float* grad_x,
                                    float* grad_wt, void* ws, size_t ws_bytes, void* stream);

/*
 * qs_quant_sparse_ffn -- BitNet b1.58 + Q-Sparse FFN layer: every projection
 *   input is quantized per token and sparsified before an int8 x ternary
 *   projection.
 *   Sources: Q-Sparse news article, Top-K section, quantized-model paragraphs
 *   (quantize before top-K; ternary weights scaled by mean|W|) and
 *   feed-forward paragraph (squared ReLU, Hadamard product); aibase.com
 *   summary (top-K on every linear projection); Turbo Sparse summary, Eq. 2
 *   (dReLU).  Read as, each step exact integer arithmetic or a float32 step:
 *     q_x = quantize(x) (as qs_quant_sparse_linear);  keep = topK(|q_x|, k_in)
 *     u = int8 x ternary(q_x, up),  g = int8 x ternary(q_x, gate)   (float32)
 *     relu2_glu: r = max(u, 0); h = (r * r) * g
 *     drelu:     h = max(g + b_gate, 0) * max(u + b_up, 0)
 *     q_h = quantize(h);  keep_h = topK(|q_h|, k_h);  y = int8 x ternary(q_h, down)
 *   so y is defined bit for bit.  block > 1: Block Q-Sparse selections on |q_x|
 *   and |q_h| (see qs_block_sparse_linear); block = 1 is per token.
 *
 *   x         [T, d_model] `dtype` (bf16 or f32).
 *   wp_up, wp_gate  [d_model, d_ff/16] packed ternary W^T (qs_ternary_pack),
 *             alpha_up, alpha_gate their scales.   wp_down [d_ff, d_model/16], alpha_down.
 *   b_up, b_gate    [d_ff] f32 or NULL (dReLU only).
 *   y         [T, d_model] f32 out.    h_out  [T, d_ff] f32 out or NULL.
 *   phase_events  NULL or QS_FFN_PHASE_EVENTS events (as qs_sparse_ffn).
 *   ws        qs_workspace_size(QS_OP_QUANT_SPARSE_FFN, T, d_model, d_ff, k_h) bytes.
 *   d_model and d_ff must be multiples of 64; 127 * d_model and 127 * d_ff < 2^24.
 *   Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED, CUDA.
 */
qs_status qs_quant_sparse_ffn(const void* x, int dtype, int T, int d_model, int d_ff, int act,
                              int k_in, int k_h, int block, const uint32_t* wp_up, float alpha_up,
                              const uint32_t* wp_gate, float alpha_gate, const uint32_t* wp_down,
                              float alpha_down, float eps, const float* b_up, const float* b_gate,
                              float* y, float* h_out, void* const* phase_events, void* ws,
                              size_t ws_bytes, void* stream);

/* Bytes of workspace `op` needs for these sizes (0 if the sizes are invalid).
 * Arguments: QS_OP_TOPK_MASK (T, d, 0, k); QS_OP_SPARSE_LINEAR (T, d_in, d_out,
 * k); QS_OP_SPARSE_FFN, QS_OP_SPARSE_FFN_GATE_FIRST and QS_OP_QUANT_SPARSE_FFN (T,
 * d_model, d_ff, k_h);
 * QS_OP_QUANT_SPARSE_LINEAR (T, d_in, d_out, k); QS_OP_TERNARY_PACK (0, d_in,
 * d_out, 0).  The dtype does
 * not change the size, and a workspace of this size also serves calls with the
 * same sizes and any other k. */
size_t qs_workspace_size(int op, int T, int d_in, int d_out, int k);

/* Zero-fill `ws_bytes` of workspace on `stream` (enqueued, not synchronous). */
qs_status qs_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the workspace's device status word.
 * Returns QS_OK, QS_ERR_TIMEOUT or QS_ERR_DEVICE_CHECK (or QS_ERR_CUDA). */
qs_status qs_device_status(void* ws, void* stream);

/* Synchronise `stream` and report, for the last call of `op` made with this
 * workspace and these sizes, how many weight rows its projections streamed:
 * rows[0] = distinct inputs with a kept nonzero value across the T tokens (the
 * rows of wt / wt_up / wt_gate read), rows[1] = the same for h (rows of
 * wt_down read; the FFN ops only, else 0), and for
 * QS_OP_SPARSE_FFN_GATE_FIRST only (then `rows` holds 3) rows[2] = open gates
 * across the T tokens (the rows of w_up read).  These counts are the
 * algorithmic weight traffic: rows * row length * sizeof(weight). */
qs_status qs_workspace_stats(const void* ws, int op, int T, int d_in, int d_out, int k,
                             int32_t* rows, void* stream);

/* Synchronise `stream` and copy to HOST memory the kept-row list that the
 * last call of `op` made with this workspace and these sizes left in it (for
 * inspection and tests; the two FFN ops report their last chunk of at most
 * QS_PREFILL_MIN_T tokens).
 *   which  0: the projection input's list: the inputs with a kept nonzero
 *             value (rows of wt, wt_up / wt_gate or wt_packed that were read),
 *             ascending, the union over the tokens;
 *          1: (QS_OP_SPARSE_FFN, QS_OP_SPARSE_FFN_GATE_FIRST,
 *             QS_OP_QUANT_SPARSE_FFN) the same for h (rows of wt_down read).
 *   rows   host int32 [cap] out: the first min(count, cap) listed rows.
 *   vals   host out or NULL: for calls with one token (T == 1) the listed
 *          rows' values, in list order: float32 (the kept x, exactly as given;
 *          the kept h) or, for QS_OP_QUANT_SPARSE_LINEAR and
 *          QS_OP_QUANT_SPARSE_FFN, the int8 codes.
 *          Must be NULL when T > 1 (several tokens keep dense masked values).
 *   count  host out: the number of listed rows.
 * Errors: INVALID_ARG (bad op/which/sizes, NULL rows/count, vals with T > 1),
 * CUDA. */
qs_status qs_workspace_list(const void* ws, int op, int T, int d_in, int d_out, int k, int which,
                            int32_t* rows, int cap, void* vals, int32_t* count, void* stream);

/* Failure-detection test hook (host side; process-wide; not thread-safe).
 * QS_FAULT_GATHER_NO_COPIES makes the gather-GEMV launches that follow (the
 * FMA kernel that serves one or two tokens, and the one-kernel FFN layer of
 * qs_sparse_ffn) issue no weight copies at all:
 * their producer warp stays idle, so no copy is ever in flight, and the
 * consumers' bounded waits run out after `wait_polls` polls (0: the normal
 * limit).  The kernel then records QS_ERR_TIMEOUT in the workspace's status
 * word, skips its remaining waits and still finishes its split sums and
 * tickets, so the workspace stays usable; its results are meaningless.
 * QS_FAULT_NONE restores normal operation.  Nothing here faults or hangs the
 * GPU.  Errors: INVALID_ARG (unknown mode). */
typedef enum qs_fault { QS_FAULT_NONE = 0, QS_FAULT_GATHER_NO_COPIES = 1 } qs_fault;
qs_status qs_debug_inject(int mode, unsigned wait_polls);

/* Human-readable name of a status code (static string). */
const char* qs_status_string(int status);

/* Device state kept per process: the library caches, per device ordinal, the
 * address of two static device arrays (a vector of 1.0 used by the gate-first
 * FFN, and the scratch array of qs_sparse_linear_noalloc).  cudaDeviceReset
 * (or any new primary context on a device) invalidates them and is not
 * supported while the library is in use in the process. */

/* Size of the fixed device scratch array behind qs_sparse_linear_noalloc. */
#define QS_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * qs_sparse_linear_noalloc -- qs_sparse_linear without a caller workspace.
 *   The pages have no counterpart to this: it exists for callers that may not
 *   allocate device memory (an op slot inside a framework that owns every
 *   allocation, a service that freezes its memory after start-up, a plugin
 *   without access to the host process's allocator).  Arguments and results
 *   are those of qs_sparse_linear; the scratch space comes from one
 *   QS_NOALLOC_SCRATCH_BYTES array built into the library, which every GPU
 *   that loads the library holds until the process exits.
 *
 *   - Nothing is allocated or freed, by this call or by anything it calls.
 *   - The first call on a device looks the array's address up for that device
 *     (cudaGetSymbolAddress), so make that first call before any stream
 *     capture.
 *   - Every argument check of qs_sparse_linear runs first; an invalid call
 *     returns its code with nothing enqueued.  A valid call then clears the
 *     array's counters on `stream` (cudaMemsetAsync); the rest of the array
 *     is rewritten before it is read.
 *   - All calls share the array: calls whose kernels can overlap on the GPU
 *     (different streams without ordering) race and give wrong results.
 *   - Device-side failures (a bounded wait that gave up, an internal check)
 *     go to the array's status word, which keeps the first one until
 *     qs_sparse_linear_noalloc_status reads it.
 *   - Errors: as qs_sparse_linear, plus QS_ERR_UNSUPPORTED when these sizes
 *     need more than QS_NOALLOC_SCRATCH_BYTES of scratch (that is,
 *     qs_workspace_size(QS_OP_SPARSE_LINEAR, T, d_in, d_out, k) is larger),
 *     returned before anything is enqueued.
 */
qs_status qs_sparse_linear_noalloc(const void* x, int dtype, int T, int d_in, int d_out, int k,
                                   const void* wt, void* y, void* stream);

/* Synchronise `stream`, then read and clear the status word of the current
 * device's fixed scratch array (the qs_device_status of
 * qs_sparse_linear_noalloc): QS_OK, QS_ERR_TIMEOUT or QS_ERR_DEVICE_CHECK for
 * the calls since the last read (or QS_ERR_CUDA).  Allocates nothing. */
qs_status qs_sparse_linear_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QS_H */
