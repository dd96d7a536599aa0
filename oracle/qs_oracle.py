"""CPU oracle for the Q-Sparse top-K sparse projection path.

TEST INFRASTRUCTURE.  This module is the slow, plain definition that the CUDA
path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference`` arm) may import
it.  It shares no code with ``top_activation_sparse_b200`` and imports nothing
from it; the product never calls it.

What it computes, and where each step comes from:

* Q-Sparse news article (zxwl-tech.com), section "用Top-K函數實現稀疏化"
  (Top-K sparsification): the linear layer Y = X.W^T of attention and FFN
  takes a sparsified input; |X| is computed and sorted, the K largest entries
  are kept, a 0/1 mask M of X's shape marks them, X_sparse = X (.) M, and
  X_sparse replaces X in the matmul.  K is a preset hyperparameter.
  -> :func:`topk_keep`, :func:`topk_mask`, :func:`sparse_linear`.
* same section, the paragraph on the feed-forward layer: squared ReLU replaces
  ReLU and is combined with a Hadamard product (the formula itself was lost in
  extraction).  Reading used: h = ReLU(x_s.W_up^T)^2 (.) (x_s.W_gate^T), then
  top-K on |h| and y = h_s.W_down^T, because the aibase.com summary
  ("Vantagens da ativacao esparsa") says top-K is applied to every linear
  projection.  -> :func:`sparse_ffn` with act="relu2_glu".
* Turbo Sparse summary (blog.csdn.net), Eq. 2 (dReLU: ReLU after both the gate
  and the up projection) and Eq. 3-4 (keep the top k% of the activation output
  by absolute value, then apply W_down).  Reading used:
  h = ReLU(x.W_gate^T + b_gate) (.) ReLU(x.W_up^T + b_up).
  -> :func:`sparse_ffn` with act="drelu".
* Q-Sparse paper summary (shd-paper.top), abstract and method section (key
  design 3): Block Q-Sparse for batched training and inference, by splitting
  the activations into blocks.  No mechanism survives on the pages; reading
  used: blocks of consecutive tokens share one selection, the k features with
  the largest block magnitude max_t |x_ti|.  -> :func:`block_topk_keep` (its
  result is passed as ``keep`` / ``keep_h`` to the projection and FFN oracles).
* Q-Sparse news article, the same Top-K section, the paragraphs on the
  straight-through estimator (STE): top-K
  has zero gradient almost everywhere, so the loss gradient with respect to
  the sparsified tensor is copied unchanged to the tensor before it was
  sparsified.  -> :func:`sparse_linear_backward_ste` (the backward of
  :func:`sparse_linear`; no CUDA kernel implements it yet).
* Q-Sparse news article, same section, the paragraph on quantized models: the
  input is quantized before top-K, with a small epsilon that keeps a
  denominator away from zero, and 1-bit weights use alpha = mean|W| (both
  formulas lost).  Readings used (per-token absmax int8, ternary round-clip):
  :func:`absmax_quantize`, :func:`ternary_quantize`, :func:`quant_sparse_linear`;
  the quantized FFN layer built from them, with the gating in float32 steps:
  :func:`ffn_hidden_f32`, :func:`quant_sparse_ffn`.

Readings of what the pages leave open:

* order of "the K largest |X|": larger |x| first; equal |x| -> lower index
  first; -0.0 and +0.0 are the same magnitude.  Kept indices are reported in
  ascending order.  Inputs must be finite.
* K counts *selected* positions: the mask has exactly K ones even when fewer
  than K entries are nonzero (h after ReLU), so nnz(X_sparse) <= K.
* floating point: fp64 everywhere except the two quantizers, which are defined
  as float32 IEEE round-to-nearest-even steps in a fixed order (so that their
  integer outputs are reproducible bit for bit):
      gamma = amax + eps;  s = 127 / gamma;  q = clamp(rint(x * s), -127, 127)
      alpha = float32(sum|W| in fp64 / N);  t = clamp(rint(W / (alpha + eps)), -1, 1)
      r = (alpha * gamma) / 127;  y = float32(acc) * r
* the int8 x ternary accumulator is exact (int64 here); float32(acc) is exact
  while |acc| < 2^24, i.e. 127 * d_in < 2^24.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# top-K on |x|  (Q-Sparse article, Top-K sparsification section)
# --------------------------------------------------------------------------


def topk_keep(x, k: int) -> np.ndarray:
    """Indices kept by top-K on |x|, per row, ascending.  int64 [T, k].

    Full sort of every row by (|x| descending, index ascending), first k taken.
    """
    x = np.asarray(x)
    if x.ndim != 2:
        raise ValueError("x must be [T, d]")
    T, d = x.shape
    if not 0 <= k <= d:
        raise ValueError(f"k={k} outside [0, {d}]")
    mag = np.abs(x.astype(np.float64))
    if not np.all(np.isfinite(mag)):
        raise ValueError("top-K oracle takes finite inputs only")
    # A stable sort of -|x| keeps equal magnitudes in index order, which is the
    # lower-index-first tie rule.
    order = np.argsort(-mag, axis=1, kind="stable")
    return np.sort(order[:, :k], axis=1)


def block_topk_keep(x, k: int, block: int) -> np.ndarray:
    """Block Q-Sparse selection: int64 [T, k] kept indices per token.

    Q-Sparse paper summary (shd-paper.top), abstract and method section (key
    design 3): Block Q-Sparse splits the activations into blocks so that
    batched training and inference use the hardware well.  The pages give no
    mechanism; this library's reading: the T token rows are cut into blocks of
    `block` consecutive rows (the last one may be shorter); a block ranks its
    features by the block magnitude s_i = max over the block's rows of |x_ti|
    and keeps the k largest (ties -> lower index, as for one token); every row
    of the block keeps those same k features.  block = 1 is per-token top-K.
    """
    x = np.asarray(x)
    if x.ndim != 2:
        raise ValueError("x must be [T, d]")
    if block < 1:
        raise ValueError("block must be >= 1")
    T, d = x.shape
    keep = np.zeros((T, k), dtype=np.int64)
    for b0 in range(0, T, block):
        rows = slice(b0, min(T, b0 + block))
        s = np.max(np.abs(x[rows].astype(np.float64)), axis=0)   # block magnitude per feature
        keep[rows] = topk_keep(s[None, :], k)[0]
    return keep


def mask_from_keep(keep: np.ndarray, T: int, d: int) -> np.ndarray:
    """Binary mask M [T, d] (uint8) with ones at the kept positions."""
    m = np.zeros((T, d), dtype=np.uint8)
    rows = np.repeat(np.arange(T), keep.shape[1])
    m[rows, keep.reshape(-1)] = 1
    return m


def topk_mask(x, k: int):
    """(keep [T,k] int64, mask [T,d] uint8, x_sparse [T,d] float64) for top-K on |x|."""
    x = np.asarray(x)
    keep = topk_keep(x, k)
    m = mask_from_keep(keep, *x.shape)
    xs = x.astype(np.float64) * m          # Hadamard product with the mask
    return keep, m, xs


def kept_values(x, keep: np.ndarray) -> np.ndarray:
    """x[t, keep[t, j]] in the input's own dtype (the compacted value list)."""
    x = np.asarray(x)
    return np.take_along_axis(x, keep, axis=1)


# --------------------------------------------------------------------------
# sparse linear projection  Y = (X (.) M) . W^T
# --------------------------------------------------------------------------


def sparse_linear(x, wt, k: int, keep: np.ndarray | None = None) -> np.ndarray:
    """Y [T, d_out] float64 = X_sparse . W^T with W^T given input-major [d_in, d_out].

    The mask multiply is applied to the whole of X and the product uses all of
    W^T: the oracle does not skip anything.  ``keep`` overrides the top-K
    selection (used to re-run the projection on a selection made elsewhere).
    """
    x = np.asarray(x)
    wt = np.asarray(wt, dtype=np.float64)
    T, d_in = x.shape
    if wt.shape[0] != d_in:
        raise ValueError("W^T must be [d_in, d_out]")
    if keep is None:
        keep = topk_keep(x, k)
    m = mask_from_keep(keep, T, d_in)
    xs = x.astype(np.float64) * m
    return xs @ wt


def sparse_linear_backward_ste(x, wt, k: int, grad_y, keep: np.ndarray | None = None) -> dict:
    """Gradients of Y = X_sparse . W^T for an upstream gradient dL/dY [T, d_out].

    Q-Sparse news article, section "Top-K sparsification", STE paragraphs: the
    gradient with respect to the sparsified tensor is used as the gradient
    with respect to the tensor before sparsification.  With W^T input-major:

        dL/dX_sparse = dL/dY . (W^T)^T          [T, d_in]
        dL/dX       := dL/dX_sparse             (the estimator: no mask applied)
        dL/dW^T      = X_sparse^T . dL/dY        [d_in, d_out]

    A row i of dL/dW^T can be nonzero only if some token kept input i, so a
    backward pass needs to write only the kept rows.  All fp64.
    """
    x = np.asarray(x)
    wt = np.asarray(wt, dtype=np.float64)
    g = np.asarray(grad_y, dtype=np.float64)
    T, d_in = x.shape
    if wt.shape[0] != d_in or g.shape != (T, wt.shape[1]):
        raise ValueError("need x [T, d_in], W^T [d_in, d_out], dL/dY [T, d_out]")
    if keep is None:
        keep = topk_keep(x, k)
    xs = x.astype(np.float64) * mask_from_keep(keep, T, d_in)
    return {"grad_x": g @ wt.T, "grad_wt": xs.T @ g, "keep": keep}


# --------------------------------------------------------------------------
# sparse FFN: squared-ReLU GLU (Q-Sparse) and dReLU (Turbo Sparse)
# --------------------------------------------------------------------------


def relu(v):
    return np.maximum(v, 0.0)


def ffn_hidden(u, g, act: str, b_up=None, b_gate=None):
    """The gating epilogue h from the two projections u (up) and g (gate)."""
    if act == "relu2_glu":
        # squared ReLU on the up branch, Hadamard product with the gate branch
        return relu(u) ** 2 * g
    if act == "drelu":
        bu = 0.0 if b_up is None else np.asarray(b_up, dtype=np.float64)
        bg = 0.0 if b_gate is None else np.asarray(b_gate, dtype=np.float64)
        # ReLU after both the gate and the up projection
        return relu(g + bg) * relu(u + bu)
    raise ValueError(f"unknown activation {act!r}")


def sparse_ffn(x, wt_up, wt_gate, wt_down, act: str, k_in: int, k_h: int,
               b_up=None, b_gate=None, keep_h: np.ndarray | None = None,
               block: int = 1) -> dict:
    """One sparse FFN layer.

    x_s = topK(x, k_in);  u = x_s.W_up^T;  g = x_s.W_gate^T;  h = act(u, g);
    h_s = topK(h, k_h);   y = h_s.W_down^T.    All fp64.

    ``keep_h`` overrides the top-K on |h| (the CUDA path computes h in fp32, so
    near the threshold its selection may legitimately differ; the projection is
    then re-run here on that selection).  ``block`` > 1 selects with Block
    Q-Sparse (:func:`block_topk_keep`) on x and on h.
    """
    x = np.asarray(x)
    T, d_model = x.shape
    wt_up = np.asarray(wt_up, dtype=np.float64)
    wt_gate = np.asarray(wt_gate, dtype=np.float64)
    wt_down = np.asarray(wt_down, dtype=np.float64)
    d_ff = wt_up.shape[1]
    keep_x = block_topk_keep(x, k_in, block)
    xs = x.astype(np.float64) * mask_from_keep(keep_x, T, d_model)
    u = xs @ wt_up
    g = xs @ wt_gate
    h = ffn_hidden(u, g, act, b_up, b_gate)
    keep_h_own = block_topk_keep(h, k_h, block)
    kh = keep_h_own if keep_h is None else np.asarray(keep_h)
    hs = h * mask_from_keep(kh, T, d_ff)
    y = hs @ wt_down
    return {"y": y, "h": h, "u": u, "g": g, "keep_x": keep_x, "keep_h": keep_h_own,
            "hs": hs}


# --------------------------------------------------------------------------
# BitNet b1.58 + Q-Sparse: int8 activations, ternary weights
# --------------------------------------------------------------------------


def absmax_quantize(x, eps: float = 1e-5):
    """Per-token absmax int8 quantizer (float32 steps, fixed order).

    gamma_t = max_j |x_tj| + eps;  s_t = 127 / gamma_t;
    q_tj = clamp(rint(x_tj * s_t), -127, 127)      (rint = nearest-even)
    Returns (q int64 [T, d], gamma float32 [T]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    if x32.ndim != 2:
        raise ValueError("x must be [T, d]")
    amax = np.max(np.abs(x32), axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    gamma = (amax + np.float32(eps)).astype(np.float32)
    s = (np.float32(127.0) / gamma).astype(np.float32)
    q = np.clip(np.rint(x32 * s[:, None]), -127, 127).astype(np.int64)
    return q, gamma


def ternary_quantize(w, eps: float = 1e-5):
    """Ternary weight quantizer with alpha = mean|W|.

    alpha = float32(sum|W| (fp64) / N);  t = clamp(rint(W / (alpha + eps)), -1, 1)
    with the division in float32.  Returns (t int8 [d_out, d_in], alpha float32).
    """
    w32 = np.asarray(w, dtype=np.float32)
    alpha = np.float32(np.sum(np.abs(w32.astype(np.float64))) / w32.size)
    denom = np.float32(alpha + np.float32(eps))
    t = np.clip(np.rint(w32 / denom), -1, 1).astype(np.int8)
    return t, alpha


# 2-bit code per weight: 00 -> 0, 01 -> +1, 10 -> -1 (11 unused).  Packed
# input-major: word [i, j // 16] holds weight W[j, i] at bits 2*(j % 16).
def ternary_pack(t) -> np.ndarray:
    """t [d_out, d_in] in {-1, 0, 1}  ->  packed W^T [d_in, d_out / 16] uint32."""
    t = np.asarray(t)
    d_out, d_in = t.shape
    if d_out % 16:
        raise ValueError("d_out must be a multiple of 16")
    code = np.zeros(t.shape, dtype=np.uint32)
    code[t == 1] = 1
    code[t == -1] = 2
    ct = code.T.reshape(d_in, d_out // 16, 16)
    shifts = (2 * np.arange(16)).astype(np.uint32)
    return np.ascontiguousarray(np.bitwise_or.reduce(ct << shifts, axis=2), dtype=np.uint32)


def ternary_unpack(packed, d_out: int) -> np.ndarray:
    """Inverse of :func:`ternary_pack`: packed [d_in, d_out/16] -> t [d_out, d_in] int8."""
    p = np.asarray(packed, dtype=np.uint32)
    d_in = p.shape[0]
    shifts = (2 * np.arange(16)).astype(np.uint32)
    code = (p[:, :, None] >> shifts) & np.uint32(3)
    code = code.reshape(d_in, d_out)
    if np.any(code == 3):
        raise ValueError("code 11 is not a ternary value")
    t = np.zeros((d_in, d_out), dtype=np.int8)
    t[code == 1] = 1
    t[code == 2] = -1
    return t.T.copy()


def quant_sparse_linear(x, t, alpha, k: int, eps: float = 1e-5,
                        keep: np.ndarray | None = None) -> dict:
    """int8 x ternary sparse projection.

    q, gamma = absmax_quantize(x);  keep = topK(|q|, k);  q_s = q (.) M;
    acc_tj = sum_i q_s[t, i] * t[j, i]  (exact integer);
    r_t = (alpha * gamma_t) / 127  (float32);  y_tj = float32(acc_tj) * r_t.
    """
    q, gamma = absmax_quantize(x, eps)
    T, d_in = q.shape
    t = np.asarray(t, dtype=np.int64)
    if t.shape[1] != d_in:
        raise ValueError("t must be [d_out, d_in]")
    if keep is None:
        keep = topk_keep(q, k)
    qs = q * mask_from_keep(keep, T, d_in)
    acc = qs @ t.T
    r = (np.float32(alpha) * gamma).astype(np.float32) / np.float32(127.0)
    r = r.astype(np.float32)
    y = acc.astype(np.float32) * r[:, None]
    return {"q": q, "gamma": gamma, "keep": keep, "acc": acc, "r": r,
            "y": y.astype(np.float32)}


def ffn_hidden_f32(u, g, act: str, b_up=None, b_gate=None) -> np.ndarray:
    """The gating epilogue in float32 steps (each operation rounded to float32,
    nearest-even, in this order), for the quantized FFN whose projections
    produce float32:  relu2_glu: r = max(u, 0); h = (r * r) * g.
    drelu: h = max(g + b_gate, 0) * max(u + b_up, 0)."""
    u = np.asarray(u, dtype=np.float32)
    g = np.asarray(g, dtype=np.float32)
    if act == "relu2_glu":
        r = np.maximum(u, np.float32(0.0))
        return ((r * r).astype(np.float32) * g).astype(np.float32)
    if act == "drelu":
        bu = np.float32(0.0) if b_up is None else np.asarray(b_up, dtype=np.float32)
        bg = np.float32(0.0) if b_gate is None else np.asarray(b_gate, dtype=np.float32)
        a = np.maximum((g + bg).astype(np.float32), np.float32(0.0))
        b = np.maximum((u + bu).astype(np.float32), np.float32(0.0))
        return (a * b).astype(np.float32)
    raise ValueError(f"unknown activation {act!r}")


def quant_sparse_ffn(x, t_up, alpha_up, t_gate, alpha_gate, t_down, alpha_down, act: str,
                     k_in: int, k_h: int, eps: float = 1e-5, b_up=None, b_gate=None,
                     block: int = 1) -> dict:
    """BitNet b1.58 + Q-Sparse FFN layer: every projection input is quantized
    (per-token absmax int8) and sparsified (top-K on |q|) before an int8 x
    ternary projection (Q-Sparse news article, Top-K section, quantized-model
    paragraphs, applied to each linear projection as the aibase.com summary
    says top-K is):
      u = quant_sparse_linear(x, t_up), g = quant_sparse_linear(x, t_gate)
          (one quantization and one selection of x shared by both)
      h = ffn_hidden_f32(u, g)                    float32 steps
      y = quant_sparse_linear(h, t_down, k_h)     (h quantized per token)
    block > 1 selects with Block Q-Sparse on |q| (:func:`block_topk_keep`).
    Every step is exact integer arithmetic or a fixed float32 step, so y is
    defined bit for bit."""
    q, _ = absmax_quantize(x, eps)
    keep_x = block_topk_keep(q, k_in, block)
    ru = quant_sparse_linear(x, t_up, alpha_up, k_in, eps, keep=keep_x)
    rg = quant_sparse_linear(x, t_gate, alpha_gate, k_in, eps, keep=keep_x)
    h = ffn_hidden_f32(ru["y"], rg["y"], act, b_up, b_gate)
    qh, _ = absmax_quantize(h, eps)
    keep_h = block_topk_keep(qh, k_h, block)
    rd = quant_sparse_linear(h, t_down, alpha_down, k_h, eps, keep=keep_h)
    return {"u": ru["y"], "g": rg["y"], "h": h, "keep_x": keep_x, "keep_h": keep_h,
            "acc_u": ru["acc"], "acc_g": rg["acc"], "acc_down": rd["acc"], "q_h": rd["q"],
            "y": rd["y"]}


# --------------------------------------------------------------------------
# error measure used by the parity tests
# --------------------------------------------------------------------------


def max_rel_err(y, ref) -> float:
    """max over rows of max_j |y - ref| / max_j |ref| (row infinity norm).

    Rows whose reference is all zero are measured against 1.0 instead.
    """
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if y.shape != ref.shape:
        raise ValueError(f"shape mismatch {y.shape} vs {ref.shape}")
    if y.size == 0:
        return 0.0
    y2 = y.reshape(-1, y.shape[-1])
    r2 = ref.reshape(-1, ref.shape[-1])
    den = np.max(np.abs(r2), axis=1)
    den[den == 0.0] = 1.0
    return float(np.max(np.max(np.abs(y2 - r2), axis=1) / den))
