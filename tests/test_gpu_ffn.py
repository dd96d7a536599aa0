"""qs_sparse_ffn on the GPU against the fp64 oracle.

h is computed on the GPU in f32 and on the oracle in fp64, so the top-K on
|h| may pick a different element where two magnitudes sit within rounding of
the threshold.  The checks therefore are: (1) h within the f32 tolerance;
(2) the GPU's kept set is a valid top-K of the oracle's h up to
eps_sel = 4 * TOL_F32 * max|h_t|; (3) y against the oracle re-run on the
GPU's own selection of h (the input top-K, of given data, is bit-exact and
checked through the row count)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, check_status, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu

_weights = {}


def _ffn_weights(name):
    if name not in _weights:
        w = workloads.WORKLOADS[name]
        _weights[name] = workloads.ffn_weights(w)
    return _weights[name]


def _check_ffn(x, up, gate, down, act, k_in, k_h, dtype, bias=None):
    T, d_model = x.shape
    d_ff = up.shape[1]
    xt = to_dev(x, dtype)
    upt, gatet, downt = to_dev(up, dtype), to_dev(gate, dtype), to_dev(down, dtype)
    b = None if bias is None else torch.full((d_ff,), bias, dtype=torch.float32, device="cuda")
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h, xt.device)
    r = qs.qs_sparse_ffn(xt, upt, gatet, downt, act, k_in, k_h, b_up=b, b_gate=b,
                         h_out=True, idx_h_out=True, ws=ws)
    check_status(ws)
    bnp = None if bias is None else np.full(d_ff, bias)
    ref = oracle.sparse_ffn(x, up, gate, down, act, k_in, k_h, b_up=bnp, b_gate=bnp)
    h_gpu = r.h.cpu().numpy()
    assert oracle.max_rel_err(h_gpu, ref["h"]) <= TOL_F32
    idx_h = r.idx_h.cpu().numpy().astype(np.int64)
    swaps = 0
    for t in range(T):
        assert np.all(np.diff(idx_h[t]) > 0)
        kept = np.zeros(d_ff, bool)
        kept[idx_h[t]] = True
        mag = np.abs(ref["h"][t])
        eps_sel = 4 * TOL_F32 * mag.max()
        if 0 < k_h < d_ff:
            assert mag[kept].min() >= mag[~kept].max() - eps_sel
        swaps += k_h - np.intersect1d(idx_h[t], ref["keep_h"][t]).size
    ref_sel = oracle.sparse_ffn(x, up, gate, down, act, k_in, k_h, b_up=bnp, b_gate=bnp,
                                keep_h=idx_h)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    err = oracle.max_rel_err(to_np(r.y), ref_sel["y"])
    assert err <= tol, err
    # the row counts describe the last chunk of (at most 64) tokens
    rows_x, rows_h = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h)
    t0 = ((T - 1) // qs.QS_PREFILL_MIN_T) * qs.QS_PREFILL_MIN_T
    kx = ref["keep_x"][t0:]
    assert rows_x == np.unique(kx[np.take_along_axis(x[t0:], kx, 1) != 0]).size
    assert rows_h == np.unique(np.concatenate(
        [idx_h[t][h_gpu[t, idx_h[t]] != 0] for t in range(t0, T)] + [np.zeros(0, np.int64)])).size
    return swaps, ref


@pytest.mark.parametrize("T", [1, 8])
def test_ffn_relu2_llama7b(T):
    """Llama-7B FFN decode, bf16: K = 0.7 d on x and on |h|, squared-ReLU gating."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    up, gate, down = _ffn_weights(w.name)
    x = workloads.activations(w, T)
    swaps, ref = _check_ffn(x, up, gate, down, "relu2_glu", w.k, w.k_h, "bf16")
    assert swaps <= 2 * T


@pytest.mark.parametrize("T", [1, 4])
def test_ffn_drelu_mistral7b(T):
    """Mistral-7B dReLU FFN decode, bf16: dense x, biases -0.8, keep top 10% of |h|."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_drelu_mistral7b"]
    up, gate, down = _ffn_weights(w.name)
    x = workloads.activations(w, T)
    swaps, ref = _check_ffn(x, up, gate, down, "drelu", w.k, w.k_h, "bf16", bias=w.bias)
    assert swaps <= 2 * T
    assert np.all(ref["h"] >= 0)


@pytest.mark.parametrize("act", ["relu2_glu", "drelu"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,dm,dff", [(1, 64, 96), (3, 200, 328), (9, 128, 256), (66, 64, 64)])
def test_ffn_small_and_ragged(act, dtype, T, dm, dff):
    need_gpu()
    g = workloads.rng(T * 1000 + dm + dff)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, dm)), dtype)
    up = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    down = workloads.round_to_dtype(workloads.normal_f32(g, (dff, dm), dff ** -0.5), dtype)
    bias = -0.3 if act == "drelu" else None
    for k_in, k_h in ((dm, dff), ((7 * dm) // 10, (7 * dff) // 10), (1, 1), (dm, 0)):
        _check_ffn(x, up, gate, down, act, k_in, k_h, dtype, bias=bias)


def _check_ffn_list_path(x, up, gate, down, act, k_in, k_h, dtype, bias=None, ws=None):
    """One token, no idx_h_out: the up/gate epilogue marks the nonzero h in a
    bitmask and the top-K on h starts from it (all nonzeros when there are at
    most K of them, else a full selection).  The kept set is checked through
    the row count and y against the oracle re-run on the top-K of the GPU's
    own h (ranking given f32 values is exact)."""
    T, d_model = x.shape
    d_ff = up.shape[1]
    xt = to_dev(x, dtype)
    upt, gatet, downt = to_dev(up, dtype), to_dev(gate, dtype), to_dev(down, dtype)
    b = None if bias is None else torch.full((d_ff,), bias, dtype=torch.float32, device="cuda")
    if ws is None:
        ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h, xt.device)
    r = qs.qs_sparse_ffn(xt, upt, gatet, downt, act, k_in, k_h, b_up=b, b_gate=b, h_out=True, ws=ws)
    check_status(ws)
    bnp = None if bias is None else np.full(d_ff, bias)
    ref = oracle.sparse_ffn(x, up, gate, down, act, k_in, k_h, b_up=bnp, b_gate=bnp)
    h_gpu = r.h.cpu().numpy()
    assert oracle.max_rel_err(h_gpu, ref["h"]) <= TOL_F32
    keep_h = oracle.topk_keep(h_gpu.astype(np.float64), k_h)
    ref_sel = oracle.sparse_ffn(x, up, gate, down, act, k_in, k_h, b_up=bnp, b_gate=bnp,
                                keep_h=keep_h)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert oracle.max_rel_err(to_np(r.y), ref_sel["y"]) <= tol
    _, rows_h = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h)
    assert rows_h == int(np.count_nonzero(h_gpu[0, keep_h[0]]))
    return r, ws


def test_ffn_one_token_list_path_llama7b():
    """Llama-7B shape: about half of h is zero, fewer than K_h nonzeros, so the
    kept rows are exactly the nonzero h.  Two tokens in a row on one workspace
    (the bitmask must be left clear), then a several-token call."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    up, gate, down = _ffn_weights(w.name)
    x2 = workloads.activations(w, 2)
    # two different tokens in a row: a bitmask left over from the first call
    # would add the first token's nonzero h to the second token's row count
    _, ws = _check_ffn_list_path(x2[:1], up, gate, down, "relu2_glu", w.k, w.k_h, "bf16")
    _check_ffn_list_path(x2[1:], up, gate, down, "relu2_glu", w.k, w.k_h, "bf16", ws=ws)
    x8 = workloads.activations(w, 8)
    _check_ffn(x8, up, gate, down, "relu2_glu", w.k, w.k_h, "bf16")


@pytest.mark.parametrize("fused", [1, 2, 0])       # ordinary launch, cooperative launch, off
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dm,dff", [(64, 96), (200, 328), (128, 1000), (96, 16384)])
def test_ffn_one_token_list_path_small(dtype, dm, dff, fused):
    """Both branches of the bitmask start (or, one-kernel path, of the kept-h
    choice): K_h above and below the nonzero count of h (and K_h = 0,
    K_h = d_ff), ragged d_ff, the largest d_ff it takes."""
    need_gpu()
    if fused and dtype == "f32":
        pytest.skip("the one-kernel path serves bf16 only")
    qs.qs_set_ffn_fused(fused)
    try:
        _list_path_small(dtype, dm, dff)
    finally:
        qs.qs_set_ffn_fused(True)


def _list_path_small(dtype, dm, dff):
    g = workloads.rng(dm * 7 + dff)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (1, dm)), dtype)
    up = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    down = workloads.round_to_dtype(workloads.normal_f32(g, (dff, dm), dff ** -0.5), dtype)
    k_hs = (dff, (7 * dff) // 10, dff // 5, 1, 0)
    need = max(qs.qs_workspace_size(qs.QS_OP_SPARSE_FFN, 1, dm, dff, k) for k in k_hs)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")      # one workspace for every call
    for act, bias in (("relu2_glu", None), ("drelu", -0.3)):
        for k_h in k_hs:
            _check_ffn_list_path(x, up, gate, down, act, (7 * dm) // 10, k_h, dtype, bias=bias, ws=ws)


def test_ffn_one_token_fused_llama7b():
    """The one-kernel path of a one-token bf16 layer (every CTA resident, grid
    barriers) against the oracle and against the separate kernels: the input
    list is the same bit for bit, y matches the oracle re-run on the GPU's own
    kept h; then K_h below the nonzero count (every CTA selects the K_h-th
    largest |h| itself); then tokens back to back on one workspace (the
    barrier counters must be reset by each call), launched both ways (an
    ordinary and a cooperative launch; the down projection's partial sums are
    float atomic additions, so y is checked against the oracle each time)."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    assert qs.qs_sparse_ffn_fused(qs.QS_BF16, 1, w.d_in, w.d_out, False)
    assert not qs.qs_sparse_ffn_fused(qs.QS_BF16, 1, w.d_in, w.d_out, True)
    assert not qs.qs_sparse_ffn_fused(qs.QS_BF16, 2, w.d_in, w.d_out, False)
    assert not qs.qs_sparse_ffn_fused(qs.QS_F32, 1, w.d_in, w.d_out, False)
    up, gate, down = _ffn_weights(w.name)
    x4 = workloads.activations(w, 4)
    lists = {}
    for fused in (True, False):
        qs.qs_set_ffn_fused(fused)
        try:
            _, ws = _check_ffn_list_path(x4[:1], up, gate, down, "relu2_glu", w.k, w.k_h, "bf16")
        finally:
            qs.qs_set_ffn_fused(True)
        lists[fused] = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_FFN, 1, w.d_in, w.d_out, w.k_h, 0,
                                            values=True)
    rows_f, vals_f = lists[True]
    rows_g, vals_g = lists[False]
    assert np.array_equal(rows_f, rows_g) and np.array_equal(vals_f, vals_g)
    keep = oracle.topk_keep(x4[:1], w.k)[0]
    xb = x4[0, keep]
    assert np.array_equal(rows_f, keep[xb != 0])
    assert np.array_equal(vals_f, xb[xb != 0].astype(np.float32))
    # fewer kept h than nonzero h: the radix select over |h| in every CTA
    _check_ffn_list_path(x4[1:2], up, gate, down, "relu2_glu", w.k, w.d_out // 10, "bf16")
    # back to back on one workspace, without a host synchronisation in between
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, 1, w.d_in, w.d_out, w.k_h, torch.device("cuda"))
    upt, gatet, downt = to_dev(up, "bf16"), to_dev(gate, "bf16"), to_dev(down, "bf16")
    xs = [to_dev(x4[t:t + 1], "bf16") for t in range(4)]
    ys = [qs.qs_sparse_ffn(xs[t], upt, gatet, downt, "relu2_glu", w.k, w.k_h, ws=ws).y
          for t in range(4)]
    check_status(ws)
    qs.qs_set_ffn_fused(2)
    try:
        ys_coop = [qs.qs_sparse_ffn(xs[t], upt, gatet, downt, "relu2_glu", w.k, w.k_h, ws=ws).y
                   for t in range(4)]
        check_status(ws)
    finally:
        qs.qs_set_ffn_fused(True)
    for t in range(4):
        ref = oracle.sparse_ffn(x4[t:t + 1], up, gate, down, "relu2_glu", w.k, w.k_h)
        assert oracle.max_rel_err(to_np(ys[t]), ref["y"]) <= 2 * TOL_BF16
        assert oracle.max_rel_err(to_np(ys_coop[t]), ref["y"]) <= 2 * TOL_BF16
