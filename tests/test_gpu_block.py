"""Block Q-Sparse on the GPU against the oracle (oracle.block_topk_keep).

Blocks of consecutive tokens share one selection: the k features with the
largest block magnitude max_t |x_t,i| (Q-Sparse paper summary, shd-paper.top,
abstract and method section key design 3; the mechanism is this library's
reading).  The selection is of given data, so the listed weight rows are
compared bit for bit; projections are compared within the stated tolerances,
the int8 x ternary path bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, check_status, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu

_cache = {}


def _cached(key, make):
    if key not in _cache:
        _cache[key] = make()
    return _cache[key]


def _rows_of_last_chunk(x, keep, block):
    """Weight rows the last chunk streams: the kept features with a nonzero
    value in some token of that chunk (chunks hold whole blocks, <= 64 tokens)."""
    T = x.shape[0]
    chunk = (64 // block) * block
    t0 = ((T - 1) // chunk) * chunk
    vals = np.take_along_axis(x[t0:], keep[t0:], 1)
    return np.unique(keep[t0:][vals != 0]).astype(np.int32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,block", [(2, 2), (5, 2), (8, 8), (8, 4), (13, 8), (3, 8), (70, 16),
                                     (64, 64)])
def test_block_linear_llama_up_shape(dtype, T, block):
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.round_to_dtype(workloads.activations(w, T), dtype)
    wt = _cached(("wt", dtype), lambda: workloads.weight_t(4096, 11008 if dtype == "bf16" else 1024,
                                                           78, dtype))
    d_out = wt.shape[1]
    xt, wtt = to_dev(x, dtype), to_dev(wt, dtype)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, 4096, d_out, w.k, xt.device)
    y = qs.qs_sparse_linear(xt, wtt, w.k, ws=ws, block=block)
    check_status(ws)
    keep = oracle.block_topk_keep(x, w.k, block)
    ref = oracle.sparse_linear(x, wt, w.k, keep=keep)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    if T < 64 or dtype == "f32":
        rows, _ = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_LINEAR, T, 4096, d_out, w.k, 0)
        assert np.array_equal(rows, _rows_of_last_chunk(x, keep, block))
    assert oracle.max_rel_err(to_np(y), ref) <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_block_selection_ties_zeros_and_block_of_one(dtype):
    """Adversarial rows (few magnitudes, one magnitude everywhere, signed
    zeros); block = 1 must give the per-token entry point's result exactly."""
    need_gpu()
    d, d_out = 1000, 64
    x = workloads.adversarial_rows(11, 6, d)
    wt = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(12), (d, d_out), 0.05), dtype)
    xt, wtt = to_dev(x, dtype), to_dev(wt, dtype)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    for k in (1, 333, 500, 999, 1000):
        for block in (2, 3, 6):
            ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, 6, d, d_out, k, xt.device)
            y = qs.qs_sparse_linear(xt, wtt, k, ws=ws, block=block)
            check_status(ws)
            keep = oracle.block_topk_keep(x, k, block)
            rows, _ = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_LINEAR, 6, d, d_out, k, 0)
            assert np.array_equal(rows, _rows_of_last_chunk(x, keep, block)), (k, block)
            assert oracle.max_rel_err(to_np(y), oracle.sparse_linear(x, wt, k, keep=keep)) <= tol
        ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, 6, d, d_out, k, xt.device)
        y1 = qs.qs_sparse_linear(xt, wtt, k, ws=ws, block=1)
        y0 = qs.qs_sparse_linear(xt, wtt, k, ws=ws)
        assert oracle.max_rel_err(to_np(y1), to_np(y0)) <= 1e-6


def test_block_prefill_tensor_cores():
    """bf16 with >= 64 tokens: the block-masked X_sparse goes to the tcgen05
    GEMM (two blocks of 64 tokens, outlier channels as in the prefill workload)."""
    need_gpu()
    w = workloads.WORKLOADS["prefill_bf16_2048"]
    T, block = 128, 64
    x = workloads.activations(w, T)
    wt = workloads.weight_t(w.d_in, 1024, 5, "bf16")
    xt, wtt = to_dev(x, "bf16"), to_dev(wt, "bf16")
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, w.d_in, 1024, w.k, xt.device)
    y = qs.qs_sparse_linear(xt, wtt, w.k, ws=ws, block=block)
    check_status(ws)
    ref = oracle.sparse_linear(x, wt, w.k, keep=oracle.block_topk_keep(x, w.k, block))
    assert oracle.max_rel_err(to_np(y), ref) <= TOL_BF16


def test_block_rejects_long_rows_and_bad_block():
    need_gpu()
    x = torch.zeros(2, 20000, device="cuda")
    wt = torch.zeros(20000, 64, device="cuda")
    with pytest.raises(qs.QSError) as e:
        qs.qs_sparse_linear(x, wt, 10, block=2)
    assert e.value.status == qs.QS_ERR_UNSUPPORTED
    for bad in (0, qs.QS_MAX_BLOCK + 1):
        with pytest.raises(qs.QSError) as e:
            qs.qs_sparse_linear(x[:, :64].contiguous(), wt[:64].contiguous(), 10, block=bad)
        assert e.value.status == qs.QS_ERR_INVALID_ARG


@pytest.mark.parametrize("T,block", [(8, 8), (8, 4), (4, 4)])
@pytest.mark.parametrize("name,act", [("ffn_relu2_llama7b", "relu2_glu"),
                                      ("ffn_drelu_mistral7b", "drelu")])
def test_block_ffn_7b_shapes(name, act, T, block):
    """Block selections on x and on h.  x: the listed rows bit-exact; h within
    the f32 tolerance, the GPU's block selection of h valid against the
    oracle's h up to eps_sel, y against the oracle re-run on that selection."""
    need_gpu()
    w = workloads.WORKLOADS[name]
    up, gate, down = _cached(name, lambda: workloads.ffn_weights(w))
    x = workloads.activations(w, T)
    dev = torch.device("cuda")
    b = None if w.bias is None else torch.full((w.d_out,), w.bias, dtype=torch.float32, device=dev)
    bnp = None if w.bias is None else np.full(w.d_out, w.bias)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, T, w.d_in, w.d_out, w.k_h, dev)
    r = qs.qs_sparse_ffn(to_dev(x, "bf16"), to_dev(up, "bf16"), to_dev(gate, "bf16"),
                         to_dev(down, "bf16"), act, w.k, w.k_h, b_up=b, b_gate=b, h_out=True,
                         idx_h_out=True, ws=ws, block=block)
    check_status(ws)
    ref = oracle.sparse_ffn(x, up, gate, down, act, w.k, w.k_h, b_up=bnp, b_gate=bnp, block=block)
    rows_x, _ = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_FFN, T, w.d_in, w.d_out, w.k_h, 0)
    assert np.array_equal(rows_x, _rows_of_last_chunk(x, ref["keep_x"], block))
    h = r.h.cpu().numpy()
    assert oracle.max_rel_err(h, ref["h"]) <= TOL_F32
    idx_h = r.idx_h.cpu().numpy().astype(np.int64)
    for b0 in range(0, T, block):
        rows = list(range(b0, min(T, b0 + block)))
        assert all(np.array_equal(idx_h[t], idx_h[rows[0]]) for t in rows)
        s = np.max(np.abs(ref["h"][rows]), axis=0)
        kept = np.zeros(w.d_out, bool)
        kept[idx_h[rows[0]]] = True
        assert s[kept].min() >= s[~kept].max() - 4 * TOL_F32 * s.max()
    ref_sel = oracle.sparse_ffn(x, up, gate, down, act, w.k, w.k_h, b_up=bnp, b_gate=bnp,
                                keep_h=idx_h, block=block)
    assert oracle.max_rel_err(to_np(r.y), ref_sel["y"]) <= TOL_BF16
    # the block streams at most k_h rows of W_down, fewer than the per-token union
    _, rows_h = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_FFN, T, w.d_in, w.d_out, w.k_h)
    assert rows_h <= w.k_h * ((T + block - 1) // block)


@pytest.mark.parametrize("T,block", [(32, 32), (32, 8), (8, 8), (12, 5), (70, 32)])
@pytest.mark.parametrize("name", ["quant_up_4096x11008", "quant_down_11008x4096"])
def test_block_quant_bit_exact(name, T, block):
    """int8 x ternary with block selections on |q|: q, kept indices, acc and y
    bit-exact (each token quantized with its own gamma, the block ranks max |q|)."""
    need_gpu()
    w = workloads.WORKLOADS[name]
    def make():
        t_, a_ = oracle.ternary_quantize(workloads.weight_out_major(w.d_out, w.d_in, w.d_out + w.d_in))
        return t_, a_, oracle.ternary_pack(t_)
    t, alpha, packed_np = _cached(name, make)
    packed = torch.from_numpy(packed_np.view(np.int32)).cuda()
    x = workloads.activations(w, T)
    xt = to_dev(x, "bf16")
    ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k, xt.device)
    r = qs.qs_quant_sparse_linear(xt, packed, float(alpha), w.k, 1e-5, acc=True, q=True, idx=True,
                                  ws=ws, block=block)
    check_status(ws)
    q, _ = oracle.absmax_quantize(x)
    keep = oracle.block_topk_keep(q, w.k, block)
    ref = oracle.quant_sparse_linear(x, t, alpha, w.k, keep=keep)
    assert np.array_equal(r.q.cpu().numpy().astype(np.int64), ref["q"])
    assert np.array_equal(r.idx.cpu().numpy().astype(np.int64), keep)
    assert np.array_equal(r.acc.cpu().numpy().astype(np.int64), ref["acc"])
    assert np.array_equal(r.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))
    # product path without optional outputs: y bit-exact as well
    r2 = qs.qs_quant_sparse_linear(xt, packed, float(alpha), w.k, 1e-5, ws=ws, block=block)
    check_status(ws)
    assert np.array_equal(r2.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))
