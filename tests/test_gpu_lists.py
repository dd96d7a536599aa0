"""The one-token decode path's row lists, bit for bit against the oracle.

With one token and no optional outputs (the call a decoder makes), the top-K
runs the list kernel, which writes only the kept nonzero inputs' indices and
values into the workspace.  qs_workspace_list copies them out, and they must
equal, bit for bit, the oracle's kept indices whose value is nonzero
(ascending) and the values at those indices (Q-Sparse news article, section
"Top-K sparsification": the K largest |x| are kept; zero values contribute
nothing, so they are not streamed)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import check_status, need_gpu, to_dev

pytestmark = pytest.mark.gpu


def _expect(x_row, k):
    """(kept nonzero indices ascending, their values as float32) from the oracle."""
    keep = oracle.topk_keep(x_row[None, :], k)[0]
    vals = oracle.kept_values(x_row[None, :], keep[None, :])[0]
    nz = vals != 0
    return keep[nz].astype(np.int32), vals[nz].astype(np.float32)


def _linear_list(x_row, dtype, k, d_out=64):
    d_in = x_row.size
    xt = to_dev(x_row[None, :], dtype)
    wt = torch.zeros(d_in, d_out, dtype=xt.dtype, device="cuda")
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, 1, d_in, d_out, k, xt.device)
    qs.qs_sparse_linear(xt, wt, k, ws=ws)
    check_status(ws)
    return qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_LINEAR, 1, d_in, d_out, k, 0, values=True)


def _check_linear(x_row, dtype, k):
    rows, vals = _linear_list(x_row, dtype, k)
    want_rows, want_vals = _expect(x_row, k)
    assert np.array_equal(rows, want_rows), (dtype, k)
    assert np.array_equal(vals.view(np.int32), want_vals.view(np.int32)), (dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_list_kernel_llama_input_row(dtype):
    """The x row of the Llama-7B FFN decode step: d = 4096, K = floor(0.7 d)."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.round_to_dtype(workloads.activations(w, 1)[0], dtype)
    for k in (w.k, 1, 2048, 4095, 4096, 0):
        _check_linear(x, dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [1, 7, 1000, 1025, 11008, 14336, 16384, 20000])
def test_list_kernel_random_rows(dtype, d):
    """Every register-slot count of the list kernel (d up to 16 K) and the
    shared-memory kernel for longer rows (d = 20000)."""
    need_gpu()
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(d + 3), (d,)), dtype)
    for k in sorted({1, d // 3, (7 * d) // 10, d - 1, d}):
        _check_linear(x, dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [5, 64, 1000, 4096])
def test_list_kernel_ties_and_zeros(dtype, d):
    """Few distinct magnitudes, one magnitude everywhere, signed zeros."""
    need_gpu()
    x = workloads.adversarial_rows(d, 3, d)
    for r in range(3):
        for k in sorted({1, d // 3, d // 2, (7 * d) // 10, d - 1, d}):
            _check_linear(x[r], dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("zero_frac", [0.5, 0.95])
def test_list_kernel_rows_with_many_zeros(dtype, zero_frac):
    """K below, at and above the nonzero count (the nonzero-count shortcut)."""
    need_gpu()
    d = 11008
    g = workloads.rng(int(zero_frac * 1000))
    x = workloads.round_to_dtype(workloads.normal_f32(g, (d,)), dtype)
    x[g.random(d) < zero_frac] = 0.0
    x[::7] = np.where(x[::7] == 0, np.float32(-0.0), x[::7])
    nnz = int(np.count_nonzero(x))
    for k in sorted({1, nnz - 1, nnz, nnz + 1, (7 * d) // 10}):
        _check_linear(x, dtype, k)


def test_list_kernel_integer_magnitudes():
    """128 distinct magnitudes over 4096 entries: heavy ties at the threshold."""
    need_gpu()
    x = workloads.rng(5).integers(-127, 128, size=4096).astype(np.float32)
    for dtype in ("f32", "bf16"):
        for k in (1597, 1, 4095):
            _check_linear(x, dtype, k)


# ---- int8 x ternary, one token, no optional outputs -------------------------

@pytest.mark.parametrize("name", ["quant_up_4096x11008", "quant_down_11008x4096"])
def test_quant_one_token_product_path_bit_exact(name):
    """qs_quant_sparse_linear with acc = q = idx = NULL at T = 1 (the decode
    call): the quantized top-K runs the list kernel.  Its list (kept nonzero
    codes, ascending) and codes, and y, are bit-exact against the oracle."""
    need_gpu()
    w = workloads.WORKLOADS[name]
    W = workloads.weight_out_major(w.d_out, w.d_in, w.d_out + w.d_in)
    t, alpha = oracle.ternary_quantize(W)
    packed = torch.from_numpy(oracle.ternary_pack(t).view(np.int32)).cuda()
    for salt in range(3):
        x = workloads.activations(w, 1, salt=salt)
        xt = to_dev(x, "bf16")
        ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_LINEAR, 1, w.d_in, w.d_out, w.k, xt.device)
        r = qs.qs_quant_sparse_linear(xt, packed, float(alpha), w.k, 1e-5, ws=ws)
        check_status(ws)
        assert r.acc is None and r.q is None and r.idx is None
        ref = oracle.quant_sparse_linear(x, t, alpha, w.k)
        assert np.array_equal(r.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))
        rows, codes = qs.qs_workspace_list(ws, qs.QS_OP_QUANT_SPARSE_LINEAR, 1, w.d_in, w.d_out,
                                           w.k, 0, values=True)
        keep = ref["keep"][0]
        q_kept = ref["q"][0, keep]
        assert np.array_equal(rows, keep[q_kept != 0].astype(np.int32))
        assert np.array_equal(codes.astype(np.int64), q_kept[q_kept != 0])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quant_one_token_edge_rows(dtype):
    """Zero row, one nonzero, all ties, epsilon-sized magnitudes, through the
    one-token product path (no optional outputs): y bit-exact."""
    need_gpu()
    d_in, d_out = 300, 64
    W = workloads.weight_out_major(d_out, d_in, 9)
    t, alpha = oracle.ternary_quantize(W)
    packed = torch.from_numpy(oracle.ternary_pack(t).view(np.int32)).cuda()
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(10), (5, d_in)), dtype)
    x[1] = 0.0
    x[2] = 0.0
    x[2, 17] = -7.5
    x[3] = np.float32(0.5)
    x[4, :5] = workloads.round_to_dtype(np.array([3e-5, 1e-5, -2.2e-5, 0, 0], np.float32), dtype)
    x[4, 5:] = 0.0
    for r in range(5):
        for k in (0, 1, 117, d_in - 1, d_in):
            xt = to_dev(x[r:r + 1], dtype)
            ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_LINEAR, 1, d_in, d_out, k, xt.device)
            res = qs.qs_quant_sparse_linear(xt, packed, float(alpha), k, 1e-5, ws=ws)
            check_status(ws)
            ref = oracle.quant_sparse_linear(x[r:r + 1], t, alpha, k)
            assert np.array_equal(res.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32)), (r, k)


# ---- the FFN's two lists, one token -------------------------------------------

@pytest.mark.parametrize("name,act", [("ffn_relu2_llama7b", "relu2_glu"),
                                      ("ffn_drelu_mistral7b", "drelu")])
def test_ffn_one_token_lists_bit_exact(name, act):
    """One token, no idx_h_out (the decode call): the x list must be the
    oracle's top-K of the given x, bit for bit; the h list (started from the
    epilogue's bitmask of nonzero h, or a full selection) must be the oracle's
    top-K of the GPU's own h, bit for bit (ranking given f32 values is exact)."""
    need_gpu()
    w = workloads.WORKLOADS[name]
    up, gate, down = workloads.ffn_weights(w)
    dev = torch.device("cuda")
    upt, gatet, downt = to_dev(up, "bf16"), to_dev(gate, "bf16"), to_dev(down, "bf16")
    b = None if w.bias is None else torch.full((w.d_out,), w.bias, dtype=torch.float32, device=dev)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, 1, w.d_in, w.d_out, w.k_h, dev)
    for salt in range(2):
        x = workloads.activations(w, 1, salt=salt)
        for k_h in (w.k_h, w.d_out // 50):
            r = qs.qs_sparse_ffn(to_dev(x, "bf16"), upt, gatet, downt, act, w.k, k_h, b_up=b,
                                 b_gate=b, h_out=True, ws=ws)
            check_status(ws)
            rows_x, vals_x = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_FFN, 1, w.d_in, w.d_out, k_h,
                                                  0, values=True)
            want_rows, want_vals = _expect(x[0], w.k)
            assert np.array_equal(rows_x, want_rows)
            assert np.array_equal(vals_x.view(np.int32), want_vals.view(np.int32))
            h = r.h.cpu().numpy()[0]
            rows_h, vals_h = qs.qs_workspace_list(ws, qs.QS_OP_SPARSE_FFN, 1, w.d_in, w.d_out, k_h,
                                                  1, values=True)
            want_rows, want_vals = _expect(h, k_h)
            assert np.array_equal(rows_h, want_rows), k_h
            assert np.array_equal(vals_h.view(np.int32), want_vals.view(np.int32)), k_h
