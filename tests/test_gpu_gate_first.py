"""qs_sparse_ffn_gate_first on the GPU against the fp64 oracle.

The gate-first layer computes the dReLU FFN of the Turbo Sparse summary
(Eq. 2, then the top k% of |h| of Eq. 3-4) with dense x: the oracle is
oracle.sparse_ffn with act "drelu" and k_in = d_model.  Skipping W_up rows of
closed gates leaves only products that are exactly 0, so the checks are those
of qs_sparse_ffn: h within the f32 tolerance, the kept set a valid top-K of
the oracle's h, y against the oracle re-run on the GPU's own selection.  The
W_up rows read must be the open gates: every column where some token's h is
nonzero, and the oracle's count of g + b_gate > 0 except for columns whose gate
sum lies within float32 rounding of 0 (there either decision is right)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, check_status, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu

_weights = {}


def _mistral():
    w = workloads.WORKLOADS["ffn_drelu_mistral7b"]
    if w.name not in _weights:
        _weights[w.name] = workloads.ffn_weights(w)
    return w, _weights[w.name]


def _check_gate_first(x, up, gate, down, k_h, dtype, bias=None, idx=True, ws=None):
    T, d_model = x.shape
    d_ff = up.shape[1]
    xt = to_dev(x, dtype)
    gatet, downt = to_dev(gate, dtype), to_dev(down, dtype)
    w_up = to_dev(np.ascontiguousarray(up.T), dtype)            # [d_ff, d_model]
    b = None if bias is None else torch.full((d_ff,), bias, dtype=torch.float32, device="cuda")
    if ws is None:
        ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN_GATE_FIRST, T, d_model, d_ff, k_h, xt.device)
    r = qs.qs_sparse_ffn_gate_first(xt, gatet, w_up, downt, k_h, b_up=b, b_gate=b, h_out=True,
                                    idx_h_out=True if idx else None, ws=ws)
    check_status(ws)
    bnp = None if bias is None else np.full(d_ff, bias)
    ref = oracle.sparse_ffn(x, up, gate, down, "drelu", d_model, k_h, b_up=bnp, b_gate=bnp)
    h_gpu = r.h.cpu().numpy()
    assert oracle.max_rel_err(h_gpu, ref["h"]) <= TOL_F32
    if idx:
        keep_h = r.idx_h.cpu().numpy().astype(np.int64)
        for t in range(T):
            assert np.all(np.diff(keep_h[t]) > 0)
            kept = np.zeros(d_ff, bool)
            kept[keep_h[t]] = True
            mag = np.abs(ref["h"][t])
            if 0 < k_h < d_ff:
                assert mag[kept].min() >= mag[~kept].max() - 4 * TOL_F32 * mag.max()
    else:
        keep_h = oracle.topk_keep(h_gpu.astype(np.float64), k_h)
    ref_sel = oracle.sparse_ffn(x, up, gate, down, "drelu", d_model, k_h, b_up=bnp, b_gate=bnp,
                                keep_h=keep_h)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    err = oracle.max_rel_err(to_np(r.y), ref_sel["y"])
    assert err <= tol, err

    # the row counts describe the last chunk of (at most 64) tokens
    rows_x, rows_h, rows_up = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_FFN_GATE_FIRST, T,
                                                    d_model, d_ff, k_h)
    t0 = ((T - 1) // qs.QS_PREFILL_MIN_T) * qs.QS_PREFILL_MIN_T
    assert rows_x == int(np.count_nonzero(np.any(x[t0:] != 0, axis=0)))
    assert rows_h == np.unique(np.concatenate(
        [keep_h[t][h_gpu[t, keep_h[t]] != 0] for t in range(t0, T)] + [np.zeros(0, np.int64)])).size
    gb = ref["g"][t0:] + (0.0 if bias is None else bias)
    scale = np.abs(x[t0:]).astype(np.float64) @ np.abs(gate.astype(np.float64))
    tol_g = 1e-5 * (1.0 + scale)          # float32 rounding bound of a gate sum, generous
    lower = np.count_nonzero(np.any(gb > tol_g, axis=0))
    upper = np.count_nonzero(np.any(gb > -tol_g, axis=0))
    assert lower <= rows_up <= upper
    assert rows_up >= np.count_nonzero(np.any(h_gpu[t0:] != 0, axis=0))
    return r, ref, rows_up


@pytest.mark.parametrize("T", [1, 4])
def test_gate_first_mistral7b(T):
    """Mistral-7B dReLU shape, bf16, biases -0.8, K_h = 10% of 14336: the same
    layer as qs_sparse_ffn's dReLU, with about a fifth of W_up read per token."""
    need_gpu()
    w, (up, gate, down) = _mistral()
    x = workloads.activations(w, T)
    r, ref, rows_up = _check_gate_first(x, up, gate, down, w.k_h, "bf16", bias=w.bias)
    assert np.all(ref["h"] >= 0)
    assert rows_up < w.d_out                   # rows of closed gates were skipped
    # and the GPU's own dReLU layer agrees on h
    xt = to_dev(x, "bf16")
    b = torch.full((w.d_out,), w.bias, dtype=torch.float32, device="cuda")
    r2 = qs.qs_sparse_ffn(xt, to_dev(up, "bf16"), to_dev(gate, "bf16"), to_dev(down, "bf16"),
                          "drelu", w.d_in, w.k_h, b_up=b, b_gate=b, h_out=True)
    assert oracle.max_rel_err(r.h.cpu().numpy(), r2.h.cpu().numpy()) <= TOL_F32


def test_gate_first_one_token_list_path_twice():
    """One token without idx_h_out: the up kernel marks the nonzero h and the
    top-K on h starts from that bitmask.  Two tokens in a row on one workspace:
    the open-gate and nonzero-h bitmasks must be cleared between calls."""
    need_gpu()
    w, (up, gate, down) = _mistral()
    x2 = workloads.activations(w, 2)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN_GATE_FIRST, 1, w.d_in, w.d_out, w.k_h,
                          torch.device("cuda"))
    for t in range(2):
        _check_gate_first(x2[t:t + 1], up, gate, down, w.k_h, "bf16", bias=w.bias, idx=False, ws=ws)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,dm,dff", [(1, 64, 96), (3, 200, 328), (9, 128, 256), (66, 64, 64)])
def test_gate_first_small_and_ragged(dtype, T, dm, dff):
    """Row lengths that are not multiples of the 256- and 512-element sweeps,
    1-9 tokens and a second chunk (66 tokens), each K_h case, with and without
    idx_h_out."""
    need_gpu()
    g = workloads.rng(7 * T + 3 * dm + dff)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, dm)), dtype)
    up = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), dtype)
    down = workloads.round_to_dtype(workloads.normal_f32(g, (dff, dm), dff ** -0.5), dtype)
    for k_h in (dff, (7 * dff) // 10, 1, 0):
        _check_gate_first(x, up, gate, down, k_h, dtype, bias=-0.3)
    if T == 1:
        _check_gate_first(x, up, gate, down, dff // 3, dtype, bias=-0.3, idx=False)


def test_gate_first_no_bias_and_zero_inputs():
    """No biases (plain dReLU), and a token of zeros (every gate closed for
    it, while the other token opens gates)."""
    need_gpu()
    g = workloads.rng(31)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (2, 256)), "bf16")
    x[1] = 0.0
    up = workloads.round_to_dtype(workloads.normal_f32(g, (256, 512), 256 ** -0.5), "bf16")
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (256, 512), 256 ** -0.5), "bf16")
    down = workloads.round_to_dtype(workloads.normal_f32(g, (512, 256), 512 ** -0.5), "bf16")
    r, ref, _ = _check_gate_first(x, up, gate, down, 100, "bf16")
    assert not np.any(r.h.cpu().numpy()[1])


def test_gate_first_all_gates_closed():
    """A bias far below every gate sum closes all gates: no W_up row is read,
    h = 0 and y = 0."""
    need_gpu()
    g = workloads.rng(32)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (3, 128)), "bf16")
    up = workloads.round_to_dtype(workloads.normal_f32(g, (128, 192), 128 ** -0.5), "bf16")
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (128, 192), 128 ** -0.5), "bf16")
    down = workloads.round_to_dtype(workloads.normal_f32(g, (192, 128), 192 ** -0.5), "bf16")
    r, _, rows_up = _check_gate_first(x, up, gate, down, 50, "bf16", bias=-100.0)
    assert rows_up == 0
    assert not np.any(r.h.cpu().numpy())
    assert not np.any(to_np(r.y))
