"""qs_sparse_linear on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, bits, check_status, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu


def _run(x, wt, k, dtype):
    xt, wtt = to_dev(x, dtype), to_dev(wt, dtype)
    T, d_in = x.shape
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, d_in, wt.shape[1], k, xt.device)
    y = qs.qs_sparse_linear(xt, wtt, k, ws=ws)
    check_status(ws)
    return y, ws


def test_linear_f32_512_workload():
    """4 tokens, 512 -> 512 f32, K = 256 (50% kept)."""
    need_gpu()
    w = workloads.WORKLOADS["linear_f32_512"]
    x = workloads.activations(w, 4)
    wt = workloads.weight_t(w.d_in, w.d_out, w.seed(0, 1), "f32")
    y, ws = _run(x, wt, w.k, "f32")
    ref = oracle.sparse_linear(x, wt, w.k)
    assert oracle.max_rel_err(to_np(y), ref) <= TOL_F32
    rows, _ = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_LINEAR, 4, w.d_in, w.d_out, w.k)
    union = np.unique(oracle.topk_keep(x, w.k)).size
    assert rows == union


@pytest.mark.parametrize("T", [1, 2, 3, 8, 13])
def test_linear_bf16_llama_up_shape(T):
    """4096 -> 11008 bf16, K = floor(0.7 * 4096)."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.activations(w, T)
    wt = workloads.weight_t(4096, 11008, 77, "bf16")
    y, ws = _run(x, wt, w.k, "bf16")
    ref = oracle.sparse_linear(x, wt, w.k)
    assert oracle.max_rel_err(to_np(y), ref) <= TOL_BF16
    rows, _ = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_LINEAR, T, 4096, 11008, w.k)
    assert rows == np.unique(oracle.topk_keep(x, w.k)).size


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d_in,d_out", [(1, 1, 8), (5, 1000, 264), (2, 77, 136), (70, 300, 96),
                                           (6, 333, 1552), (4, 20, 160)])
def test_linear_ragged_sizes(dtype, T, d_in, d_out):
    """Ragged sizes; bf16 with 3-64 tokens and d_out % 16 == 0 takes the
    tensor-core path: (6, 333, 1552) has a short last column tile (97 blocks
    of 16 in 2 tiles), (4, 20, 160) fewer kept rows than one 16-row stage."""
    need_gpu()
    g = workloads.rng(T + d_in + d_out)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), dtype)
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), 0.05), dtype)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    for k in sorted({0, 1, d_in // 2, d_in}):
        y, _ = _run(x, wt, k, dtype)
        ref = oracle.sparse_linear(x, wt, k)
        if k == 0:
            assert torch.count_nonzero(y).item() == 0
        else:
            assert oracle.max_rel_err(to_np(y), ref) <= tol, k


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_linear_dense_k_equals_d(dtype):
    need_gpu()
    g = workloads.rng(31)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (3, 2048)), dtype)
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (2048, 1024), 2048 ** -0.5), dtype)
    y, _ = _run(x, wt, 2048, dtype)
    dense = x.astype(np.float64) @ wt.astype(np.float64)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert oracle.max_rel_err(to_np(y), dense) <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_linear_never_reads_unselected_rows(dtype):
    """NaN in every weight row no token keeps must not reach y: the gather
    reads kept rows only (masked columns contribute nothing)."""
    need_gpu()
    g = workloads.rng(41)
    T, d_in, d_out, k = 2, 4096, 2048, 600
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), dtype)
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), 0.02), dtype)
    y_clean, _ = _run(x, wt, k, dtype)
    union = np.unique(oracle.topk_keep(x, k))
    dropped = np.setdiff1d(np.arange(d_in), union)
    wt_nan = wt.copy()
    wt_nan[dropped] = np.nan
    y_poison, _ = _run(x, wt_nan, k, dtype)
    assert torch.isfinite(y_poison.float()).all()       # a single NaN read would spread
    # split sums are added in no fixed order, so compare to rounding only
    tol = 1e-5 if dtype == "f32" else 2 ** -7
    assert oracle.max_rel_err(to_np(y_poison), to_np(y_clean)) <= tol


# ---- prefill: bf16 with >= 64 tokens runs the tcgen05 masked-dense GEMM ----

def test_prefill_2048_tokens_outliers():
    """2048 tokens x 4096 -> 11008, 1% outlier channels x20, K = 2048: rows
    sampled across all 16 M-blocks checked against the fp64 oracle."""
    need_gpu()
    w = workloads.WORKLOADS["prefill_bf16_2048"]
    x = workloads.activations(w, 2048)
    wt = workloads.weight_t(w.d_in, w.d_out, w.seed(0, 1), "bf16")
    y, _ = _run(x, wt, w.k, "bf16")
    rows = np.arange(0, 2048, 16)
    ref = oracle.sparse_linear(x[rows], wt, w.k)
    assert oracle.max_rel_err(to_np(y)[rows], ref) <= TOL_BF16


@pytest.mark.parametrize("T,d_in,d_out,k", [
    (64, 64, 256, 32),        # one k-block, one N tile, M tail (64 < 128)
    (200, 136, 264, 70),      # K tail (136 = 2 x 64 + 8), N tail (264 = 256 + 8), M tail
    (130, 4096, 512, 4096),   # dense (K = d_in), M tail of 2 rows
    (256, 1000, 1024, 1),     # one kept input per token
    (128, 512, 520, 0),       # K = 0: all zero
    (1024, 256, 8200, 100),   # 264 tiles: CTAs take a second tile (the other accumulator), N tail
    (2048, 128, 8192, 64),    # 512 tiles: 3-4 tiles per CTA, each accumulator reused
])
def test_prefill_ragged_tiles(T, d_in, d_out, k):
    need_gpu()
    g = workloads.rng(T + d_in + d_out + k)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), "bf16")
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), d_in ** -0.5), "bf16")
    y, _ = _run(x, wt, k, "bf16")
    if k == 0:
        assert torch.count_nonzero(y).item() == 0
        return
    assert oracle.max_rel_err(to_np(y), oracle.sparse_linear(x, wt, k)) <= TOL_BF16
