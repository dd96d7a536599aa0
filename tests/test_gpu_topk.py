"""qs_topk_mask on the GPU against the oracle: indices, values, mask and
X_sparse must be bit-exact (integer / selection work)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import bits, check_status, need_gpu, np_bits, to_dev

pytestmark = pytest.mark.gpu


def _ks(d):
    return sorted({k for k in (0, 1, 2, d // 3, d // 2, (7 * d) // 10, d - 1, d) if 0 <= k <= d})


def _check_row_block(x, dtype, k):
    xt = to_dev(x, dtype)
    ws = qs.new_workspace(qs.QS_OP_TOPK_MASK, x.shape[0], x.shape[1], 0, k, xt.device)
    r = qs.qs_topk_mask(xt, k, val=True, mask=True, xs=True, ws=ws)
    check_status(ws)
    keep, m, xs = oracle.topk_mask(x, k)
    assert np.array_equal(r.idx.cpu().numpy(), keep), f"indices differ (k={k})"
    assert np.array_equal(bits(r.val), np_bits(oracle.kept_values(x, keep), dtype))
    assert np.array_equal(r.mask.cpu().numpy(), m)
    got_xs = r.xs.float().cpu().numpy()
    assert np.array_equal(got_xs, xs)                       # value equality (+0 == -0)
    kept_bits = np.where(m == 1, np_bits(x, dtype), 0)
    assert np.array_equal(np.where(m == 1, bits(r.xs), 0), kept_bits)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d", [(1, 1), (1, 7), (3, 33), (2, 1000), (1, 1024), (1, 1025),
                                 (5, 4096), (1, 11008), (2, 14336)])
def test_topk_random_rows(dtype, T, d):
    need_gpu()
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(T * 7919 + d), (T, d)), dtype)
    for k in _ks(d):
        _check_row_block(x, dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [5, 64, 1000, 4096])
def test_topk_ties_signed_zero_all_equal(dtype, d):
    need_gpu()
    x = workloads.adversarial_rows(d, 3, d)
    for k in _ks(d):
        _check_row_block(x, dtype, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_topk_max_row_length(dtype):
    need_gpu()
    d = qs.QS_MAX_ROW
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(d), (1, d)), dtype)
    for k in (1, d // 2, d - 1):
        _check_row_block(x, dtype, k)


def test_topk_prefill_rows_with_outliers():
    """2048 tokens x 4096 (the many-row launch shape), 1% outlier channels x20, K=2048."""
    need_gpu()
    w = workloads.WORKLOADS["prefill_bf16_2048"]
    x = workloads.activations(w, 2048)
    _check_row_block(x, "bf16", w.k)
    # outlier channels are kept for nearly every token (|20 z| beats the median
    # |x| unless |z| < ~0.034, about 3% of draws)
    keep = oracle.topk_keep(x, w.k)
    ch = workloads.outlier_channels(w, 2048)
    frac = np.mean([np.isin(ch, keep[t]).mean() for t in range(2048)])
    assert frac > 0.9


def test_topk_quantized_magnitudes_many_ties():
    """Keys with only 128 distinct magnitudes (int8-like) stress the tie order."""
    need_gpu()
    g = workloads.rng(5)
    x = (g.integers(-127, 128, size=(4, 4096))).astype(np.float32)
    for k in (1597, 1, 4095):
        _check_row_block(x, "f32", k)
        _check_row_block(x, "bf16", k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("zero_frac", [0.5, 0.9, 1.0])
def test_topk_rows_with_many_zeros(dtype, zero_frac):
    """Rows like ReLU outputs: K below, at and above the nonzero count (the
    nonzero-count shortcut must give exactly the sort's answer)."""
    need_gpu()
    d = 11008
    g = workloads.rng(int(zero_frac * 100) + len(dtype))
    x = workloads.round_to_dtype(workloads.normal_f32(g, (3, d)), dtype)
    x[g.random((3, d)) < zero_frac] = 0.0
    x[1, ::5] = -0.0
    nnz = int((x[0] != 0).sum())
    for k in sorted({1, max(nnz - 1, 0), nnz, min(nnz + 1, d), (7 * d) // 10, d - 1}):
        _check_row_block(x, dtype, k)
