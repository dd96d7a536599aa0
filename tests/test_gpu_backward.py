"""Straight-through-estimator backward of the sparse projection on the GPU
against oracle.sparse_linear_backward_ste (Q-Sparse news article, section
"Top-K sparsification", STE paragraphs): grad_x = dL/dY . W (no mask) and
grad_wt += X_sparse^T . dL/dY, accumulated into the kept rows only.

grad_wt starts from random values (with -0.0 among them): rows that no token
kept must come back bit for bit unchanged; kept rows must equal start +
oracle within the f32 tolerance."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_F32, check_status, need_gpu, to_dev

pytestmark = pytest.mark.gpu

_cache = {}


def _start_grad(d_in, d_out, seed):
    g = workloads.rng(seed)
    G0 = workloads.normal_f32(g, (d_in, d_out))
    G0[::7, ::5] = np.float32(-0.0)
    return G0


def _check(x, wt, gy, k, dtype, block=1, rows_sample=None, tok_sample=None):
    T, d_in = x.shape
    d_out = wt.shape[1]
    xt, wtt, gyt = to_dev(x, dtype), to_dev(wt, dtype), to_dev(gy, dtype)
    G0 = _start_grad(d_in, d_out, T + d_in + d_out)
    gwt = torch.from_numpy(G0.copy()).cuda()
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, xt.device)
    r = qs.qs_sparse_linear_backward(xt, wtt, gyt, k, grad_wt=gwt, block=block, ws=ws)
    check_status(ws)
    keep = oracle.block_topk_keep(x, k, block)
    xs = x.astype(np.float64) * oracle.mask_from_keep(keep, T, d_in)
    kept_rows = np.any(xs != 0, axis=0)
    got_wt = r.grad_wt.cpu().numpy()
    # untouched rows: bit for bit
    assert np.array_equal(got_wt[~kept_rows].view(np.int32), G0[~kept_rows].view(np.int32))
    rows = np.flatnonzero(kept_rows) if rows_sample is None else \
        np.intersect1d(np.flatnonzero(kept_rows), rows_sample)
    gy64 = gy.astype(np.float64)
    ref_wt = G0[rows].astype(np.float64) + xs[:, rows].T @ gy64
    assert oracle.max_rel_err(got_wt[rows], ref_wt) <= TOL_F32
    toks = np.arange(T) if tok_sample is None else tok_sample
    ref_x = gy64[toks] @ wt.astype(np.float64).T
    assert oracle.max_rel_err(r.grad_x.cpu().numpy()[toks], ref_x) <= TOL_F32
    if rows_sample is None and tok_sample is None:
        # the full oracle on small cases
        ref = oracle.sparse_linear_backward_ste(x, wt, k, gy, keep=keep)
        assert oracle.max_rel_err(r.grad_x.cpu().numpy(), ref["grad_x"]) <= TOL_F32
        full = G0.astype(np.float64) + ref["grad_wt"]
        assert oracle.max_rel_err(got_wt[kept_rows], full[kept_rows]) <= TOL_F32
    return r


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_backward_decode_llama_up_shape(dtype, T):
    """4096 -> 11008, K = floor(0.7 * 4096): grad_x streams every row of W^T,
    grad_wt adds into the rows the tokens kept."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.round_to_dtype(workloads.activations(w, T), dtype)
    key = ("wt", dtype)
    if key not in _cache:
        _cache[key] = workloads.weight_t(4096, 11008, 91, dtype)
    wt = _cache[key]
    gy = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(T), (T, 11008), 0.01), dtype)
    _check(x, wt, gy, w.k, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d_in,d_out,k,block", [
    (1, 300, 64, 0, 1),        # K = 0: grad_wt untouched, grad_x still dL/dY . W
    (1, 300, 64, 300, 1),      # K = d: every row
    (3, 77, 136, 20, 1),       # ragged rows, short last column tile
    (8, 1000, 264, 400, 4),    # Block Q-Sparse selections
    (70, 256, 96, 100, 1),     # chunks of 64 tokens (f32; bf16 takes the tensor-core path)
    (13, 512, 1552, 256, 13),  # one block of 13
])
def test_backward_ragged_and_blocks(dtype, T, d_in, d_out, k, block):
    need_gpu()
    g = workloads.rng(T * 3 + d_in + d_out + k)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), dtype)
    x[:, 5] = 0.0                    # an input no token keeps with a nonzero value
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), d_in ** -0.5), dtype)
    gy = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_out)), dtype)
    _check(x, wt, gy, k, dtype, block=block)


@pytest.mark.parametrize("T,d_in,d_out,k,block", [
    (64, 64, 256, 32, 1),        # one tile of each GEMM
    (200, 136, 264, 70, 1),      # M, N and K tails in both GEMMs (K = T for grad_wt, d_out for grad_x)
    (130, 512, 1032, 512, 1),    # K = d: dense
    (128, 256, 512, 100, 64),    # Block Q-Sparse, two blocks
    (1024, 1024, 2048, 300, 1),  # several tiles per CTA
])
def test_backward_tensor_core_ragged_tiles(T, d_in, d_out, k, block):
    """bf16 with >= 64 tokens: both gradients are tcgen05 GEMMs (K-major A and
    B for grad_x, MN-major A and B accumulating into grad_wt)."""
    need_gpu()
    g = workloads.rng(T + d_in + d_out + k + block)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), "bf16")
    x[:, 3] = 0.0
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), d_in ** -0.5), "bf16")
    gy = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_out)), "bf16")
    _check(x, wt, gy, k, "bf16", block=block)


def test_backward_prefill_full_size_sampled():
    """2048 tokens x 4096 -> 11008, K = 2048, 1% outlier channels x20: sampled
    tokens of grad_x and sampled rows of grad_wt against the oracle."""
    need_gpu()
    w = workloads.WORKLOADS["prefill_bf16_2048"]
    x = workloads.activations(w, 2048)
    wt = workloads.weight_t(w.d_in, w.d_out, w.seed(0, 1), "bf16")
    gy = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(4), (2048, w.d_out), 0.01), "bf16")
    _check(x, wt, gy, w.k, "bf16", rows_sample=np.arange(0, w.d_in, 37),
           tok_sample=np.arange(0, 2048, 61))


def test_backward_needs_an_output():
    need_gpu()
    x = torch.zeros(1, 64, device="cuda")
    wt = torch.zeros(64, 64, device="cuda")
    with pytest.raises(qs.QSError) as e:
        qs.qs_sparse_linear_backward(x, wt, torch.zeros(1, 64, device="cuda"), 8, grad_x=None,
                                     grad_wt=None)
    assert e.value.status == qs.QS_ERR_INVALID_ARG
