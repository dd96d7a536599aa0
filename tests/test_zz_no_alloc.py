"""qs_sparse_linear_noalloc, the entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), checked
against qs_sparse_linear with a caller workspace on the same inputs and
against the fp64 oracle, on two calls in a row (the second call finds the
array as the first one left it); the array's status word is read after each
call."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,T,d_in,d_out,k", [
    ("bf16", 1, 4096, 11008, 2867),     # Llama-7B up projection shape, 70% kept
    ("bf16", 8, 4096, 11008, 2867),
    ("f32", 4, 512, 512, 256),
])
def test_noalloc_matches_workspace_entry_point(dtype, T, d_in, d_out, k):
    need_gpu()
    g = workloads.rng(T * 31 + d_in)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, d_in)), dtype)
    wt = workloads.round_to_dtype(workloads.normal_f32(g, (d_in, d_out), d_in ** -0.5), dtype)
    xt, wtt = to_dev(x, dtype), to_dev(wt, dtype)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, xt.device)
    y_ref = qs.qs_sparse_linear(xt, wtt, k, ws=ws)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    ref = oracle.sparse_linear(x, wt, k)
    for _ in range(2):
        y = torch.full_like(y_ref, float("nan"))
        qs.qs_sparse_linear_noalloc(xt, wtt, k, y=y)
        assert qs.qs_sparse_linear_noalloc_status() == qs.QS_OK
        assert torch.isfinite(y.float()).all()
        assert oracle.max_rel_err(to_np(y), to_np(y_ref)) <= tol
        assert oracle.max_rel_err(to_np(y), ref) <= tol


def test_noalloc_rejects_sizes_beyond_its_scratch():
    need_gpu()
    T, d = 64, 16384
    assert qs.qs_workspace_size(qs.QS_OP_SPARSE_LINEAR, T, d, d, d) > qs.QS_NOALLOC_SCRATCH_BYTES
    x = torch.zeros(T, d, device="cuda")
    wt = torch.zeros(d, d, device="cuda")
    with pytest.raises(qs.QSError) as e:
        qs.qs_sparse_linear_noalloc(x, wt, d // 2)
    assert e.value.status == qs.QS_ERR_UNSUPPORTED
