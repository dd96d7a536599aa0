"""Failure detection on the GPU without a fault: every device-side wait is
bounded, and a wait that runs out becomes QS_ERR_TIMEOUT on the host while
the context stays usable.

The failure is made on the host (qs_debug_inject): the gather kernel's
producer warp issues no weight copies at all, so no copy is ever in flight and
the consumers' waits on the stage barriers, which nothing will complete, run
out after a short limit.  The kernel records the timeout in the workspace's
status word and still finishes its tickets, so the next normal call on the
same workspace is correct."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import TOL_BF16, TOL_F32, check_status, need_gpu, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gather_wait_that_runs_out_reports_timeout_then_recovers(dtype):
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    T, d_in, d_out, k = 1, 4096, 11008, w.k
    x = workloads.round_to_dtype(workloads.activations(w, 1)[0:1], dtype)
    wt = workloads.weight_t(d_in, d_out, 99, dtype)
    xt, wtt = to_dev(x, dtype), to_dev(wt, dtype)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, xt.device)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    ref = oracle.sparse_linear(x, wt, k)
    for _ in range(2):
        try:
            qs.qs_debug_inject(qs.QS_FAULT_GATHER_NO_COPIES, 4096)
            qs.qs_sparse_linear(xt, wtt, k, ws=ws)
        finally:
            qs.qs_debug_inject(qs.QS_FAULT_NONE)
        assert qs.qs_device_status(ws) == qs.QS_ERR_TIMEOUT
        assert qs.qs_device_status(ws) == qs.QS_OK          # read and cleared
        # the next normal call on the same workspace
        y = qs.qs_sparse_linear(xt, wtt, k, ws=ws)
        check_status(ws)
        assert oracle.max_rel_err(to_np(y), ref) <= tol


def test_timeout_in_the_ffn_down_projection_is_reported():
    """The whole layer: up/gate and down gathers time out, the status says so,
    the next normal layer on the same workspace matches the oracle."""
    need_gpu()
    g = workloads.rng(3)
    dm, dff = 256, 512
    x = workloads.round_to_dtype(workloads.normal_f32(g, (1, dm)), "bf16")
    up = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), "bf16")
    gate = workloads.round_to_dtype(workloads.normal_f32(g, (dm, dff), dm ** -0.5), "bf16")
    down = workloads.round_to_dtype(workloads.normal_f32(g, (dff, dm), dff ** -0.5), "bf16")
    ts = [to_dev(a, "bf16") for a in (x, up, gate, down)]
    ws = qs.new_workspace(qs.QS_OP_SPARSE_FFN, 1, dm, dff, dff // 2, ts[0].device)
    try:
        qs.qs_debug_inject(qs.QS_FAULT_GATHER_NO_COPIES, 4096)
        qs.qs_sparse_ffn(*ts, "relu2_glu", (7 * dm) // 10, dff // 2, ws=ws)
    finally:
        qs.qs_debug_inject(qs.QS_FAULT_NONE)
    assert qs.qs_device_status(ws) == qs.QS_ERR_TIMEOUT
    r = qs.qs_sparse_ffn(*ts, "relu2_glu", (7 * dm) // 10, dff // 2, h_out=True, ws=ws)
    check_status(ws)
    h = r.h.cpu().numpy()
    ref = oracle.sparse_ffn(x, up, gate, down, "relu2_glu", (7 * dm) // 10, dff // 2,
                            keep_h=oracle.topk_keep(h.astype(np.float64), dff // 2))
    assert oracle.max_rel_err(h, ref["h"]) <= TOL_F32
    assert oracle.max_rel_err(to_np(r.y), ref["y"]) <= TOL_BF16
