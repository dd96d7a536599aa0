"""BitNet b1.58 + Q-Sparse FFN layer on the GPU against oracle.quant_sparse_ffn:
every projection input quantized per token and top-K'd, int8 x ternary up,
gate and down projections, the gating in float32 steps.  Every step is exact
integer arithmetic or a fixed float32 operation, so y is compared bit for bit
(and h by value: the sign of an exact zero is not part of the definition)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import check_status, need_gpu, to_dev

pytestmark = pytest.mark.gpu

_cache = {}


def _weights(dm, dff, seed):
    key = (dm, dff, seed)
    if key not in _cache:
        out = []
        for j, (o, i) in enumerate(((dff, dm), (dff, dm), (dm, dff))):
            t, alpha = oracle.ternary_quantize(workloads.weight_out_major(o, i, seed + j))
            out.append((t, alpha, torch.from_numpy(oracle.ternary_pack(t).view(np.int32)).cuda()))
        _cache[key] = out
    return _cache[key]


def _check(x, dtype, dm, dff, act, k_in, k_h, bias=None, block=1, seed=5):
    (tu, au, pu), (tg, ag, pg), (td, ad, pd) = _weights(dm, dff, seed)
    T = x.shape[0]
    xt = to_dev(x, dtype)
    b = None if bias is None else torch.full((dff,), bias, dtype=torch.float32, device="cuda")
    ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_FFN, T, dm, dff, k_h, xt.device)
    r = qs.qs_quant_sparse_ffn(xt, pu, au, pg, ag, pd, ad, act, k_in, k_h, b_up=b, b_gate=b,
                               h_out=True, block=block, ws=ws)
    check_status(ws)
    bnp = None if bias is None else np.full(dff, bias, np.float32)
    ref = oracle.quant_sparse_ffn(x, tu, au, tg, ag, td, ad, act, k_in, k_h, b_up=bnp, b_gate=bnp,
                                  block=block)
    assert np.array_equal(r.h.cpu().numpy(), ref["h"])
    assert np.array_equal(r.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))
    # product path without h_out: the same bits
    r2 = qs.qs_quant_sparse_ffn(xt, pu, au, pg, ag, pd, ad, act, k_in, k_h, b_up=b, b_gate=b,
                                block=block, ws=ws)
    check_status(ws)
    assert np.array_equal(r2.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))
    return ref, ws


@pytest.mark.parametrize("T", [1, 8, 32])
def test_quant_ffn_llama7b_shape(T):
    """4096 -> 11008 -> 4096, squared-ReLU gating, 39% of |q| kept at both inputs."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_relu2_llama7b"]
    x = workloads.activations(w, T)
    k_in, k_h = workloads.keep_count(0.39, 4096), workloads.keep_count(0.39, 11008)
    ref, ws = _check(x, "bf16", 4096, 11008, "relu2_glu", k_in, k_h)
    if T == 1:
        rows, codes = qs.qs_workspace_list(ws, qs.QS_OP_QUANT_SPARSE_FFN, 1, 4096, 11008, k_h, 1,
                                           values=True)
        kh = ref["keep_h"][0]
        qk = ref["q_h"][0, kh]
        assert np.array_equal(rows, kh[qk != 0].astype(np.int32))
        assert np.array_equal(codes.astype(np.int64), qk[qk != 0])


@pytest.mark.parametrize("T", [1, 4])
def test_quant_ffn_drelu_mistral7b_shape(T):
    """4096 -> 14336 -> 4096, dReLU with biases -0.8, dense x, top 10% of |q_h|."""
    need_gpu()
    w = workloads.WORKLOADS["ffn_drelu_mistral7b"]
    x = workloads.activations(w, T)
    _check(x, "bf16", 4096, 14336, "drelu", 4096, w.k_h, bias=-0.8)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("act", ["relu2_glu", "drelu"])
@pytest.mark.parametrize("T,dm,dff,block", [(1, 64, 128, 1), (3, 128, 192, 1), (9, 64, 256, 1),
                                            (70, 128, 128, 1), (8, 256, 320, 4), (12, 64, 64, 12)])
def test_quant_ffn_ragged_chunks_blocks(dtype, act, T, dm, dff, block):
    need_gpu()
    g = workloads.rng(T * 5 + dm + dff + block)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (T, dm)), dtype)
    x[0, :] = 0.0                          # a zero token: y = 0
    bias = -0.1 if act == "drelu" else None
    for k_in, k_h in ((dm, dff), ((4 * dm) // 10, (4 * dff) // 10), (1, 1), (dm, 0)):
        _check(x, dtype, dm, dff, act, k_in, k_h, bias=bias, block=block, seed=dm + dff)


def test_quant_ffn_rejects_rows_not_multiple_of_64():
    need_gpu()
    x = torch.zeros(1, 64, device="cuda")
    p1 = torch.zeros(64, 6, dtype=torch.int32, device="cuda")     # d_ff = 96
    p2 = torch.zeros(96, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(qs.QSError) as e:
        qs.qs_quant_sparse_ffn(x, p1, 1.0, p1, 1.0, p2, 1.0, "relu2_glu", 8, 8)
    assert e.value.status == qs.QS_ERR_ALIGNMENT
