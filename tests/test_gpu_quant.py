"""BitNet b1.58 + Q-Sparse path on the GPU against the oracle: the ternary
pack, alpha, the int8 codes, the kept indices, the int32 accumulators and the
f32 outputs are all bit-exact (fixed float32 op order on both sides)."""
import numpy as np
import pytest
import torch

import oracle
import top_activation_sparse_b200 as qs
import workloads
from gpu_common import check_status, need_gpu, to_dev

pytestmark = pytest.mark.gpu

_packed = {}


def _pack_on_gpu(W):
    wt = torch.from_numpy(W).cuda()
    ws = qs.new_workspace(qs.QS_OP_TERNARY_PACK, 0, W.shape[1], W.shape[0], 0, wt.device)
    p, alpha = qs.qs_ternary_pack(wt, 1e-5, ws=ws)
    check_status(ws)
    return p, alpha


def _weights(d_out, d_in, seed):
    key = (d_out, d_in, seed)
    if key not in _packed:
        W = workloads.weight_out_major(d_out, d_in, seed)
        t, alpha = oracle.ternary_quantize(W)
        _packed[key] = (W, t, alpha, oracle.ternary_pack(t))
    return _packed[key]


@pytest.mark.parametrize("d_out,d_in", [(11008, 4096), (4096, 11008), (32, 5)])
def test_ternary_pack_bit_exact(d_out, d_in):
    need_gpu()
    W, t, alpha, packed = _weights(d_out, d_in, d_out + d_in)
    p, a = _pack_on_gpu(W)
    assert np.float32(a.item()) == alpha
    assert np.array_equal(p.cpu().numpy().view(np.uint32), packed)


def _check_quant(x, dtype, t, alpha, packed, k):
    T, d_in = x.shape
    d_out = t.shape[0]
    xt = to_dev(x, dtype)
    pt = torch.from_numpy(packed.view(np.int32)).cuda()
    ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_LINEAR, T, d_in, d_out, k, xt.device)
    r = qs.qs_quant_sparse_linear(xt, pt, float(alpha), k, 1e-5, acc=True, q=True, idx=True, ws=ws)
    check_status(ws)
    ref = oracle.quant_sparse_linear(x, t, alpha, k)
    assert np.array_equal(r.q.cpu().numpy().astype(np.int64), ref["q"])
    assert np.array_equal(r.idx.cpu().numpy().astype(np.int64), ref["keep"])
    assert np.array_equal(r.acc.cpu().numpy().astype(np.int64), ref["acc"])
    assert np.array_equal(r.y.cpu().numpy().view(np.int32), ref["y"].view(np.int32))


@pytest.mark.parametrize("T", [1, 8, 32])
@pytest.mark.parametrize("name", ["quant_up_4096x11008", "quant_down_11008x4096"])
def test_quant_sparse_linear_bitnet_shapes(name, T):
    """7B shapes, 39% kept, int8 x ternary, batch 1 / 8 / 32: everything bit-exact."""
    need_gpu()
    w = workloads.WORKLOADS[name]
    W, t, alpha, packed = _weights(w.d_out, w.d_in, w.d_out + w.d_in)
    x = workloads.activations(w, T)
    _check_quant(x, "bf16", t, alpha, packed, w.k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quant_edge_cases(dtype):
    need_gpu()
    d_in, d_out = 300, 64
    W = workloads.weight_out_major(d_out, d_in, 9)
    t, alpha = oracle.ternary_quantize(W)
    packed = oracle.ternary_pack(t)
    g = workloads.rng(10)
    x = workloads.round_to_dtype(workloads.normal_f32(g, (5, d_in)), dtype)
    x[1] = 0.0                               # zero row: q = 0, y = 0
    x[2] = 0.0
    x[2, 17] = -7.5                          # one nonzero: q = -127 there
    x[3] = np.float32(0.5)                   # all ties
    x[4, :5] = workloads.round_to_dtype(np.array([3e-5, 1e-5, -2.2e-5, 0, 0], np.float32), dtype)
    x[4, 5:] = 0.0                           # tiny magnitudes: epsilon matters
    for k in (0, 1, 117, d_in - 1, d_in):
        _check_quant(x, dtype, t, alpha, packed, k)


def test_quant_chunked_tokens():
    need_gpu()
    d_in, d_out = 256, 64
    W = workloads.weight_out_major(d_out, d_in, 12)
    t, alpha = oracle.ternary_quantize(W)
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(13), (70, d_in)), "bf16")
    _check_quant(x, "bf16", t, alpha, oracle.ternary_pack(t), 100)


def test_quant_rejects_unaligned_packed_rows():
    """Packed rows move in 16-byte bulk copies: d_out must be a multiple of 64."""
    need_gpu()
    x = torch.zeros(1, 32, device="cuda")
    p = torch.zeros(32, 3, dtype=torch.int32, device="cuda")      # d_out = 48
    with pytest.raises(qs.QSError) as e:
        qs.qs_quant_sparse_linear(x, p, 1.0, 8)
    assert e.value.status == qs.QS_ERR_ALIGNMENT


@pytest.mark.parametrize("T", [12, 20])
@pytest.mark.parametrize("k", [1, 37, 300])
def test_quant_tensor_core_token_groups(T, k):
    """8 or more tokens take the tensor-core kernel (m16n8k32 s8): 12 and 20
    tokens use 16- and 24-token groups with empty token slots; K = 1 and 37
    leave a short last stage of 32 rows.  Everything bit-exact."""
    need_gpu()
    d_in, d_out = 300, 320
    W = workloads.weight_out_major(d_out, d_in, 21)
    t, alpha = oracle.ternary_quantize(W)
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(22 + T), (T, d_in)), "bf16")
    _check_quant(x, "bf16", t, alpha, oracle.ternary_pack(t), k)


@pytest.mark.parametrize("T,d_in,d_out,k", [
    (8, 304, 320, 100),       # rows not a multiple of 32, a 64-column last tile
    (9, 112, 64, 111),        # 16-token padding, one short tile
    (16, 512, 1088, 200),
    (17, 1024, 256, 400),     # 32-token padding
    (33, 2048, 4096, 800),    # 48-token padding
    (64, 4096, 11008, 1597),  # 64 tokens at the 7B shape
    (24, 608, 384, 0),        # K = 0: y = 0
    (40, 608, 384, 608),      # K = d: every input
])
def test_quant_tcgen05_int8_kernel(T, d_in, d_out, k):
    """8 to 64 tokens with per-token selections (d_in % 16 == 0) run the
    tcgen05 kind::i8 kernel (every packed row streamed, int32 in tensor
    memory): q, kept indices, acc and y bit-exact against the oracle."""
    need_gpu()
    W = workloads.weight_out_major(d_out, d_in, d_out + 3 * d_in)
    t, alpha = oracle.ternary_quantize(W)
    x = workloads.round_to_dtype(workloads.normal_f32(workloads.rng(T + d_in), (T, d_in)), "bf16")
    x[T // 2] = 0.0                          # a zero token
    _check_quant(x, "bf16", t, alpha, oracle.ternary_pack(t), k)
