"""Python binding of libqs.so, the C ABI declared in include/qs.h.

Argument marshalling only: every function here checks tensor placement and
dtypes, allocates missing outputs with torch (device memory is torch's job),
and calls the C entry point of the same name on torch's current CUDA stream.
All computation happens in the library's CUDA kernels.  There is no CPU path:
if libqs.so is missing or cannot load, every call raises.

Build the library with ``python -m top_activation_sparse_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import NamedTuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqs.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "qs.h")

# ---- constants mirrored from include/qs.h ----------------------------------
QS_OK = 0
QS_ERR_INVALID_ARG = 1
QS_ERR_ALIGNMENT = 2
QS_ERR_WORKSPACE = 3
QS_ERR_CUDA = 4
QS_ERR_TIMEOUT = 5
QS_ERR_DEVICE_CHECK = 6
QS_ERR_UNSUPPORTED = 7

QS_F32 = 0
QS_BF16 = 1
QS_ACT_RELU2_GLU = 0
QS_ACT_DRELU = 1
QS_OP_TOPK_MASK = 0
QS_OP_SPARSE_LINEAR = 1
QS_OP_SPARSE_FFN = 2
QS_OP_QUANT_SPARSE_LINEAR = 3
QS_OP_TERNARY_PACK = 4
QS_OP_SPARSE_FFN_GATE_FIRST = 5
QS_OP_QUANT_SPARSE_FFN = 6

QS_FAULT_NONE = 0
QS_FAULT_GATHER_NO_COPIES = 1

QS_MAX_ROW = 49152
QS_MAX_BLOCK = 64
QS_NOALLOC_SCRATCH_BYTES = 4 << 20
QS_PREFILL_MIN_T = 64
QS_FFN_PHASE_EVENTS = 5
QS_LINEAR_PHASE_EVENTS = 3

_ACTS = {"relu2_glu": QS_ACT_RELU2_GLU, "drelu": QS_ACT_DRELU}


class QSError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {qs_status_string(status)} (status {status})")


_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float

_SIGNATURES = {
    "qs_topk_mask": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qs_sparse_linear": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qs_sparse_ffn": (_i, [_vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           _vp, _vp, _vp, _sz, _vp]),
    "qs_sparse_ffn_gate_first": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _vp, _vp, _sz, _vp]),
    "qs_quant_sparse_linear": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _f, _f, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _sz, _vp]),
    "qs_ternary_pack": (_i, [_vp, _i, _i, _f, _vp, _vp, _vp, _sz, _vp]),
    "qs_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "qs_workspace_init": (_i, [_vp, _sz, _vp]),
    "qs_device_status": (_i, [_vp, _vp]),
    "qs_workspace_stats": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "qs_status_string": (ctypes.c_char_p, [_i]),
    "qs_block_sparse_linear": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qs_block_sparse_ffn": (_i, [_vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qs_block_quant_sparse_linear": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _f, _f, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _sz, _vp]),
    "qs_sparse_linear_backward": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz,
                                       _vp]),
    "qs_quant_sparse_ffn": (_i, [_vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _f, _vp, _f,
                                 _f, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qs_sparse_linear_noalloc": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "qs_sparse_linear_noalloc_status": (_i, [_vp]),
    "qs_workspace_list": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "qs_debug_inject": (_i, [_i, ctypes.c_uint]),
    "qs_sparse_ffn_fused": (_i, [_i, _i, _i, _i, _i]),
    "qs_set_ffn_fused": (_i, [_i]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libqs.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build the CUDA library with "
                "`python -m top_activation_sparse_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/qs.h declares (for export checks)."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qs_[a-z_0-9]+)\s*\(", text)))


def qs_status_string(status: int) -> str:
    return lib().qs_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != QS_OK:
        raise QSError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return QS_F32
    if t.dtype == torch.bfloat16:
        return QS_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (the library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on one device")
    return dev


def _out(spec, shape, dtype, device):
    """spec: a tensor (used as is), True (allocate), or None/False (skip)."""
    if spec is None or spec is False:
        return None
    if spec is True:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(spec.shape) != tuple(shape) or spec.dtype != dtype:
        raise ValueError(f"output must be {tuple(shape)} {dtype}, got {tuple(spec.shape)} {spec.dtype}")
    return spec


# ---- workspace ----------------------------------------------------------------

def qs_workspace_size(op: int, T: int, d_in: int, d_out: int, k: int) -> int:
    return int(lib().qs_workspace_size(op, T, d_in, d_out, k))


def qs_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check("qs_workspace_init", lib().qs_workspace_init(ws.data_ptr(), ws.numel(), _stream_ptr(stream)))


def new_workspace(op: int, T: int, d_in: int, d_out: int, k: int, device) -> torch.Tensor:
    """A zero-filled workspace of qs_workspace_size(...) bytes on `device`."""
    n = qs_workspace_size(op, T, d_in, d_out, k)
    if n == 0:
        raise ValueError("invalid sizes for this op")
    return torch.zeros(n, dtype=torch.uint8, device=device)


_ws_cache: dict = {}


def _workspace(ws, op, T, d_in, d_out, k, device):
    if ws is not None:
        return ws
    need = qs_workspace_size(op, T, d_in, d_out, k)
    key = (device, op)
    cur = _ws_cache.get(key)
    if cur is None or cur.numel() < need:
        cur = torch.zeros(max(need, 1), dtype=torch.uint8, device=device)
        _ws_cache[key] = cur
    return cur


def qs_device_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().qs_device_status(ws.data_ptr(), _stream_ptr(stream)))


def qs_workspace_stats(ws: torch.Tensor, op: int, T: int, d_in: int, d_out: int, k: int,
                       stream=None) -> tuple[int, ...]:
    """Weight rows the last call streamed: (input rows, h rows), plus the
    rows of W_up read for QS_OP_SPARSE_FFN_GATE_FIRST."""
    rows = (ctypes.c_int32 * 3)()
    _check("qs_workspace_stats",
           lib().qs_workspace_stats(ws.data_ptr(), op, T, d_in, d_out, k, rows, _stream_ptr(stream)))
    if op == QS_OP_SPARSE_FFN_GATE_FIRST:
        return int(rows[0]), int(rows[1]), int(rows[2])
    return int(rows[0]), int(rows[1])


def qs_workspace_list(ws: torch.Tensor, op: int, T: int, d_in: int, d_out: int, k: int,
                      which: int = 0, values: bool = False, stream=None):
    """The kept-row list the last call left in `ws` (see include/qs.h):
    (rows int32 [n], values or None).  values (one-token calls only): float32
    of the kept inputs, or the int8 codes for QS_OP_QUANT_SPARSE_LINEAR."""
    import numpy as np
    cap = d_in if which == 0 else d_out
    rows = np.zeros(max(cap, 1), dtype=np.int32)
    vals = None
    if values:
        codes = op in (QS_OP_QUANT_SPARSE_LINEAR, QS_OP_QUANT_SPARSE_FFN)
        vals = np.zeros(max(cap, 1), dtype=np.int8 if codes else np.float32)
    count = ctypes.c_int32(0)
    _check("qs_workspace_list", lib().qs_workspace_list(
        ws.data_ptr(), op, T, d_in, d_out, k, which, rows.ctypes.data, cap,
        None if vals is None else vals.ctypes.data, ctypes.byref(count), _stream_ptr(stream)))
    n = int(count.value)
    if not 0 <= n <= cap:
        raise RuntimeError(f"qs_workspace_list: inconsistent row count {n}")
    return rows[:n].copy(), (None if vals is None else vals[:n].copy())


def qs_sparse_ffn_fused(dtype: int, T: int, d_model: int, d_ff: int, with_idx_h: bool = False) -> bool:
    """True if qs_sparse_ffn with these sizes runs as one persistent kernel."""
    return bool(lib().qs_sparse_ffn_fused(int(dtype), int(T), int(d_model), int(d_ff),
                                          1 if with_idx_h else 0))


def qs_set_ffn_fused(mode) -> None:
    """The one-kernel path of one-token bf16 FFN calls (process-wide): False/0 off,
    True/1 on with an ordinary launch (the default), 2 on with a cooperative launch."""
    _check("qs_set_ffn_fused", lib().qs_set_ffn_fused(int(mode)))


def qs_debug_inject(mode: int, wait_polls: int = 0) -> None:
    """Failure-detection test hook (see include/qs.h)."""
    _check("qs_debug_inject", lib().qs_debug_inject(int(mode), int(wait_polls)))


def qs_sparse_linear_noalloc_status(stream=None) -> int:
    """Read and clear the status word of the no-allocation entry point's scratch."""
    return int(lib().qs_sparse_linear_noalloc_status(_stream_ptr(stream)))


# ---- operations -------------------------------------------------------------

class TopkResult(NamedTuple):
    idx: torch.Tensor
    val: torch.Tensor | None
    mask: torch.Tensor | None
    xs: torch.Tensor | None


def qs_topk_mask(x: torch.Tensor, k: int, idx=True, val=None, mask=None, xs=None, ws=None,
                 stream=None) -> TopkResult:
    """Top-K on |x| per row: kept indices (ascending), values, mask and X_sparse."""
    dev = _need_cuda(x)
    T, d = x.shape
    idx = _out(idx if idx is not None else True, (T, k), torch.int32, dev)
    val = _out(val, (T, k), x.dtype, dev)
    mask = _out(mask, (T, d), torch.uint8, dev)
    xs = _out(xs, (T, d), x.dtype, dev)
    _need_cuda(idx, val, mask, xs)
    ws = _workspace(ws, QS_OP_TOPK_MASK, T, d, 0, k, dev)
    _check("qs_topk_mask", lib().qs_topk_mask(
        x.data_ptr(), _dtype_code(x), T, d, k, _ptr(idx), _ptr(val), _ptr(mask), _ptr(xs),
        ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    return TopkResult(idx, val, mask, xs)


def _events(phase_events, n):
    if phase_events is None:
        return None
    if len(phase_events) != n:
        raise ValueError(f"phase_events must hold {n} events")
    return (ctypes.c_void_p * n)(*[e.cuda_event for e in phase_events])


def qs_sparse_linear(x: torch.Tensor, wt: torch.Tensor, k: int, y=None, phase_events=None,
                     ws=None, stream=None, block: int = 1) -> torch.Tensor:
    """Y = (X (.) topK-mask(|X|)) . W^T with wt = W^T [d_in, d_out].
    block > 1: Block Q-Sparse (qs_block_sparse_linear)."""
    dev = _need_cuda(x, wt)
    T, d_in = x.shape
    d_out = wt.shape[1]
    if wt.shape[0] != d_in or wt.dtype != x.dtype:
        raise ValueError("wt must be [d_in, d_out] with x's dtype")
    y = _out(y if y is not None else True, (T, d_out), x.dtype, dev)
    _need_cuda(y)
    ws = _workspace(ws, QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, dev)
    ev = _events(phase_events, QS_LINEAR_PHASE_EVENTS)
    if block == 1:
        _check("qs_sparse_linear", lib().qs_sparse_linear(
            x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, wt.data_ptr(), y.data_ptr(), ev,
            ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    else:
        _check("qs_block_sparse_linear", lib().qs_block_sparse_linear(
            x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, int(block), wt.data_ptr(),
            y.data_ptr(), ev, ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    return y


def qs_sparse_linear_noalloc(x: torch.Tensor, wt: torch.Tensor, k: int, y=None,
                             stream=None) -> torch.Tensor:
    """qs_sparse_linear for callers that cannot allocate device memory: the
    scratch comes from a fixed array inside the library (all calls share it;
    calls that overlap on the GPU race).  y must be passed in by such callers;
    if it is omitted it is allocated here, for convenience only."""
    dev = _need_cuda(x, wt)
    T, d_in = x.shape
    d_out = wt.shape[1]
    if wt.shape[0] != d_in or wt.dtype != x.dtype:
        raise ValueError("wt must be [d_in, d_out] with x's dtype")
    y = _out(y if y is not None else True, (T, d_out), x.dtype, dev)
    _need_cuda(y)
    _check("qs_sparse_linear_noalloc", lib().qs_sparse_linear_noalloc(
        x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, wt.data_ptr(), y.data_ptr(),
        _stream_ptr(stream)))
    return y


class BackwardResult(NamedTuple):
    grad_x: torch.Tensor | None
    grad_wt: torch.Tensor | None


def qs_sparse_linear_backward(x, wt, grad_y, k: int, grad_x=True, grad_wt=True, block: int = 1,
                              ws=None, stream=None) -> BackwardResult:
    """Straight-through-estimator gradients of Y = X_sparse . W^T:
    grad_x = grad_y . W (f32, overwritten) and grad_wt += X_sparse^T . grad_y
    (f32, accumulated into the kept rows only; True allocates zeros)."""
    dev = _need_cuda(x, wt, grad_y)
    T, d_in = x.shape
    d_out = wt.shape[1]
    if wt.shape[0] != d_in or wt.dtype != x.dtype or tuple(grad_y.shape) != (T, d_out) \
            or grad_y.dtype != x.dtype:
        raise ValueError("need wt [d_in, d_out] and grad_y [T, d_out] with x's dtype")
    grad_x = _out(grad_x, (T, d_in), torch.float32, dev)
    if grad_wt is True:
        grad_wt = torch.zeros(d_in, d_out, dtype=torch.float32, device=dev)
    grad_wt = _out(grad_wt, (d_in, d_out), torch.float32, dev)
    _need_cuda(grad_x, grad_wt)
    ws = _workspace(ws, QS_OP_SPARSE_LINEAR, T, d_in, d_out, k, dev)
    _check("qs_sparse_linear_backward", lib().qs_sparse_linear_backward(
        x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, int(block), wt.data_ptr(),
        grad_y.data_ptr(), _ptr(grad_x), _ptr(grad_wt), ws.data_ptr(), ws.numel(),
        _stream_ptr(stream)))
    return BackwardResult(grad_x, grad_wt)


class FfnResult(NamedTuple):
    y: torch.Tensor
    h: torch.Tensor | None
    idx_h: torch.Tensor | None


def qs_sparse_ffn(x, wt_up, wt_gate, wt_down, act, k_in: int, k_h: int, b_up=None, b_gate=None,
                  y=None, h_out=None, idx_h_out=None, phase_events=None, ws=None,
                  stream=None, block: int = 1) -> FfnResult:
    """One sparse gated FFN layer (top-K on x, up/gate, gating, top-K on |h|, down).
    block > 1: Block Q-Sparse selections on x and h (qs_block_sparse_ffn)."""
    dev = _need_cuda(x, wt_up, wt_gate, wt_down, b_up, b_gate)
    T, d_model = x.shape
    d_ff = wt_up.shape[1]
    for w, shp in ((wt_up, (d_model, d_ff)), (wt_gate, (d_model, d_ff)), (wt_down, (d_ff, d_model))):
        if tuple(w.shape) != shp or w.dtype != x.dtype:
            raise ValueError(f"weight must be {shp} {x.dtype}")
    for b in (b_up, b_gate):
        if b is not None and (tuple(b.shape) != (d_ff,) or b.dtype != torch.float32):
            raise ValueError("biases must be [d_ff] float32")
    act_code = _ACTS[act] if isinstance(act, str) else int(act)
    y = _out(y if y is not None else True, (T, d_model), x.dtype, dev)
    h_out = _out(h_out, (T, d_ff), torch.float32, dev)
    idx_h_out = _out(idx_h_out, (T, k_h), torch.int32, dev)
    _need_cuda(y, h_out, idx_h_out)
    ev = _events(phase_events, QS_FFN_PHASE_EVENTS)
    ws = _workspace(ws, QS_OP_SPARSE_FFN, T, d_model, d_ff, k_h, dev)
    if block == 1:
        _check("qs_sparse_ffn", lib().qs_sparse_ffn(
            x.data_ptr(), _dtype_code(x), T, d_model, d_ff, act_code, k_in, k_h,
            wt_up.data_ptr(), wt_gate.data_ptr(), _ptr(b_up), _ptr(b_gate), wt_down.data_ptr(),
            y.data_ptr(), _ptr(h_out), _ptr(idx_h_out), ev, ws.data_ptr(), ws.numel(),
            _stream_ptr(stream)))
    else:
        _check("qs_block_sparse_ffn", lib().qs_block_sparse_ffn(
            x.data_ptr(), _dtype_code(x), T, d_model, d_ff, act_code, k_in, k_h, int(block),
            wt_up.data_ptr(), wt_gate.data_ptr(), _ptr(b_up), _ptr(b_gate), wt_down.data_ptr(),
            y.data_ptr(), _ptr(h_out), _ptr(idx_h_out), ev, ws.data_ptr(), ws.numel(),
            _stream_ptr(stream)))
    return FfnResult(y, h_out, idx_h_out)


def qs_sparse_ffn_gate_first(x, wt_gate, w_up, wt_down, k_h: int, b_up=None, b_gate=None,
                             y=None, h_out=None, idx_h_out=None, phase_events=None, ws=None,
                             stream=None) -> FfnResult:
    """dReLU FFN layer with dense x, the gate first and the up projection
    only over open gates.  w_up is [d_ff, d_model] (output-major)."""
    dev = _need_cuda(x, wt_gate, w_up, wt_down, b_up, b_gate)
    T, d_model = x.shape
    d_ff = wt_gate.shape[1]
    for w, shp in ((wt_gate, (d_model, d_ff)), (w_up, (d_ff, d_model)), (wt_down, (d_ff, d_model))):
        if tuple(w.shape) != shp or w.dtype != x.dtype:
            raise ValueError(f"weight must be {shp} {x.dtype}")
    for b in (b_up, b_gate):
        if b is not None and (tuple(b.shape) != (d_ff,) or b.dtype != torch.float32):
            raise ValueError("biases must be [d_ff] float32")
    y = _out(y if y is not None else True, (T, d_model), x.dtype, dev)
    h_out = _out(h_out, (T, d_ff), torch.float32, dev)
    idx_h_out = _out(idx_h_out, (T, k_h), torch.int32, dev)
    _need_cuda(y, h_out, idx_h_out)
    ev = _events(phase_events, QS_FFN_PHASE_EVENTS)
    ws = _workspace(ws, QS_OP_SPARSE_FFN_GATE_FIRST, T, d_model, d_ff, k_h, dev)
    _check("qs_sparse_ffn_gate_first", lib().qs_sparse_ffn_gate_first(
        x.data_ptr(), _dtype_code(x), T, d_model, d_ff, k_h, wt_gate.data_ptr(), w_up.data_ptr(),
        _ptr(b_up), _ptr(b_gate), wt_down.data_ptr(), y.data_ptr(), _ptr(h_out), _ptr(idx_h_out),
        ev, ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    return FfnResult(y, h_out, idx_h_out)


class QuantResult(NamedTuple):
    y: torch.Tensor
    acc: torch.Tensor | None
    q: torch.Tensor | None
    idx: torch.Tensor | None


def qs_quant_sparse_linear(x, wt_packed, alpha: float, k: int, eps: float = 1e-5, y=None,
                           acc=None, q=None, idx=None, phase_events=None, ws=None,
                           stream=None, block: int = 1) -> QuantResult:
    """int8 (per-token absmax) x ternary (packed 2-bit) projection of the top-K of |q|.
    block > 1: Block Q-Sparse on |q| (qs_block_quant_sparse_linear)."""
    dev = _need_cuda(x, wt_packed)
    T, d_in = x.shape
    if wt_packed.dtype != torch.int32 or wt_packed.shape[0] != d_in:
        raise ValueError("wt_packed must be [d_in, d_out/16] int32 (uint32 bit patterns)")
    d_out = wt_packed.shape[1] * 16
    y = _out(y if y is not None else True, (T, d_out), torch.float32, dev)
    acc = _out(acc, (T, d_out), torch.int32, dev)
    q = _out(q, (T, d_in), torch.int8, dev)
    idx = _out(idx, (T, k), torch.int32, dev)
    _need_cuda(y, acc, q, idx)
    ws = _workspace(ws, QS_OP_QUANT_SPARSE_LINEAR, T, d_in, d_out, k, dev)
    ev = _events(phase_events, QS_LINEAR_PHASE_EVENTS)
    if block == 1:
        _check("qs_quant_sparse_linear", lib().qs_quant_sparse_linear(
            x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, wt_packed.data_ptr(), float(alpha),
            float(eps), y.data_ptr(), _ptr(acc), _ptr(q), _ptr(idx), ev, ws.data_ptr(),
            ws.numel(), _stream_ptr(stream)))
    else:
        _check("qs_block_quant_sparse_linear", lib().qs_block_quant_sparse_linear(
            x.data_ptr(), _dtype_code(x), T, d_in, d_out, k, int(block), wt_packed.data_ptr(),
            float(alpha), float(eps), y.data_ptr(), _ptr(acc), _ptr(q), _ptr(idx), ev,
            ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    return QuantResult(y, acc, q, idx)


class QuantFfnResult(NamedTuple):
    y: torch.Tensor
    h: torch.Tensor | None


def qs_quant_sparse_ffn(x, wp_up, alpha_up: float, wp_gate, alpha_gate: float, wp_down,
                        alpha_down: float, act, k_in: int, k_h: int, eps: float = 1e-5,
                        b_up=None, b_gate=None, y=None, h_out=None, block: int = 1,
                        phase_events=None, ws=None, stream=None) -> QuantFfnResult:
    """BitNet b1.58 + Q-Sparse FFN layer: int8 x ternary up, gate and down
    projections, each input quantized per token and top-K'd (wp_*: packed
    ternary W^T from qs_ternary_pack)."""
    dev = _need_cuda(x, wp_up, wp_gate, wp_down, b_up, b_gate)
    T, d_model = x.shape
    d_ff = wp_up.shape[1] * 16
    for p_, shp in ((wp_up, (d_model, d_ff // 16)), (wp_gate, (d_model, d_ff // 16)),
                    (wp_down, (d_ff, d_model // 16))):
        if tuple(p_.shape) != shp or p_.dtype != torch.int32:
            raise ValueError(f"packed weight must be {shp} int32")
    act_code = _ACTS[act] if isinstance(act, str) else int(act)
    y = _out(y if y is not None else True, (T, d_model), torch.float32, dev)
    h_out = _out(h_out, (T, d_ff), torch.float32, dev)
    _need_cuda(y, h_out)
    ws = _workspace(ws, QS_OP_QUANT_SPARSE_FFN, T, d_model, d_ff, k_h, dev)
    _check("qs_quant_sparse_ffn", lib().qs_quant_sparse_ffn(
        x.data_ptr(), _dtype_code(x), T, d_model, d_ff, act_code, k_in, k_h, int(block),
        wp_up.data_ptr(), float(alpha_up), wp_gate.data_ptr(), float(alpha_gate),
        wp_down.data_ptr(), float(alpha_down), float(eps), _ptr(b_up), _ptr(b_gate),
        y.data_ptr(), _ptr(h_out), _events(phase_events, QS_FFN_PHASE_EVENTS), ws.data_ptr(),
        ws.numel(), _stream_ptr(stream)))
    return QuantFfnResult(y, h_out)


def qs_ternary_pack(w: torch.Tensor, eps: float = 1e-5, wt_packed=None, alpha_out=None, ws=None,
                    stream=None):
    """Ternary-quantize W [d_out, d_in] f32 and pack it input-major 2-bit.

    Returns (wt_packed [d_in, d_out/16] int32 holding uint32 bit patterns,
    alpha [1] float32 on the device)."""
    dev = _need_cuda(w)
    if w.dtype != torch.float32:
        raise ValueError("w must be float32 [d_out, d_in]")
    d_out, d_in = w.shape
    wt_packed = _out(wt_packed if wt_packed is not None else True, (d_in, d_out // 16),
                     torch.int32, dev)
    alpha_out = _out(alpha_out if alpha_out is not None else True, (1,), torch.float32, dev)
    ws = _workspace(ws, QS_OP_TERNARY_PACK, 0, d_in, d_out, 0, dev)
    _check("qs_ternary_pack", lib().qs_ternary_pack(
        w.data_ptr(), d_out, d_in, float(eps), wt_packed.data_ptr(), alpha_out.data_ptr(),
        ws.data_ptr(), ws.numel(), _stream_ptr(stream)))
    return wt_packed, alpha_out


__all__ = [n for n in dir() if n.startswith(("qs_", "QS_"))] + [
    "lib", "new_workspace", "header_functions", "QSError", "TopkResult", "FfnResult",
    "QuantResult", "BackwardResult", "QuantFfnResult"]
