"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

* libqs.so loads and exports every function include/qs.h declares;
* argument validation happens on the host before anything is enqueued, so
  bad arguments return their status code even without a device;
* workspace sizing is a pure function of the sizes.
"""
import ctypes

import pytest

import top_activation_sparse_b200 as qs
from top_activation_sparse_b200 import build as qs_build


@pytest.fixture(scope="module")
def L():
    qs_build.build()
    return qs.lib()


def test_header_declares_the_boundary():
    names = qs.header_functions()
    for n in ("qs_topk_mask", "qs_sparse_linear", "qs_sparse_ffn", "qs_sparse_ffn_gate_first",
              "qs_quant_sparse_linear",
              "qs_ternary_pack", "qs_workspace_size", "qs_workspace_init", "qs_device_status",
              "qs_workspace_stats", "qs_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in qs.header_functions():
        assert hasattr(L, n), f"libqs.so does not export {n}"


def test_status_strings(L):
    for code in range(8):
        s = qs.qs_status_string(code)
        assert s.startswith("QS_")
    assert qs.qs_status_string(99) == "unknown qs_status"


def test_workspace_size_is_host_only_and_sane(L):
    f = qs.qs_workspace_size
    assert f(qs.QS_OP_TOPK_MASK, 1, 4096, 0, 2867) > 0
    assert f(qs.QS_OP_TOPK_MASK, 1, 4096, 0, 4097) == 0            # k > d
    assert f(qs.QS_OP_TOPK_MASK, 0, 4096, 0, 1) == 0               # T < 1
    assert f(qs.QS_OP_TOPK_MASK, 1, qs.QS_MAX_ROW + 1, 0, 1) == 0  # row too long
    a = f(qs.QS_OP_SPARSE_FFN, 1, 4096, 11008, 7705)
    b = f(qs.QS_OP_SPARSE_FFN, 8, 4096, 11008, 7705)
    assert 0 < a < b
    assert f(qs.QS_OP_QUANT_SPARSE_LINEAR, 32, 4096, 11008, 1597) > 0
    assert f(qs.QS_OP_QUANT_SPARSE_LINEAR, 1, 4096, 11000, 1597) == 0   # d_out % 64
    assert f(qs.QS_OP_QUANT_SPARSE_LINEAR, 1, 4096, 48, 1597) == 0
    assert f(qs.QS_OP_TERNARY_PACK, 0, 4096, 11008, 0) > 0
    assert f(99, 1, 1, 1, 1) == 0
    # the gate-first layer needs the FFN's buffers, with partial sums sized for
    # the gate alone
    assert f(qs.QS_OP_SPARSE_FFN_GATE_FIRST, 1, 4096, 14336, 1433) > 0
    assert f(qs.QS_OP_SPARSE_FFN_GATE_FIRST, 1, 4096, 14336, 14337) == 0
    # more than the decode chunk of tokens does not grow the decode buffers
    c = f(qs.QS_OP_SPARSE_FFN, 64, 4096, 11008, 7705)
    assert f(qs.QS_OP_SPARSE_FFN, 640, 4096, 11008, 7705) == c


def _p(v):
    return ctypes.c_void_p(v)


FAKE = 0x10000      # 16-byte aligned, never dereferenced: validation fails first


def test_invalid_arguments_are_rejected_on_the_host(L):
    s = None
    ws, wsb = _p(FAKE), 1 << 30
    # qs_topk_mask: NULL x, bad dtype, k > d, k > 0 with NULL idx, T < 1, misaligned x
    assert L.qs_topk_mask(None, 0, 1, 8, 2, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_topk_mask(_p(FAKE), 7, 1, 8, 2, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_topk_mask(_p(FAKE), 0, 1, 8, 9, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_topk_mask(_p(FAKE), 0, 1, 8, 2, None, None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_topk_mask(_p(FAKE), 0, 0, 8, 2, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_topk_mask(_p(FAKE + 4), 0, 1, 8, 2, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_ALIGNMENT
    assert L.qs_topk_mask(_p(FAKE), 0, 1, qs.QS_MAX_ROW + 1, 2, _p(FAKE), None, None, None, ws, wsb, s) == qs.QS_ERR_UNSUPPORTED
    # workspace too small / missing
    assert L.qs_topk_mask(_p(FAKE), 0, 1, 8, 2, _p(FAKE), None, None, None, ws, 16, s) == qs.QS_ERR_WORKSPACE
    assert L.qs_topk_mask(_p(FAKE), 0, 1, 8, 2, _p(FAKE), None, None, None, None, wsb, s) == qs.QS_ERR_WORKSPACE
    # qs_sparse_linear: d_out not a multiple of the vector width (bf16 needs 8)
    assert L.qs_sparse_linear(_p(FAKE), 1, 1, 64, 12, 8, _p(FAKE), _p(FAKE), None, ws, wsb, s) == qs.QS_ERR_ALIGNMENT
    assert L.qs_sparse_linear(_p(FAKE), 1, 1, 64, 16, 65, _p(FAKE), _p(FAKE), None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_sparse_linear(_p(FAKE), 1, 1, 64, 16, -1, _p(FAKE), _p(FAKE), None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_sparse_linear(_p(FAKE), 1, 1, 64, 16, 8, None, _p(FAKE), None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    # qs_sparse_ffn: bad activation, k_h > d_ff
    args = [_p(FAKE), 1, 1, 64, 128, 0, 32, 64, _p(FAKE), _p(FAKE), None, None, _p(FAKE), _p(FAKE),
            None, None, None, ws, wsb, s]
    bad = list(args); bad[5] = 5
    assert L.qs_sparse_ffn(*bad) == qs.QS_ERR_INVALID_ARG
    bad = list(args); bad[7] = 129
    assert L.qs_sparse_ffn(*bad) == qs.QS_ERR_INVALID_ARG
    bad = list(args); bad[4] = 100            # d_ff % 8 != 0
    assert L.qs_sparse_ffn(*bad) == qs.QS_ERR_ALIGNMENT
    # qs_sparse_ffn_gate_first: k_h > d_ff, NULL w_up, d_model % 8, tiny workspace
    gf = [_p(FAKE), 1, 1, 64, 128, 32, _p(FAKE), _p(FAKE), None, None, _p(FAKE), _p(FAKE),
          None, None, None, ws, wsb, s]
    bad = list(gf); bad[5] = 129
    assert L.qs_sparse_ffn_gate_first(*bad) == qs.QS_ERR_INVALID_ARG
    bad = list(gf); bad[7] = None
    assert L.qs_sparse_ffn_gate_first(*bad) == qs.QS_ERR_INVALID_ARG
    bad = list(gf); bad[3] = 60
    assert L.qs_sparse_ffn_gate_first(*bad) == qs.QS_ERR_ALIGNMENT
    bad = list(gf); bad[16] = 64
    assert L.qs_sparse_ffn_gate_first(*bad) == qs.QS_ERR_WORKSPACE
    # qs_quant_sparse_linear: d_out % 16, negative eps
    assert L.qs_quant_sparse_linear(_p(FAKE), 1, 1, 64, 40, 8, _p(FAKE), ctypes.c_float(1.0),
                                    ctypes.c_float(1e-5), _p(FAKE), None, None, None, None, ws, wsb, s) == qs.QS_ERR_ALIGNMENT
    assert L.qs_quant_sparse_linear(_p(FAKE), 1, 1, 64, 32, 8, _p(FAKE), ctypes.c_float(1.0),
                                    ctypes.c_float(-1.0), _p(FAKE), None, None, None, None, ws, wsb, s) == qs.QS_ERR_INVALID_ARG
    # qs_ternary_pack: d_out % 16
    assert L.qs_ternary_pack(_p(FAKE), 24, 8, ctypes.c_float(1e-5), _p(FAKE), None, ws, wsb, s) == qs.QS_ERR_ALIGNMENT
    assert L.qs_workspace_init(None, 16, s) == qs.QS_ERR_INVALID_ARG
    assert L.qs_device_status(None, s) == qs.QS_ERR_INVALID_ARG


def test_python_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(1, 8)
    with pytest.raises(ValueError):
        qs.qs_topk_mask(x, 2)


def test_noalloc_entry_point_checks_sizes_on_the_host(L):
    # rejected before any CUDA call: works without a device
    big = (64, 16384, 16384, 8192)
    assert qs.qs_workspace_size(qs.QS_OP_SPARSE_LINEAR, *big) > qs.QS_NOALLOC_SCRATCH_BYTES
    assert L.qs_sparse_linear_noalloc(_p(FAKE), 0, *big, _p(FAKE), _p(FAKE), None) == qs.QS_ERR_UNSUPPORTED
    assert L.qs_sparse_linear_noalloc(None, 0, 1, 8, 8, 4, _p(FAKE), _p(FAKE), None) == qs.QS_ERR_INVALID_ARG
    assert L.qs_sparse_linear_noalloc(_p(FAKE), 0, 1, 8, 8, 9, _p(FAKE), _p(FAKE), None) == qs.QS_ERR_INVALID_ARG


def test_noalloc_entry_point_checks_arguments_before_enqueuing(L):
    """Every argument check of qs_sparse_linear runs before the no-allocation
    entry point touches its scratch array: these return their codes without a
    device, i.e. nothing was enqueued."""
    s = None
    assert L.qs_sparse_linear_noalloc(_p(FAKE), 7, 1, 64, 64, 8, _p(FAKE), _p(FAKE), s) == \
        qs.QS_ERR_INVALID_ARG                                          # dtype
    assert L.qs_sparse_linear_noalloc(_p(FAKE + 4), 0, 1, 64, 64, 8, _p(FAKE), _p(FAKE), s) == \
        qs.QS_ERR_ALIGNMENT                                            # misaligned x
    assert L.qs_sparse_linear_noalloc(_p(FAKE), 1, 1, 64, 60, 8, _p(FAKE), _p(FAKE), s) == \
        qs.QS_ERR_ALIGNMENT                                            # bf16 d_out % 8
    assert L.qs_sparse_linear_noalloc(_p(FAKE), 0, 1, 64, 64, 65, _p(FAKE), _p(FAKE), s) == \
        qs.QS_ERR_INVALID_ARG                                          # k > d_in


def test_workspace_list_and_fault_hook_check_arguments_on_the_host(L):
    rows = (ctypes.c_int32 * 8)()
    vals = (ctypes.c_float * 8)()
    cnt = ctypes.c_int32(0)
    ws = _p(FAKE)
    lin = qs.QS_OP_SPARSE_LINEAR
    assert L.qs_workspace_list(None, lin, 1, 64, 64, 8, 0, rows, 8, None, ctypes.byref(cnt), None) == \
        qs.QS_ERR_INVALID_ARG                                          # no workspace
    assert L.qs_workspace_list(ws, lin, 1, 64, 64, 8, 1, rows, 8, None, ctypes.byref(cnt), None) == \
        qs.QS_ERR_INVALID_ARG                                          # no h list here
    assert L.qs_workspace_list(ws, lin, 2, 64, 64, 8, 0, rows, 8, vals, ctypes.byref(cnt), None) == \
        qs.QS_ERR_INVALID_ARG                                          # values: one token only
    assert L.qs_workspace_list(ws, qs.QS_OP_TOPK_MASK, 1, 64, 0, 8, 0, rows, 8, None,
                               ctypes.byref(cnt), None) == qs.QS_ERR_INVALID_ARG
    assert L.qs_workspace_list(ws, lin, 1, 64, 64, 65, 0, rows, 8, None, ctypes.byref(cnt), None) == \
        qs.QS_ERR_INVALID_ARG                                          # k > d_in
    assert L.qs_debug_inject(9, 0) == qs.QS_ERR_INVALID_ARG
    assert L.qs_debug_inject(qs.QS_FAULT_NONE, 0) == qs.QS_OK


def test_ffn_fused_switch_takes_three_modes(L):
    for bad in (-1, 3):
        assert L.qs_set_ffn_fused(bad) == qs.QS_ERR_INVALID_ARG
    for mode in (0, 2, 1):                             # ends on the default
        assert L.qs_set_ffn_fused(mode) == qs.QS_OK
