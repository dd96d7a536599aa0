"""Shared helpers for the GPU parity tests (inputs from workloads.py go to
both sides; expected values come only from oracle/)."""
import numpy as np
import pytest
import torch

import top_activation_sparse_b200 as qs

# Tolerances (max relative error, row infinity norm as denominator), from the
# stated accuracy targets: f32 outputs 2e-3, bf16 outputs (f32 accumulate) 1.5e-2.
TOL_F32 = 2e-3
TOL_BF16 = 1.5e-2


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from top_activation_sparse_b200 import build
    build.build()


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.cuda()


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a float tensor (for bit-exact comparisons)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).cpu().numpy()
    return t.cpu().numpy()


def np_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "bf16":
        return (a.view(np.uint32) >> 16).astype(np.uint16).view(np.int16)
    return a.view(np.int32)


def check_status(ws):
    st = qs.qs_device_status(ws)
    assert st == qs.QS_OK, qs.qs_status_string(st)
