"""Seeded synthetic workloads for the Q-Sparse top-K sparse projection path.

This module only *draws inputs* and names the workload shapes.  It holds none
of the method's arithmetic (no top-K, no masking, no quantizer, no matmul), so
both the CPU oracle (``oracle/``) and the CUDA path (``top_activation_sparse_b200``)
can be fed the very same bytes from here without sharing any code that
computes a result.

Shapes follow the 7B-class workloads the Q-Sparse and Turbo Sparse pages talk
about (Llama-7B FFN 4096 -> 11008, Mistral-7B FFN 4096 -> 14336).  K is
``floor(ratio * d)`` for the keep ratios those pages use (70% top-K for the
Q-Sparse FFN, 39% kept for the 1.58-bit model, top 10% of |h| for dReLU).

Values:
  * activations x ~ N(0, 1), drawn in float32 and then rounded once to the
    compute dtype (bf16 round-to-nearest-even) where the workload is bf16;
  * weights W ~ N(0, 1/fan_in), stored input-major as W^T [d_in, d_out];
  * the prefill workload scales floor(0.01 * d_in) channels (drawn without
    replacement from the seed) by 20 for every token, so that top-K has a
    fixed set of outlier channels to keep.

Random numbers come from numpy's PCG64 generator seeded with
``0x5EED0000 + workload index (+ 0x100 * batch)``; the same seed always gives
the same bytes on any machine.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

SEED_BASE = 0x5EED0000


def keep_count(ratio: float, d: int) -> int:
    """K for a keep ratio: floor(ratio * d), computed without float surprises."""
    # ratio is one of the pages' round percentages; use a decimal string so that
    # 0.7 * 4096 = 2867.2 floors to 2867 exactly.
    num, den = _as_fraction(ratio)
    return (num * d) // den


def _as_fraction(ratio: float) -> tuple[int, int]:
    s = repr(float(ratio))
    if "e" in s or "E" in s:
        raise ValueError(f"keep ratio {ratio!r} must be a plain decimal")
    whole, _, frac = s.partition(".")
    den = 10 ** len(frac)
    return int(whole) * den + int(frac or 0), den


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_f32(gen: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = gen.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 -> bfloat16 (nearest-even) and return the raw uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + lsb) >> 16
    nan = np.isnan(a)
    out = rounded.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array rounded to the workload dtype, returned as float32 values."""
    if dtype == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(to_bf16_bits(a))
    raise ValueError(dtype)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    kind: str                     # "linear" | "ffn" | "quant" | "quant_ffn" | "prefill"
    dtype: str                    # "f32" | "bf16"
    d_in: int
    d_out: int
    k: int                        # top-K on the projection input
    batches: tuple
    act: str | None = None        # "relu2_glu" | "drelu" for ffn workloads
    k_h: int | None = None        # top-K on |h| before the down projection
    bias: float | None = None     # dReLU pre-activation bias
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0

    def seed(self, batch: int = 0, salt: int = 0) -> int:
        return SEED_BASE + self.index + 0x100 * batch + 0x10000 * salt


WORKLOADS = {
    # Single top-K sparse linear, fp32, 4 tokens, 512 -> 512, keep 50%.
    "linear_f32_512": Workload("linear_f32_512", 0, "linear", "f32", 512, 512,
                               keep_count(0.5, 512), (4,)),
    # Llama-7B FFN decode with squared-ReLU gating, 70% top-K on x and on |h|.
    "ffn_relu2_llama7b": Workload("ffn_relu2_llama7b", 1, "ffn", "bf16", 4096, 11008,
                                  keep_count(0.7, 4096), (1, 8), act="relu2_glu",
                                  k_h=keep_count(0.7, 11008)),
    # BitNet b1.58 + Q-Sparse projections, 39% kept, int8 x ternary.
    "quant_up_4096x11008": Workload("quant_up_4096x11008", 2, "quant", "bf16", 4096, 11008,
                                    keep_count(0.39, 4096), (1, 8, 32)),
    "quant_down_11008x4096": Workload("quant_down_11008x4096", 2, "quant", "bf16", 11008, 4096,
                                      keep_count(0.39, 11008), (1, 8, 32)),
    # Mistral-7B dReLU FFN decode: dense x, biased gate/up, top 10% of |h|.
    "ffn_drelu_mistral7b": Workload("ffn_drelu_mistral7b", 3, "ffn", "bf16", 4096, 14336,
                                    4096, (1, 4), act="drelu", k_h=keep_count(0.1, 14336),
                                    bias=-0.8),
    # BitNet b1.58 + Q-Sparse FFN layer (int8 x ternary up, gate, down), Llama-7B
    # shape, squared-ReLU gating, 39% kept at both projection inputs.
    "quant_ffn_llama7b": Workload("quant_ffn_llama7b", 5, "quant_ffn", "bf16", 4096, 11008,
                                  keep_count(0.39, 4096), (1, 8, 32), act="relu2_glu",
                                  k_h=keep_count(0.39, 11008)),
    # Prefill: 2048 tokens, 4096 -> 11008, 1% outlier channels x20, K = 2048.
    "prefill_bf16_2048": Workload("prefill_bf16_2048", 4, "prefill", "bf16", 4096, 11008,
                                  2048, (2048,), outlier_frac=0.01, outlier_scale=20.0),
}


def activations(w: Workload, T: int, salt: int = 0) -> np.ndarray:
    """x [T, d_in] as float32 values already rounded to the workload dtype."""
    g = rng(w.seed(T, salt))
    x = normal_f32(g, (T, w.d_in))
    if w.outlier_frac > 0.0:
        n_out = int(math.floor(w.outlier_frac * w.d_in))
        ch = g.choice(w.d_in, size=n_out, replace=False)
        x[:, ch] *= np.float32(w.outlier_scale)
    return round_to_dtype(x, w.dtype)


def outlier_channels(w: Workload, T: int, salt: int = 0) -> np.ndarray:
    """The channel ids :func:`activations` scaled (same draw order)."""
    g = rng(w.seed(T, salt))
    normal_f32(g, (T, w.d_in))
    n_out = int(math.floor(w.outlier_frac * w.d_in))
    return np.sort(g.choice(w.d_in, size=n_out, replace=False))


def weight_t(d_in: int, d_out: int, seed: int, dtype: str) -> np.ndarray:
    """W^T [d_in, d_out] with W ~ N(0, 1/d_in), rounded to dtype (float32 values)."""
    g = rng(seed)
    return round_to_dtype(normal_f32(g, (d_in, d_out), 1.0 / math.sqrt(d_in)), dtype)


def weight_out_major(d_out: int, d_in: int, seed: int) -> np.ndarray:
    """W [d_out, d_in] float32 with W ~ N(0, 1/d_in) (the ternary quantizer's input)."""
    g = rng(seed)
    return normal_f32(g, (d_out, d_in), 1.0 / math.sqrt(d_in))


def ffn_weights(w: Workload, layer: int = 0):
    """(W_up^T, W_gate^T, W_down^T) for an FFN workload; each ~ N(0, 1/fan_in)."""
    base = w.seed(0, 1 + 3 * layer)
    up = weight_t(w.d_in, w.d_out, base + 0x1000000, w.dtype)
    gate = weight_t(w.d_in, w.d_out, base + 0x2000000, w.dtype)
    down = weight_t(w.d_out, w.d_in, base + 0x3000000, w.dtype)
    return up, gate, down


def adversarial_rows(seed: int, T: int, d: int) -> np.ndarray:
    """Rows built to stress top-K tie handling: few distinct magnitudes, signed
    zeros, and whole rows of one value.  float32 values exactly representable
    in bf16."""
    g = rng(seed)
    palette = np.array([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 0.25, 3.0, -3.0],
                       dtype=np.float32)
    x = palette[g.integers(0, palette.size, size=(T, d))]
    if T >= 2:
        x[1, :] = np.float32(-1.5)            # one magnitude everywhere
    if T >= 3:
        x[2, :] = np.float32(0.0)             # all zeros (with -0.0 mixed in)
        x[2, ::3] = np.float32(-0.0)
    return x


def ffn_weights_device(w: Workload, layer: int, device, dtype=None):
    """(W_up^T, W_gate^T, W_down^T) drawn on the device with torch's seeded
    Philox generator: same distribution as :func:`ffn_weights` (N(0, 1/fan_in),
    rounded once to the workload dtype), much faster at 7B sizes.  Used by the
    benchmark, whose inputs do not need to match the numpy draws bit for bit."""
    import torch
    if dtype is None:
        dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    out = []
    for j, (d_in, d_out) in enumerate(((w.d_in, w.d_out), (w.d_in, w.d_out), (w.d_out, w.d_in))):
        g.manual_seed(w.seed(0, 1 + 3 * layer) + 0x1000000 * (j + 1))
        t = torch.randn(d_in, d_out, generator=g, device=device, dtype=torch.float32)
        t.mul_(1.0 / math.sqrt(d_in))
        out.append(t.to(dtype))
    return tuple(out)


def activations_device(w: Workload, T: int, device, salt: int = 0):
    """x [T, d_in] on the device from the numpy draw of :func:`activations`."""
    import torch
    x = torch.from_numpy(activations(w, T, salt))
    if w.dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x.to(device)
