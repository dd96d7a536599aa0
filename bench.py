"""Benchmark: decode tokens/s and achieved HBM GB/s per sparse FFN layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch T]
                    [--workload NAME] [--impl ours|reference]

Default workload: the Llama-7B-shaped Q-Sparse FFN decode layer, bf16,
d_model 4096 -> d_ff 11008 -> 4096, top-K keeping floor(0.7 d) of |x| and of
|h|, h = ReLU(u)^2 * g, batch 1 token.  One step = one call of the whole layer
(top-K on x, up/gate gather-GEMV with the gating epilogue, top-K on |h|, down
gather-GEMV) on inputs already resident in HBM.  Steps rotate over several
independent layers whose weights together are far larger than the 126 MB L2,
so no step reads weights another step left in L2.

Several GPUs (launched with torch.distributed.run): every rank runs its own
replica of the layer on its own tokens (weak scaling, no data-path
collective); the timed region is bracketed by barriers and the slowest rank's
device time is reported.

--impl reference times the CPU oracle (oracle/, fp64) on this machine's host
cores on the same workload; it is the only other place this file runs it.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode tokens/s and achieved HBM GB/s (% of B200 peak) per sparse FFN layer"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30000)
    ap.add_argument("--warmup", type=int, default=300)
    ap.add_argument("--batch", type=int, default=0,
                    help="tokens per step per GPU (default: 1 for decode workloads, the "
                         "workload's own token count otherwise)")
    ap.add_argument("--workload", default="ffn_relu2_llama7b",
                    choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0,
                    help="independent layers to rotate over (0: enough to exceed 4x L2)")
    ap.add_argument("--gate-first", action="store_true",
                    help="dReLU FFN workloads: gate projection first, then W_up (output-major) "
                         "read only for open gates (qs_sparse_ffn_gate_first)")
    ap.add_argument("--block", type=int, default=1,
                    help="Block Q-Sparse: tokens sharing one top-K selection (1: per token)")
    ap.add_argument("--backward", action="store_true",
                    help="linear / prefill workloads: time the straight-through-estimator "
                         "backward (grad_x and grad_wt) instead of the forward")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0)
    a = ap.parse_args(argv)
    if a.batch <= 0:
        w = workloads.WORKLOADS[a.workload]
        a.batch = 1 if w.kind in ("ffn", "quant", "quant_ffn") else w.batches[0]
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.gate_first and workloads.WORKLOADS[a.workload].act != "drelu":
        ap.error("--gate-first needs a dReLU FFN workload")
    if a.backward and workloads.WORKLOADS[a.workload].kind not in ("linear", "prefill"):
        ap.error("--backward needs a linear or prefill workload")
    if not 1 <= a.block <= 64 or (a.block > 1 and a.gate_first):
        ap.error("--block must be 1..64 (and is not available with --gate-first)")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


# ---------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def dist_init(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device) -> float:
    """Slowest rank's number (all ranks get it)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist, device) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()
        time.sleep(0.25)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        return summarize_clocks(self.lines)


def summarize_clocks(lines: list[str]) -> dict:
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    sm, smax, reasons = [], [], set()
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
            "samples": len(sm)}


# ---------------------------------------------------------------- peaks / profiles

def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured",
                "bf16_tflops": float(d.get("bf16_tflops", 0) or 0)}
    return {"hbm_gbs": 6650.0, "source": "fallback", "bf16_tflops": 1590.0}


KERNEL_SOURCES = {"gemv": "gemv.cu", "prefill": "prefill_gemm.cu", "qgemv": "quant.cu",
                  "qgemvtc": "qgemv_tc.cu", "ffn": "ffn_fused.cu"}


def quant_tc(T: int, d_in: int, d_out: int, blk: int) -> bool:
    """Whether an int8 x ternary projection of T tokens runs on the tcgen05
    kind::i8 kernel (the library's own rule: 8..64 tokens, d_in % 16 == 0,
    d_out % 64 == 0, per-token selections)."""
    return blk <= 1 and 8 <= T <= 64 and d_in % 16 == 0 and d_out % 64 == 0


def _code_only(text: str) -> str:
    """C/C++ source without comments and blank-line noise: a comment edit does
    not change the compiled kernel, so it must not void a profile."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":                       # string / char literal
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (re.sub(r"[ \t]+", " ", line).strip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_digest(profile: str) -> str:
    """Digest of the dominant kernel's code (its .cu and the shared header,
    comments stripped)."""
    import hashlib
    h = hashlib.sha256()
    main = KERNEL_SOURCES[profile.split("_")[0]]
    for name in (main, "qs_internal.cuh"):
        with open(os.path.join(ROOT, "top_activation_sparse_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def profiled_traffic(profile: str) -> float | None:
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary profiles/<profile>.md, if it was taken on the current kernel
    source; else None."""
    p = os.path.join(ROOT, "profiles", f"{profile}.md")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for ln in f:
            if ln.startswith("- ") and ":" in ln:
                k, v = ln[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_digest") != kernel_source_digest(profile):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- our arm

def _mk_events(torch, stream, n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record(stream)              # torch creates the CUDA event on its first record
    return evs, (ctypes.c_void_p * n)(*[e.cuda_event for e in evs])


def workload_desc(args, T: int) -> str:
    """The workload's description, identical in both arms' `config`."""
    blk = getattr(args, "block", 1)
    if blk > 1:
        return _workload_desc(args, T) + f", Block Q-Sparse blocks of {blk} tokens"
    return _workload_desc(args, T)


def _workload_desc(args, T: int) -> str:
    w = workloads.WORKLOADS[args.workload]
    if w.kind == "ffn":
        gf = (", gate first (W_up output-major, rows of open gates only)"
              if getattr(args, "gate_first", False) else "")
        return (f"{args.workload}: sparse FFN decode layer, d_model={w.d_in}, d_ff={w.d_out}, "
                f"act={w.act}, K_x={w.k}, K_h={w.k_h}, bf16{gf}")
    if w.kind == "quant":
        return (f"{args.workload}: int8 x ternary sparse projection, T={T}, {w.d_in}->{w.d_out}, "
                f"K={w.k}, packed 2-bit weights")
    if w.kind == "quant_ffn":
        return (f"{args.workload}: int8 x ternary sparse FFN layer, d_model={w.d_in}, d_ff={w.d_out}, "
                f"act={w.act}, K_x={w.k}, K_h={w.k_h}, packed 2-bit weights")
    if getattr(args, "backward", False):
        return (f"{args.workload}: straight-through-estimator backward of the sparse linear "
                f"(grad_x = dY.W, grad_wt += X_sparse^T.dY), T={T}, {w.d_in}->{w.d_out}, K={w.k}, "
                f"{w.dtype}")
    return f"{args.workload}: sparse linear, T={T}, {w.d_in}->{w.d_out}, K={w.k}, {w.dtype}"


def run_config(desc: str, T: int, world: int, layers: int, l2: str, parallelism: str) -> dict:
    """The `config` object; both arms emit the same keys."""
    return {"workload": desc, "batch_per_gpu": T, "global_batch": T * world,
            "layers_rotated": layers, "l2": l2, "parallelism": parallelism}


def setup_ffn(args, qs, torch, device, stream, rank):
    """One sparse FFN layer per step, rotating over independent layers."""
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    d_model, d_ff, k_in, k_h = w.d_in, w.d_out, w.k, w.k_h
    act = qs.QS_ACT_RELU2_GLU if w.act == "relu2_glu" else qs.QS_ACT_DRELU
    layer_bytes = 3 * d_model * d_ff * 2
    n_layers = args.layers or max(2, math.ceil(4 * L2_BYTES / layer_bytes))
    layers = [workloads.ffn_weights_device(w, l, device) for l in range(n_layers)]
    gate_first = bool(getattr(args, "gate_first", False))
    if gate_first:                    # W_up output-major: [d_ff, d_model]
        layers = [(up.t().contiguous(), gate, down) for up, gate, down in layers]
    op = qs.QS_OP_SPARSE_FFN_GATE_FIRST if gate_first else qs.QS_OP_SPARSE_FFN
    blk = args.block
    bias = None
    if w.bias is not None:
        bias = torch.full((d_ff,), float(w.bias), dtype=torch.float32, device=device)
    x = workloads.activations_device(w, T, device, salt=rank)
    y = torch.empty(T, d_model, dtype=torch.bfloat16, device=device)
    ws = qs.new_workspace(op, T, d_model, d_ff, k_h, device)
    sp = stream.cuda_stream
    bptr = bias.data_ptr() if bias is not None else None
    fn = (qs.lib().qs_sparse_ffn_gate_first if gate_first else
          qs.lib().qs_block_sparse_ffn if blk > 1 else qs.lib().qs_sparse_ffn)

    def c_args(l, ev, kx=k_in, kh=k_h):
        up, gate, down = layers[l]
        if gate_first:                # x is dense on this path (kx = d_model)
            return (x.data_ptr(), qs.QS_BF16, T, d_model, d_ff, kh, gate.data_ptr(),
                    up.data_ptr(), bptr, bptr, down.data_ptr(), y.data_ptr(), None, None, ev,
                    ws.data_ptr(), ws.numel(), sp)
        if blk > 1:
            return (x.data_ptr(), qs.QS_BF16, T, d_model, d_ff, act, kx, kh, blk, up.data_ptr(),
                    gate.data_ptr(), bptr, bptr, down.data_ptr(), y.data_ptr(), None, None, ev,
                    ws.data_ptr(), ws.numel(), sp)
        return (x.data_ptr(), qs.QS_BF16, T, d_model, d_ff, act, kx, kh, up.data_ptr(),
                gate.data_ptr(), bptr, bptr, down.data_ptr(), y.data_ptr(), None, None, ev,
                ws.data_ptr(), ws.numel(), sp)

    rows = []
    for l in range(n_layers):
        st = fn(*c_args(l, None))
        assert st == 0, qs.qs_status_string(st)
        rows.append(qs.qs_workspace_stats(ws, op, T, d_model, d_ff, k_h))
    assert qs.qs_device_status(ws) == qs.QS_OK
    rows_x = float(np.mean([r[0] for r in rows]))
    rows_h = float(np.mean([r[1] for r in rows]))
    if gate_first:
        # the gate kernel streams the kept rows of W_gate^T (one matrix) and
        # writes ReLU(g + b) (f32); the up kernel streams the open rows of W_up
        # and reads and rewrites those h entries
        rows_up = float(np.mean([r[2] for r in rows]))
        upgate_bytes = (rows_x * d_ff * 2 + rows_x * (4 + 4 * T) + T * d_ff * 4
                        + rows_up * d_model * 2 + T * d_model * 2 + rows_up * T * 8)
        extra_rows = {"x": rows_x, "h": rows_h, "up_open_gates": rows_up}
    else:
        # algorithmic bytes of the up/gate kernel per launch: the kept rows of
        # W_up^T and W_gate^T, the staged (index, T values) entries, h written (f32)
        upgate_bytes = rows_x * d_ff * 2 * 2 + rows_x * (4 + 4 * T) + T * d_ff * 4
        extra_rows = {"x": rows_x, "h": rows_h}
    down_bytes = rows_h * d_model * 2 + rows_h * (4 + 4 * T) + T * d_model * 2
    topk_bytes = T * d_model * 2 + T * d_ff * 4
    lw = layers

    def e2e_call(i, x_dev, y_dev):
        up, gate, down = lw[i % n_layers]
        if gate_first:
            qs.qs_sparse_ffn_gate_first(x_dev, gate, up, down, k_h, b_up=bias, b_gate=bias,
                                        y=y_dev, ws=ws)
        else:
            qs.qs_sparse_ffn(x_dev, up, gate, down, w.act, k_in, k_h, b_up=bias, b_gate=bias,
                             y=y_dev, ws=ws, block=blk)

    def cpu_rate():
        up, gate, down = (t.float().cpu().numpy() for t in layers[0])
        if gate_first:
            up = np.ascontiguousarray(up.T)
        return cpu_oracle_ffn(w, x.float().cpu().numpy(), up, gate, down, args.cpu_seconds, blk)

    phases = ["topk_x", "upgate", "topk_h", "down"]
    dominant, dom_work, launches = "upgate", upgate_bytes, 5 if gate_first else 4
    kernel = ("gemv_kernel (gate gather-GEMV) + up_rows_kernel (open gates' rows of W_up)"
              if gate_first else "gemv_kernel (up/gate gather-GEMV with the gating epilogue)")
    profile = f"gemv_{'gatefirst' if gate_first else 'upgate'}_{args.workload}_T{T}"
    fused = (not gate_first and blk <= 1 and
             qs.qs_sparse_ffn_fused(qs.QS_BF16, T, d_model, d_ff, False))
    if fused:
        # one persistent kernel per layer: it is the dominant (and only) kernel
        phases, dominant = ["ffn_fused"], "ffn_fused"
        dom_work, launches = upgate_bytes + down_bytes + topk_bytes, 1
        kernel = "ffn_fused_kernel (the whole one-token layer, one launch)"
        profile = f"ffn_fused_{args.workload}_T{T}"
    return {
        "fn": fn, "T": T, "n_layers": n_layers, "ws": ws, "x": x, "y": y,
        "args": lambda l, ev: c_args(l, ev), "n_events": qs.QS_FFN_PHASE_EVENTS,
        "dense_args": (lambda l: c_args(l, None, d_model, d_ff)),
        "dense_note": ("gate-first path with K_h = d_ff: W_up is still read only for open gates"
                       if gate_first else None),
        "phases": phases, "dominant": dominant,
        "kernel": kernel,
        "bound": "hbm", "dom_work": dom_work, "layer_work": upgate_bytes + down_bytes + topk_bytes,
        "extra": {"rows_streamed": extra_rows},
        "desc": workload_desc(args, T),
        "l2": (f"inputs larger than L2: {n_layers} independent layers "
               f"({n_layers * layer_bytes / 1e9:.2f} GB of weights) rotated per step"),
        "e2e_call": e2e_call, "cpu_rate": cpu_rate, "launches": launches,
        "dtype": "bf16",
        "profile": profile,
        "single_kernel": fused,
    }


def setup_linear(args, qs, torch, device, stream, rank):
    """One sparse projection per step (prefill GEMM for >= 64 bf16 tokens)."""
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    eb = 2 if w.dtype == "bf16" else 4
    wbytes = w.d_in * w.d_out * eb
    n_layers = args.layers or max(2, math.ceil(2 * L2_BYTES / wbytes))
    g = torch.Generator(device=device)
    wts = []
    for l in range(n_layers):
        g.manual_seed(w.seed(0, 1 + l))
        t = torch.randn(w.d_in, w.d_out, generator=g, device=device) * (w.d_in ** -0.5)
        wts.append(t.to(tdt))
    x = workloads.activations_device(w, T, device, salt=rank)
    y = torch.empty(T, w.d_out, dtype=tdt, device=device)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k, device)
    sp = stream.cuda_stream
    blk = args.block
    fn = qs.lib().qs_block_sparse_linear if blk > 1 else qs.lib().qs_sparse_linear
    dt = qs.QS_BF16 if w.dtype == "bf16" else qs.QS_F32

    def c_args(l, ev, k=w.k):
        if blk > 1:
            return (x.data_ptr(), dt, T, w.d_in, w.d_out, k, blk, wts[l].data_ptr(), y.data_ptr(),
                    ev, ws.data_ptr(), ws.numel(), sp)
        return (x.data_ptr(), dt, T, w.d_in, w.d_out, k, wts[l].data_ptr(), y.data_ptr(), ev,
                ws.data_ptr(), ws.numel(), sp)

    for l in range(n_layers):             # every layer once: validation, steady state
        assert fn(*c_args(l, None)) == 0
    assert qs.qs_device_status(ws) == qs.QS_OK
    prefill = (w.dtype == "bf16" and T >= qs.QS_PREFILL_MIN_T)
    if prefill:
        # tensor-core bound: algorithmic FLOPs (kept inputs only) per launch
        work = 2.0 * T * w.k * w.d_out
        extra = {"executed_flops": 2.0 * T * w.d_in * w.d_out}
        bound, kernel = "tensor", "prefill_gemm_kernel (tcgen05 masked-dense GEMM)"
    else:
        rows, _ = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k)
        work = rows * w.d_out * eb + rows * (4 + 4 * T) + T * w.d_out * eb
        extra = {"rows_streamed": rows}
        bound, kernel = "hbm", "gemv_kernel (gather-GEMV)"

    def e2e_call(i, x_dev, y_dev):
        qs.qs_sparse_linear(x_dev, wts[i % n_layers], w.k, y=y_dev, ws=ws, block=blk)

    def cpu_rate():
        import oracle
        xs = x.float().cpu().numpy()
        wt0 = wts[0].float().cpu().numpy()
        rows_n = min(T, 8)
        t0 = time.perf_counter()
        n = 0
        while n < 2 or time.perf_counter() - t0 < args.cpu_seconds:
            oracle.sparse_linear(xs[:rows_n], wt0, w.k,
                                 keep=oracle.block_topk_keep(xs[:rows_n], w.k, blk))
            n += 1
        dt_ = time.perf_counter() - t0
        return {"value": round(n * rows_n / dt_, 3), "unit": UNIT, "cores": _threads_in_use(),
                "kind": "oracle", "sample": f"{n} oracle calls of {rows_n} token(s), {dt_:.1f} s"}

    return {
        "fn": fn, "T": T, "n_layers": n_layers, "ws": ws, "x": x, "y": y,
        "args": c_args, "n_events": qs.QS_LINEAR_PHASE_EVENTS,
        "dense_args": (lambda l: c_args(l, None, w.d_in)),
        "phases": ["topk", "projection"], "dominant": "projection", "kernel": kernel,
        "bound": bound, "dom_work": work, "layer_work": work, "extra": extra,
        "desc": workload_desc(args, T),
        "l2": f"inputs larger than L2: {n_layers} weight copies ({n_layers * wbytes / 1e9:.2f} GB) rotated",
        "e2e_call": e2e_call, "cpu_rate": cpu_rate, "launches": 2, "dtype": w.dtype,
        "profile": f"{'prefill_gemm' if prefill else 'gemv'}_{args.workload}_T{T}",
    }


def setup_backward(args, qs, torch, device, stream, rank):
    """One straight-through-estimator backward of a sparse projection per step:
    grad_x = dY . W (every weight row) and grad_wt += X_sparse^T . dY."""
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    eb = 2 if w.dtype == "bf16" else 4
    per_layer = w.d_in * w.d_out * (eb + 4)          # weights and their f32 gradient
    n_layers = args.layers or max(2, math.ceil(2 * L2_BYTES / per_layer))
    g = torch.Generator(device=device)
    wts, gwts = [], []
    for l in range(n_layers):
        g.manual_seed(w.seed(0, 1 + l))
        wts.append((torch.randn(w.d_in, w.d_out, generator=g, device=device) * (w.d_in ** -0.5)).to(tdt))
        gwts.append(torch.zeros(w.d_in, w.d_out, dtype=torch.float32, device=device))
    x = workloads.activations_device(w, T, device, salt=rank)
    g.manual_seed(w.seed(T, 7))
    gy = (torch.randn(T, w.d_out, generator=g, device=device) * 0.01).to(tdt)
    gx = torch.empty(T, w.d_in, dtype=torch.float32, device=device)
    ws = qs.new_workspace(qs.QS_OP_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k, device)
    sp = stream.cuda_stream
    blk = args.block
    fn = qs.lib().qs_sparse_linear_backward
    dt = qs.QS_BF16 if w.dtype == "bf16" else qs.QS_F32

    def c_args(l, ev, k=w.k):
        return (x.data_ptr(), dt, T, w.d_in, w.d_out, k, blk, wts[l].data_ptr(), gy.data_ptr(),
                gx.data_ptr(), gwts[l].data_ptr(), ws.data_ptr(), ws.numel(), sp)

    for l in range(n_layers):             # every layer once: validation, steady state
        assert fn(*c_args(l, None)) == 0
    assert qs.qs_device_status(ws) == qs.QS_OK
    tensor = w.dtype == "bf16" and T >= qs.QS_PREFILL_MIN_T
    if tensor:
        # algorithmic FLOPs: grad_x is dense (the estimator applies no mask),
        # grad_wt counts the T*K kept entries only
        work = 2.0 * T * w.d_in * w.d_out + 2.0 * T * w.k * w.d_out
        extra = {"executed_flops": 4.0 * T * w.d_in * w.d_out}
        bound, kernel = "tensor", "umma_gemm_kernel (tcgen05 grad_x and grad_wt GEMMs)"
    else:
        # rows of grad_wt read and written: the inputs some token kept (the
        # library's own count for the last chunk of tokens)
        rows_kept, _ = qs.qs_workspace_stats(ws, qs.QS_OP_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k)
        # algorithmic bytes: every row of W^T read once per 8 tokens, the kept
        # rows of grad_wt read and written, dY read, grad_x written
        groups = (T + 7) // 8
        work = (groups * w.d_in * w.d_out * eb + rows_kept * w.d_out * 8 + T * w.d_out * eb
                + T * w.d_in * 4)
        extra = {"rows_kept": rows_kept}
        bound, kernel = "hbm", "rowdot_kernel (grad_x) + rowaxpy_kernel (kept rows of grad_wt)"

    def e2e_call(i, x_dev, y_dev):
        qs.qs_sparse_linear_backward(x_dev, wts[i % n_layers], gy, w.k, grad_x=y_dev,
                                     grad_wt=gwts[i % n_layers], ws=ws, block=blk)

    def cpu_rate():
        import oracle
        xs = x.float().cpu().numpy()
        wt0 = wts[0].float().cpu().numpy()
        gy0 = gy.float().cpu().numpy()
        rows_n = min(T, 8)
        t0 = time.perf_counter()
        n = 0
        while n < 2 or time.perf_counter() - t0 < args.cpu_seconds:
            oracle.sparse_linear_backward_ste(xs[:rows_n], wt0, w.k, gy0[:rows_n],
                                              keep=oracle.block_topk_keep(xs[:rows_n], w.k, blk))
            n += 1
        dt_ = time.perf_counter() - t0
        return {"value": round(n * rows_n / dt_, 3), "unit": UNIT, "cores": _threads_in_use(),
                "kind": "oracle", "sample": f"{n} oracle backward calls of {rows_n} token(s), {dt_:.1f} s"}

    return {
        "fn": fn, "T": T, "n_layers": n_layers, "ws": ws, "x": x, "y": gx,
        "args": c_args, "n_events": 0, "dense_args": None,
        "phases": [], "dominant": None, "kernel": kernel,
        "bound": bound, "dom_work": work, "layer_work": work, "extra": extra,
        "desc": workload_desc(args, T),
        "l2": f"inputs larger than L2: {n_layers} weight + gradient copies "
              f"({n_layers * per_layer / 1e9:.2f} GB) rotated",
        "e2e_call": e2e_call, "cpu_rate": cpu_rate, "e2e_inputs": [gy],
        "launches": (3 if tensor else (1 + 2 * ((T + 63) // 64) + 2)), "dtype": w.dtype,
        "profile": f"backward_{args.workload}_T{T}",
    }


def setup_quant_ffn(args, qs, torch, device, stream, rank):
    """One BitNet b1.58 + Q-Sparse FFN layer per step (int8 x packed ternary up,
    gate and down, each input quantized and top-K'd)."""
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    dm, dff = w.d_in, w.d_out
    layer_bytes = 3 * dm * dff // 4
    n_layers = args.layers or max(2, math.ceil(2 * L2_BYTES / layer_bytes))
    g = torch.Generator(device=device)
    layers = []
    wsp = qs.new_workspace(qs.QS_OP_TERNARY_PACK, 0, max(dm, dff), max(dm, dff), 0, device)
    for l in range(n_layers):
        mats = []
        for j, (o, i) in enumerate(((dff, dm), (dff, dm), (dm, dff))):
            g.manual_seed(w.seed(0, 1 + 3 * l + j))
            wf = torch.randn(o, i, generator=g, device=device) * (i ** -0.5)
            p, a = qs.qs_ternary_pack(wf, 1e-5, ws=wsp)
            mats.append((p, float(a.item())))
            del wf
        layers.append(mats)
    x = workloads.activations_device(w, T, device, salt=rank)
    y = torch.empty(T, dm, dtype=torch.float32, device=device)
    ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_FFN, T, dm, dff, w.k_h, device)
    sp = stream.cuda_stream
    blk = args.block
    act = qs.QS_ACT_RELU2_GLU if w.act == "relu2_glu" else qs.QS_ACT_DRELU
    fn = qs.lib().qs_quant_sparse_ffn
    f = ctypes.c_float

    def c_args(l, ev, kx=w.k, kh=w.k_h):
        (pu, au), (pg, ag), (pd, ad) = layers[l]
        return (x.data_ptr(), qs.QS_BF16, T, dm, dff, act, kx, kh, blk, pu.data_ptr(), f(au),
                pg.data_ptr(), f(ag), pd.data_ptr(), f(ad), f(1e-5), None, None, y.data_ptr(),
                None, ev, ws.data_ptr(), ws.numel(), sp)

    rows = []
    for l in range(n_layers):
        assert fn(*c_args(l, None)) == 0
        rows.append(qs.qs_workspace_stats(ws, qs.QS_OP_QUANT_SPARSE_FFN, T, dm, dff, w.k_h))
    assert qs.qs_device_status(ws) == qs.QS_OK
    rows_x = float(np.mean([r[0] for r in rows]))
    rows_h = float(np.mean([r[1] for r in rows]))
    # algorithmic bytes: packed rows of up and gate (kept x), of down (kept h),
    # the staged (index, code) entries, u and h written and read (f32)
    upgate = 2 * rows_x * dff // 4 + rows_x * (4 + T) + 3 * T * dff * 4
    down = rows_h * dm // 4 + rows_h * (4 + T) + T * dm * 4
    topk = T * dm * 2 + T * dff * 4

    def e2e_call(i, x_dev, y_dev):
        (pu, au), (pg, ag), (pd, ad) = layers[i % n_layers]
        qs.qs_quant_sparse_ffn(x_dev, pu, au, pg, ag, pd, ad, w.act, w.k, w.k_h, y=y_dev, ws=ws,
                               block=blk)

    def cpu_rate():
        import oracle
        (pu, au), (pg, ag), (pd, ad) = layers[0]
        ts = [oracle.ternary_unpack(p.cpu().numpy().view(np.uint32), d)
              for p, d in ((pu, dff), (pg, dff), (pd, dm))]
        xs = x.float().cpu().numpy()
        rows_n = min(T, 8)
        t0 = time.perf_counter()
        n = 0
        while n < 2 or time.perf_counter() - t0 < args.cpu_seconds:
            oracle.quant_sparse_ffn(xs[:rows_n], ts[0], au, ts[1], ag, ts[2], ad, w.act, w.k, w.k_h,
                                    block=blk)
            n += 1
        dt_ = time.perf_counter() - t0
        return {"value": round(n * rows_n / dt_, 3), "unit": UNIT, "cores": _threads_in_use(),
                "kind": "oracle", "sample": f"{n} whole-layer oracle calls of {rows_n} token(s), {dt_:.1f} s"}

    return {
        "fn": fn, "T": T, "n_layers": n_layers, "ws": ws, "x": x, "y": y,
        "args": lambda l, ev: c_args(l, ev), "n_events": qs.QS_FFN_PHASE_EVENTS,
        "dense_args": (lambda l: c_args(l, None, dm, dff)),
        "phases": ["quant_topk_x", "upgate", "quant_topk_h", "down"], "dominant": "upgate",
        "kernel": ("qgemv_tc_kernel (int8 x ternary up, then gate with the gating epilogue; "
                   "tcgen05 kind::i8)" if quant_tc(T, dm, dff, blk) else
                   "qgemv (int8 x ternary up, then gate with the gating epilogue)"),
        "bound": "hbm", "dom_work": upgate, "layer_work": upgate + down + topk,
        "extra": {"rows_streamed": {"x": rows_x, "h": rows_h}},
        "desc": workload_desc(args, T),
        "l2": (f"inputs larger than L2: {n_layers} independent packed layers "
               f"({n_layers * layer_bytes / 1e9:.2f} GB) rotated per step"),
        "e2e_call": e2e_call, "cpu_rate": cpu_rate, "launches": 5, "dtype": "int8",
        "profile": (f"qgemvtc_{args.workload}_T{T}" if quant_tc(T, dm, dff, blk)
                    else f"qgemv_{args.workload}_T{T}"),
    }


def setup_quant(args, qs, torch, device, stream, rank):
    """BitNet b1.58 + Q-Sparse projection per step (int8 x packed ternary)."""
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    n_words = w.d_out // 16
    wbytes = w.d_in * n_words * 4
    n_layers = args.layers or max(2, math.ceil(2 * L2_BYTES / wbytes))
    g = torch.Generator(device=device)
    packs, alphas = [], []
    wsp = qs.new_workspace(qs.QS_OP_TERNARY_PACK, 0, w.d_in, w.d_out, 0, device)
    for l in range(n_layers):
        g.manual_seed(w.seed(0, 1 + l))
        wf = torch.randn(w.d_out, w.d_in, generator=g, device=device) * (w.d_in ** -0.5)
        p, a = qs.qs_ternary_pack(wf, 1e-5, ws=wsp)
        packs.append(p)
        alphas.append(float(a.item()))
        del wf
    x = workloads.activations_device(w, T, device, salt=rank)
    y = torch.empty(T, w.d_out, dtype=torch.float32, device=device)
    ws = qs.new_workspace(qs.QS_OP_QUANT_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k, device)
    sp = stream.cuda_stream
    blk = args.block
    fn = qs.lib().qs_block_quant_sparse_linear if blk > 1 else qs.lib().qs_quant_sparse_linear

    def c_args(l, ev, k=w.k):
        if blk > 1:
            return (x.data_ptr(), qs.QS_BF16, T, w.d_in, w.d_out, k, blk, packs[l].data_ptr(),
                    ctypes.c_float(alphas[l]), ctypes.c_float(1e-5), y.data_ptr(), None, None,
                    None, ev, ws.data_ptr(), ws.numel(), sp)
        return (x.data_ptr(), qs.QS_BF16, T, w.d_in, w.d_out, k, packs[l].data_ptr(),
                ctypes.c_float(alphas[l]), ctypes.c_float(1e-5), y.data_ptr(), None, None, None, ev,
                ws.data_ptr(), ws.numel(), sp)

    for l in range(n_layers):             # every layer once: validation, steady state
        assert fn(*c_args(l, None)) == 0
    assert qs.qs_device_status(ws) == qs.QS_OK
    rows, _ = qs.qs_workspace_stats(ws, qs.QS_OP_QUANT_SPARSE_LINEAR, T, w.d_in, w.d_out, w.k)
    work = rows * n_words * 4 + rows * (4 + T) + T * w.d_out * 4

    def e2e_call(i, x_dev, y_dev):
        qs.qs_quant_sparse_linear(x_dev, packs[i % n_layers], alphas[i % n_layers], w.k, y=y_dev,
                                  ws=ws, block=blk)

    def cpu_rate():
        import oracle
        xs = x.float().cpu().numpy()
        t = oracle.ternary_unpack(packs[0].cpu().numpy().view(np.uint32), w.d_out)
        rows_n = min(T, 8)
        t0 = time.perf_counter()
        n = 0
        while n < 2 or time.perf_counter() - t0 < args.cpu_seconds:
            q_, _ = oracle.absmax_quantize(xs[:rows_n])
            oracle.quant_sparse_linear(xs[:rows_n], t, alphas[0], w.k,
                                       keep=oracle.block_topk_keep(q_, w.k, blk))
            n += 1
        dt_ = time.perf_counter() - t0
        return {"value": round(n * rows_n / dt_, 3), "unit": UNIT, "cores": _threads_in_use(),
                "kind": "oracle", "sample": f"{n} oracle calls of {rows_n} token(s), {dt_:.1f} s"}

    return {
        "fn": fn, "T": T, "n_layers": n_layers, "ws": ws, "x": x, "y": y,
        "args": c_args, "n_events": qs.QS_LINEAR_PHASE_EVENTS,
        "dense_args": (lambda l: c_args(l, None, w.d_in)),
        "phases": ["quant_topk", "projection"], "dominant": "projection",
        "kernel": ("qgemv_tc_kernel (int8 x ternary, tcgen05 kind::i8, TMEM accumulators)"
                   if quant_tc(T, w.d_in, w.d_out, blk) else "qgemv_kernel (int8 x ternary gather)"),
        "bound": "hbm", "dom_work": work,
        "layer_work": work, "extra": {"rows_streamed": rows},
        "desc": workload_desc(args, T),
        "l2": f"inputs larger than L2: {n_layers} packed weight copies ({n_layers * wbytes / 1e9:.2f} GB) rotated",
        "e2e_call": e2e_call, "cpu_rate": cpu_rate, "launches": 2, "dtype": "int8",
        "profile": (f"qgemvtc_{args.workload}_T{T}" if quant_tc(T, w.d_in, w.d_out, blk)
                    else f"qgemv_{args.workload}_T{T}"),
    }


def run_ours(args, rank, world, local):
    import torch
    import top_activation_sparse_b200 as qs
    from top_activation_sparse_b200 import build as qs_build

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world, "nccl")
    if rank == 0 or dist is None:
        qs_build.build()
    if dist is not None:
        dist.barrier()
    qs.lib()
    stream = torch.cuda.current_stream(device)
    kind = workloads.WORKLOADS[args.workload].kind
    setup = {"ffn": setup_ffn, "linear": setup_linear, "prefill": setup_linear,
             "quant": setup_quant, "quant_ffn": setup_quant_ffn}[kind]
    if args.backward:
        setup = setup_backward
    c = setup(args, qs, torch, device, stream, rank)
    fn, T, n_layers = c["fn"], c["T"], c["n_layers"]

    def run(a):
        st = fn(*a)
        if st != 0:
            raise RuntimeError(f"{fn.__name__}: {qs.qs_status_string(st)}")

    plain = [c["args"](l, None) for l in range(n_layers)]
    # every rotated layer was called once during setup (validation, row counts),
    # so the warm-up steps start from a steady state
    for i in range(args.warmup):
        run(plain[i % n_layers])
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):           # the timed region: plain calls only
        run(plain[i % n_layers])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    assert qs.qs_device_status(c["ws"]) == qs.QS_OK
    ms_max = max_over_ranks(ms, dist, device)
    tokens = sum_over_ranks(float(T * args.steps), dist, device)
    value = tokens / (ms_max / 1e3)

    # per-phase device time: a separate sampled pass after the timed region,
    # with CUDA events between the kernels of each step (they cost the launch
    # overlap, so they never run inside the timed region)
    names = c["phases"]
    if c["n_events"] > 0:
        n_phase = 256
        evs = [_mk_events(torch, stream, c["n_events"]) for _ in range(n_phase)]
        torch.cuda.synchronize()
        for i in range(n_phase):
            run(c["args"](i % n_layers, evs[i][1]))
        torch.cuda.synchronize()
        ph = np.array([[e[0][p].elapsed_time(e[0][p + 1]) for p in range(len(names))] for e in evs])
        ph_us = {n: round(float(v), 3) for n, v in zip(names, ph.mean(axis=0) * 1e3)}
        dom_us = ph_us[c["dominant"]]
    else:                                 # one call is the dominant unit: the whole step
        ph_us = {}
        dom_us = ms / args.steps * 1e3
    dom_from = "timed region / steps" if c["n_events"] == 0 else "per-phase event pass"
    if c.get("single_kernel"):
        # the timed region holds this kernel's launches and nothing else, so its
        # average launch duration in the stream is the region's time per step;
        # the event pass above times each launch alone (events between launches
        # remove the overlap of one launch's start with the previous one's end)
        dom_us = ms / args.steps * 1e3
        dom_from = "timed region / steps (every step is one launch of this kernel)"
    peaks = load_peaks()
    if c["bound"] == "hbm":
        achieved = c["dom_work"] / (dom_us * 1e-6) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        achieved = c["dom_work"] / (dom_us * 1e-6) / 1e12
        peak, unit = peaks["bf16_tflops"], "TFLOP/s"
    step_s = ms / 1e3 / args.steps

    # dense run of the same kernels (K = d): context for the sparsity win
    dense = None
    if c.get("dense_args") is not None:
        dargs = [c["dense_args"](l) for l in range(n_layers)]
        for i in range(args.warmup):
            run(dargs[i % n_layers])
        n_dense = max(1, min(args.steps, 2000))
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for i in range(n_dense):
            run(dargs[i % n_layers])
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms = d0.elapsed_time(d1) / n_dense
        dense = {"ms_per_step": round(dense_ms, 6), "value": round(T / (dense_ms / 1e3), 1)}
        if c.get("dense_note"):
            dense["note"] = c["dense_note"]

    # end to end through the public Python API, host buffers in and out
    x, y = c["x"], c["y"]
    x_host = x.cpu().pin_memory()
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    x_dev = torch.empty_like(x)
    # other per-step inputs (the backward's dY) are copied in from host too
    extra_in = [(t, t.cpu().pin_memory()) for t in c.get("e2e_inputs", [])]
    n_e2e = max(1, min(args.steps, 5000))
    for i in range(args.warmup):
        x_dev.copy_(x_host, non_blocking=True)
        for t_dev, t_host in extra_in:
            t_dev.copy_(t_host, non_blocking=True)
        c["e2e_call"](i, x_dev, y)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_e2e):
        x_dev.copy_(x_host, non_blocking=True)
        for t_dev, t_host in extra_in:
            t_dev.copy_(t_host, non_blocking=True)
        c["e2e_call"](i, x_dev, y)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    e_tokens = sum_over_ranks(float(T * n_e2e), dist, device)
    e2e_value = e_tokens / (e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = c["cpu_rate"]()

    chunks = (T + qs.QS_PREFILL_MIN_T - 1) // qs.QS_PREFILL_MIN_T
    if (c["launches"] == 2 and T >= qs.QS_PREFILL_MIN_T) or args.backward:
        chunks = 1
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": c["dtype"],
        "data": "synthetic: x ~ N(0,1), W ~ N(0,1/fan_in) (seeded; random-init weights)",
        "config": run_config(c["desc"], T, world, n_layers, c["l2"],
                             f"replicas x{world} (no data-path collective)"),
        "hbm": {
            "step_alg_gbs": round(c["layer_work"] / step_s / 1e9, 1) if c["bound"] == "hbm" else None,
            "frac_of_peak": (round(c["layer_work"] / step_s / 1e9 / peaks["hbm_gbs"], 4)
                             if c["bound"] == "hbm" else None),
            **c["extra"],
        },
        "phases_us": ph_us,
        "roofline": {
            "kernel": c["kernel"],
            "bound": c["bound"],
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_source": peaks["source"],
            "unit": unit,
            "frac": round(achieved / peak, 4),
            "traffic": profiled_traffic(c["profile"]),
            "alg_work_per_launch": int(c["dom_work"]),
            "duration_us": round(dom_us, 3),
            "duration_from": dom_from,
        },
        "dense_same_kernels": dense,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "steps": n_e2e,
                "h2d_bytes_per_step": int(x.numel() * x.element_size()
                                          + sum(t.numel() * t.element_size()
                                                for t, _ in extra_in)),
                "d2h_bytes_per_step": int(y.numel() * y.element_size())},
        "gpu_launches": c["launches"] * chunks * args.steps,
        "clocks": clk,
    }
    if cpu is not None:
        result["cpu_baseline"] = cpu
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result if rank == 0 else None


# ---------------------------------------------------------------- oracle arms

def _threads_in_use() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_oracle_ffn(w, x, up, gate, down, seconds: float, block: int = 1) -> dict:
    """Time the oracle as it stands on a bounded sample: whole-layer calls
    for about `seconds` of host time (at least two)."""
    import oracle
    T = x.shape[0]
    b = None if w.bias is None else np.full(w.d_out, w.bias)
    n = 0
    t0 = time.perf_counter()
    while n < 2 or time.perf_counter() - t0 < seconds:
        oracle.sparse_ffn(x, up, gate, down, w.act, w.k, w.k_h, b_up=b, b_gate=b, block=block)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(n * T / dt, 3), "unit": UNIT, "cores": _threads_in_use(),
            "kind": "oracle",
            "sample": f"{n} whole-layer oracle calls of {T} token(s) each, {dt:.1f} s, fp64 numpy"}


def run_reference(args, rank, world, local):
    """The oracle as the reference arm: rank 0 only, host cores only."""
    if rank != 0:
        return None
    import oracle
    w = workloads.WORKLOADS[args.workload]
    T = args.batch
    x = workloads.activations(w, T)
    if w.kind == "ffn":
        up, gate, down = workloads.ffn_weights(w)
        b = None if w.bias is None else np.full(w.d_out, w.bias)

        def step():
            oracle.sparse_ffn(x, up, gate, down, w.act, w.k, w.k_h, b_up=b, b_gate=b,
                              block=args.block)
    elif w.kind == "quant_ffn":
        tq = [oracle.ternary_quantize(workloads.weight_out_major(o, i, w.seed(0, 1 + j)))
              for j, (o, i) in enumerate(((w.d_out, w.d_in), (w.d_out, w.d_in), (w.d_in, w.d_out)))]

        def step():
            oracle.quant_sparse_ffn(x, tq[0][0], tq[0][1], tq[1][0], tq[1][1], tq[2][0], tq[2][1],
                                    w.act, w.k, w.k_h, block=args.block)
    elif w.kind == "quant":
        t, alpha = oracle.ternary_quantize(workloads.weight_out_major(w.d_out, w.d_in, w.seed(0, 1)))

        def step():
            q_, _ = oracle.absmax_quantize(x)
            oracle.quant_sparse_linear(x, t, alpha, w.k,
                                       keep=oracle.block_topk_keep(q_, w.k, args.block))
    elif args.backward:
        wt = workloads.weight_t(w.d_in, w.d_out, w.seed(0, 1), w.dtype)
        gy = workloads.round_to_dtype(
            workloads.normal_f32(workloads.rng(w.seed(T, 7)), (T, w.d_out), 0.01), w.dtype)

        def step():
            oracle.sparse_linear_backward_ste(x, wt, w.k, gy,
                                              keep=oracle.block_topk_keep(x, w.k, args.block))
    else:
        wt = workloads.weight_t(w.d_in, w.d_out, w.seed(0, 1), w.dtype)

        def step():
            oracle.sparse_linear(x, wt, w.k, keep=oracle.block_topk_keep(x, w.k, args.block))

    t0 = time.perf_counter()
    step()
    one = time.perf_counter() - t0
    budget = args.ref_seconds
    warm = max(0, min(args.warmup, int(0.2 * budget / max(one, 1e-9))))
    for _ in range(warm):
        step()
    n_run = max(1, min(args.steps, int(budget / max(one, 1e-9))))
    t0 = time.perf_counter()
    for _ in range(n_run):
        step()
    dt = time.perf_counter() - t0
    value = n_run * T / dt
    sample = (f"{n_run} of {args.steps} steps run (each the whole workload for {T} token(s)); "
              f"{warm} warm-up; fp64 numpy oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / n_run * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: x ~ N(0,1), W ~ N(0,1/fan_in) (seeded)",
        "config": run_config(workload_desc(args, T), T, 1, 1,
                             "not applicable: host memory (one layer's weights)",
                             "host cores (the fp64 oracle, rank 0)"),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": _threads_in_use(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        out = run_reference(args, rank, world, local)
    else:
        out = run_ours(args, rank, world, local)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
