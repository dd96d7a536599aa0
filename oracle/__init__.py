"""CPU oracle for the Q-Sparse top-K sparse projection path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (cpu_baseline leg and
``--impl reference`` arm) may import this package.
"""
from .qs_oracle import (  # noqa: F401
    topk_keep, block_topk_keep, mask_from_keep, topk_mask, kept_values, sparse_linear, sparse_linear_backward_ste,
    relu, ffn_hidden,
    sparse_ffn, absmax_quantize, ternary_quantize, ternary_pack, ternary_unpack,
    quant_sparse_linear, ffn_hidden_f32, quant_sparse_ffn, max_rel_err,
)
