"""Test infrastructure: a slow, plainly correct CPU oracle for exact attention.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package. The product path (the CUDA library and
its Python binding) never imports it, and it imports nothing from them.

Every function computes in float64 and follows the definition of attention on
the page "Flash attention optimization" (aicomputerinstitute.com), section
"Attention is not slow because of arithmetic": S = QK^T * scale, P = row
softmax(S), O = P V; with max subtraction as in that page's "Worked example:
online softmax by hand".
"""

from .exact_attention import (  # noqa: F401
    bf16_bits_to_f64,
    e4m3_bits_to_f64,
    attention_fp64,
    attention_bwd_fp64,
    attention_bwd_rows_fp64,
    attention_rows_fp64,
    softmax_rows_fp64,
    online_softmax_row_blockmax,
    online_softmax_row_runningmax,
    tiled_attention_fp64,
)
