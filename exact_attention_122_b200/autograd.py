"""torch.autograd binding: attention(q, k, v) whose backward runs fa_bwd.

The forward calls fa_fwd and keeps O and the per-row log-sum-exp; the
backward calls fa_bwd, which rebuilds P from Q, K and the LSE instead of
storing it (page "Flash attention optimization", section "Sizing a tile, and
why the backward pass recomputes instead of storing").  Argument marshalling
only: both passes run in libfa_b200.so.
"""

from __future__ import annotations

import math

import torch

from . import _binding


class _ExactAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal: bool, scale: float):
        # Views with a contiguous last dimension (e.g. BNHD transposed) go
        # through the strided entry points as they are; others are copied.
        q, k, v = (t if t.stride(-1) == 1 else t.contiguous() for t in (q, k, v))
        o, lse = _binding.fa_fwd(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal = causal
        ctx.scale = scale
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, do, _dlse):
        q, k, v, o, lse = ctx.saved_tensors
        do = do if do.stride(-1) == 1 else do.contiguous()
        dq, dk, dv = _binding.fa_bwd(q, k, v, o, lse, do, causal=ctx.causal, scale=ctx.scale)
        return dq, dk, dv, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None,
              return_lse: bool = False):
    """Exact attention softmax(scale q k^T [+ causal mask]) v for bf16 CUDA
    tensors (B, H, N, d), d in {64, 128}, differentiable in q, k and v.
    Returns O (and the fp32 LSE, not differentiable, if return_lse)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    o, lse = _ExactAttention.apply(q, k, v, bool(causal), float(scale))
    return (o, lse) if return_lse else o
