"""Autograd wrapper: exact attention as a differentiable torch operation.

``attention(q, k, v, causal, scale)`` runs the library's forward kernel and,
when gradients are needed, its recomputing backward kernel ("Flash Attention
La Gi?" (thienlv.com), Recomputation: only O and the log-sum-exp are saved,
the attention matrix is recomputed from Q, K, V).  It is a drop-in for the
scaled-dot-product attention call that "Flash Attention La Gi?" and
"DL101 chapter 9", section 3, use, restricted to what the kernels support:
bf16 q [B, H, Nq, d] and k, v [B, Hkv, Nk, d] on a B200, d in {64, 128},
Hkv dividing H (grouped-query attention).  With Nq != Nk the queries are the
last Nq positions of the key sequence, so the causal mask keeps j <= i + Nk - Nq.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import fa


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal: bool, scale: Optional[float]):
        q, k, v = (t.contiguous() for t in (q, k, v))
        o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale = causal, scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = fa.bwd(q, k, v, o, do.contiguous().to(torch.bfloat16), lse,
                            causal=ctx.causal, scale=ctx.scale)
        return dq, dk, dv, None, None


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
              scale: Optional[float] = None) -> torch.Tensor:
    """softmax(scale * q k^T [+ causal mask]) v with a recomputing backward."""
    return _Attention.apply(q, k, v, bool(causal), scale)
