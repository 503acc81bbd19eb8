"""PyTorch autograd entry point of the recurrence: the chunkwise forward
(gdr_forward_chunked) with its reverse mode (gdr_backward_chunked) as the backward.

    o, S_T = gdr_chunked(form, q, k, v, log_w, e1, e2, S0)

Tensors as gdr.gdr_forward_chunked; o and S_T are fp32.  Gradients flow to q, k, v,
log_w, e1, e2 and S0 (returned in each input's dtype), from the gradients of o and S_T.
The backward recomputes what it needs from the inputs (nothing but the inputs is saved)
and supports d_k, d_v in {64, 128}.
"""
from __future__ import annotations

import torch

from . import gdr

__all__ = ["gdr_chunked"]


class _GDRChunked(torch.autograd.Function):
    @staticmethod
    def forward(ctx, form, chunk, q, k, v, log_w, e1, e2, S0):
        o, S_T = gdr.gdr_forward_chunked(form, q, k, v, log_w, e1, e2, S0, chunk=chunk)
        ctx.form, ctx.chunk = form, chunk
        ctx.save_for_backward(q, k, v, log_w, e1, e2, S0)
        return o, S_T

    @staticmethod
    def backward(ctx, dO, dS_T):
        q, k, v, log_w, e1, e2, S0 = ctx.saved_tensors
        if dO is None:
            dO = torch.zeros(v.shape, dtype=torch.float32, device=v.device)
        g = gdr.gdr_backward_chunked(ctx.form, q, k, v, log_w, e1, e2, S0,
                                     dO.contiguous().float(),
                                     None if dS_T is None else dS_T.contiguous().float(),
                                     chunk=ctx.chunk, want_S0=S0 is not None)
        cast = lambda grad, x: None if grad is None or x is None else grad.to(x.dtype)
        return (None, None, cast(g["q"], q), cast(g["k"], k), cast(g["v"], v),
                cast(g["log_w"], log_w), cast(g["e1"], e1), cast(g["e2"], e2), cast(g["S0"], S0))


def gdr_chunked(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, chunk=64):
    """Differentiable chunkwise forward: returns (o, S_T)."""
    return _GDRChunked.apply(form, chunk, q, k, v, log_w, e1, e2, S0)
