"""torch.autograd binding of the prefill: forward through kla_chunk_fwd,
backward through kla_chunk_bwd (argument marshalling only; every step of
both runs in the CUDA kernels of libkla.so).

    o, hT = kla_prefill(q, k, v, g, eta, eps=1e-6, h0=None)

q, k, v [B,T,H,d] bf16 or fp32 CUDA tensors, g, eta [B,T,H] fp32, h0
[B,H,dk,dv] fp32 or None.  Gradients flow to q, k, v, g, eta and h0; the
library returns them in fp32 and they are handed to autograd in each
input's dtype.
"""
from __future__ import annotations

import torch

from . import api


class _KLAPrefill(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, eta, h0, eps):
        o, hT = api.chunk_fwd(q, k, v, g, eta, eps, h0)
        ctx.save_for_backward(q, k, v, g, eta, h0)
        ctx.eps = eps
        return o, hT

    @staticmethod
    def backward(ctx, grad_o, grad_hT):
        q, k, v, g, eta, h0 = ctx.saved_tensors
        if grad_o is None:
            grad_o = torch.zeros_like(q[..., :v.shape[-1]])
        grad_o = grad_o.to(q.dtype).contiguous()
        if grad_hT is not None:
            grad_hT = grad_hT.float().contiguous()
        r = api.chunk_bwd(q, k, v, g, eta, grad_o, ctx.eps, h0, grad_hT,
                          need_h0=h0 is not None and ctx.needs_input_grad[5])
        dh0 = r["dh0"] if h0 is not None else None
        return (r["dq"].to(q.dtype), r["dk"].to(k.dtype), r["dv"].to(v.dtype), r["dg"],
                r["deta"], dh0, None)


def kla_prefill(q, k, v, g, eta, eps: float = 1e-6, h0=None):
    """Differentiable KLA prefill: returns (o, hT)."""
    return _KLAPrefill.apply(q, k, v, g, eta, h0, eps)
