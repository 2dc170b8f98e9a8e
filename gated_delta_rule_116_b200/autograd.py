"""torch.autograd wiring of the library's prefill and its backward pass.

Argument marshalling only: the forward is ``chunk_fwd`` and the backward is
``chunk_bwd``, both running in ``libkda.so``.

    out, S_T = kda_prefill(q, k, v, log_alpha, beta, S0)   # differentiable in all six inputs
"""
from __future__ import annotations

import torch

from . import binding


class KDAPrefill(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, log_alpha, beta, S0, chunk):
        out, S_T = binding.chunk_fwd(q, k, v, log_alpha, beta, S0, chunk=chunk)
        ctx.save_for_backward(q, k, v, log_alpha, beta, S0)
        ctx.has_s0 = S0 is not None
        return out, S_T

    @staticmethod
    def backward(ctx, grad_out, grad_S_T):
        if not any(ctx.needs_input_grad[:6]):
            return (None,) * 7
        q, k, v, log_alpha, beta, S0 = ctx.saved_tensors
        if grad_out is None:
            grad_out = torch.zeros(*q.shape[:3], v.shape[-1], device=q.device, dtype=q.dtype)
        g = binding.chunk_bwd(q, k, v, log_alpha, beta, grad_out.to(q.dtype).contiguous(),
                              S0 if ctx.has_s0 else None,
                              None if grad_S_T is None else grad_S_T.float().contiguous())
        need = ctx.needs_input_grad
        grads = (g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                 g["S0"] if ctx.has_s0 else None)
        return tuple(x if need[i] else None for i, x in enumerate(grads)) + (None,)


def kda_prefill(q, k, v, log_alpha, beta, S0=None, chunk: int = 64):
    """Differentiable chunked prefill: returns ``(out, S_T)`` like ``chunk_fwd``;
    gradients flow to q, k, v, log_alpha, beta and S0 through ``chunk_bwd``.

    The backward kernel takes dL/d(out) in the dtype of q, so with bf16 inputs an
    fp32 upstream gradient is rounded to bf16 before it runs (the gradients of
    q, k and v are bf16 as well). The kernel computes every gradient in one
    pass; inputs that do not require a gradient receive None."""
    return KDAPrefill.apply(q, k, v, log_alpha, beta, S0, chunk)
