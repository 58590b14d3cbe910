"""Dispatch and combine as differentiable torch operations.

In training the step runs forward and backward ("How MoonEP works": the
duplicates' gradients are summed back into the home copy in the backward
pass).  These functions wire the forward kernels to their adjoints so that a
model can call them inside autograd:

* ``dispatch(x, plan)``: ``buf[slot[g,k]] = x[g]``; backward
  ``grad_x[g] = bf16(sum_k grad_buf[slot[g,k]])`` (``mep_dispatch_backward``).
* ``combine(y, topk_w, plan)``: ``out[g] = bf16(sum_k w[g,k] y[slot[g,k]])``;
  backward ``grad_y[slot[g,k]] = bf16(w[g,k] grad_out[g])`` and
  ``grad_w[g,k] = <grad_out[g], y[slot[g,k]]>`` (``mep_combine_backward``).

The plan is computed once per step (``mep_plan`` / ``mep_plan_home_first``)
and passed in; it carries no gradient.  Every operation runs in the libmep
kernels on the current stream; there is no CPU path.
"""
from __future__ import annotations

import torch

from . import (Plan, mep_combine, mep_combine_backward, mep_dispatch, mep_dispatch_backward)

__all__ = ["dispatch", "combine"]


class _Dispatch(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x: torch.Tensor, plan: Plan):
        s = plan.shape
        H = x.shape[-1]
        buf = torch.empty((s.R, s.SK, H), dtype=torch.bfloat16, device=x.device)
        mep_dispatch(s, H, plan, x.contiguous(), buf)
        ctx.plan, ctx.H = plan, H
        return buf

    @staticmethod
    def backward(ctx, grad_buf: torch.Tensor):
        plan, H = ctx.plan, ctx.H
        s = plan.shape
        grad_x = torch.empty((s.N, H), dtype=torch.bfloat16, device=grad_buf.device)
        mep_dispatch_backward(s, H, plan, grad_buf.contiguous(), grad_x)
        return grad_x, None


class _Combine(torch.autograd.Function):
    @staticmethod
    def forward(ctx, y: torch.Tensor, topk_w: torch.Tensor, plan: Plan):
        s = plan.shape
        H = y.shape[-1]
        y = y.contiguous()
        w = topk_w.contiguous()
        out = torch.empty((s.N, H), dtype=torch.bfloat16, device=y.device)
        mep_combine(s, H, plan, y, w, out)
        ctx.save_for_backward(y, w)
        ctx.plan, ctx.H = plan, H
        return out

    @staticmethod
    def backward(ctx, grad_out: torch.Tensor):
        y, w = ctx.saved_tensors
        plan, H = ctx.plan, ctx.H
        s = plan.shape
        grad_y = torch.empty((s.R, s.SK, H), dtype=torch.bfloat16, device=y.device)
        grad_w = torch.empty((s.N, s.K), dtype=torch.float32, device=y.device)
        mep_combine_backward(s, H, plan, grad_out.contiguous(), w, y, grad_y, grad_w)
        return grad_y.view_as(y), grad_w.view_as(w), None


def dispatch(x: torch.Tensor, plan: Plan) -> torch.Tensor:
    """bf16 ``x`` [R*S, H] -> the static receive buffer [R, S*K, H] (differentiable in x)."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a bf16 [N, H] tensor")
    return _Dispatch.apply(x, plan)


def combine(y: torch.Tensor, topk_w: torch.Tensor, plan: Plan) -> torch.Tensor:
    """bf16 expert outputs ``y`` [R, S*K, H] (or [R*S*K, H]) and fp32 router
    weights [R*S, K] -> bf16 [R*S, H] (differentiable in y and the weights)."""
    if y.dtype != torch.bfloat16 or topk_w.dtype != torch.float32:
        raise TypeError("y must be bf16 and topk_w float32")
    return _Combine.apply(y, topk_w, plan)
