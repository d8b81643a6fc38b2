"""The layer as a torch.autograd.Function: moe_forward on the way in, moe_backward on the way back.

Training is the setting of the kieve-moe Features (load-balancing auxiliary loss), the MoEEvolve README
(Architecture) and MoEFFN.forward in moe_stream.py.  ``MoEFunction.apply`` returns the layer output; the
load-balance statistic aux enters the gradient with weight ``aux_coef`` (L = loss(out) + aux_coef * aux), so
the aux value returned by ``moe_layer(..., return_aux=True)`` is for logging and must not be added to the loss
again.  Gradients flow to x, W_r, the routed experts' w13 and w2 and the shared expert's; the routing decision
and the exploration bias take none.  bf16 experts only.  The weight gradients are computed in fp32 and handed
to autograd, which casts them to the parameters' dtype.

Nothing is kept from the forward but its inputs: the backward recomputes the routing and the experts' [g | u].
"""

from __future__ import annotations

import torch

from . import MoeShape, moe_backward, moe_forward


class MoEFunction(torch.autograd.Function):
    """Inputs: shape (MoeShape), aux_coef (float), x [T, d] bf16, w_router [E, d] fp32, bias [E] fp32 or None,
    w13 [E, 2H, d] bf16, w2 [E, d, H] bf16, w13_sh / w2_sh (or None)."""

    @staticmethod
    def forward(ctx, shape: MoeShape, aux_coef: float, x, w_router, bias, w13, w2, w13_sh, w2_sh):
        r = moe_forward(shape, x, w_router, w13, w2, bias=bias, w13_sh=w13_sh, w2_sh=w2_sh, aux=True)
        ctx.shape, ctx.aux_coef = shape, float(aux_coef)
        ctx.save_for_backward(x, w_router, bias if bias is not None else torch.empty(0), w13, w2,
                              w13_sh if w13_sh is not None else torch.empty(0),
                              w2_sh if w2_sh is not None else torch.empty(0))
        ctx.has = (bias is not None, w13_sh is not None)
        ctx.mark_non_differentiable(r["aux"])
        return r["out"], r["aux"]

    @staticmethod
    def backward(ctx, dout, _daux):
        x, w_router, bias, w13, w2, w13_sh, w2_sh = ctx.saved_tensors
        has_bias, has_sh = ctx.has
        g = moe_backward(ctx.shape, x, w_router, w13, w2, dout.to(torch.bfloat16).contiguous(),
                         bias=bias if has_bias else None, w13_sh=w13_sh if has_sh else None,
                         w2_sh=w2_sh if has_sh else None, aux_coef=ctx.aux_coef)
        return (None, None, g["dx"], g["dw_router"], None, g["dw13"], g["dw2"],
                g["dw13_sh"] if has_sh else None, g["dw2_sh"] if has_sh else None)


def moe_layer(shape: MoeShape, x, w_router, w13, w2, *, bias=None, w13_sh=None, w2_sh=None, aux_coef=0.0,
              return_aux=False):
    """Differentiable routed MoE layer (bf16 experts).  Returns out [T, d] bf16, and aux [1] fp32 (detached)
    when ``return_aux``."""
    out, aux = MoEFunction.apply(shape, aux_coef, x, w_router, bias, w13, w2, w13_sh, w2_sh)
    return (out, aux) if return_aux else out
