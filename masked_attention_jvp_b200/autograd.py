"""Autograd binding of the fused attention forward + JVP.

    o, to, lse, tlse = attention_jvp(q, k, v, tq, tk, tv, mask)

returns what attn_fwd_jvp returns, computed by the same fused kernel, and
makes o differentiable with respect to q, k and v: backward() runs the
library's backward kernels (caj_attn_bwd) on the saved q, k, v, o and LSE.
The tangent branch is stop-gradient, as in the student's gradient step of
TF-sCM (Causal-rCM, appendix A, the JVP of the stop-gradient network): to,
lse and tlse are returned as non-differentiable, and the tangents tq, tk, tv
receive no gradient. bf16 CUDA tensors only (the backward kernels' dtype).
"""
from __future__ import annotations

from typing import Optional

import torch

__all__ = ["attention_jvp"]


class _AttentionJvp(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, tq, tk, tv, mask, scale, clean_tangent_zero):
        from . import attn_fwd_jvp
        o, to, lse, tlse = attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale=scale,
                                        clean_tangent_zero=clean_tangent_zero)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.mask, ctx.scale = mask, scale
        ctx.mark_non_differentiable(to, lse, tlse)
        return o, to, lse, tlse

    @staticmethod
    def backward(ctx, do, _dto, _dlse, _dtlse):
        from . import attn_bwd
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv, _ = attn_bwd(q, k, v, o, do.contiguous(), lse, ctx.mask, scale=ctx.scale)
        return dq, dk, dv, None, None, None, None, None, None


def attention_jvp(q, k, v, tq, tk, tv, mask, scale: Optional[float] = None,
                  clean_tangent_zero: bool = False):
    """(o, to, lse, tlse) of the fused kernel, with o differentiable in q, k, v.
    q..tv: [B, H, N, D] contiguous bf16 CUDA tensors; mask: a MaskDesc."""
    for t in (q, k, v, tq, tk, tv):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("attention_jvp: q..tv must be contiguous bf16 CUDA tensors")
    return _AttentionJvp.apply(q, k, v, tq, tk, tv, mask, scale, clean_tangent_zero)
