"""torch.autograd wrapper over the library's forward and backward.

``flashmask_attention(q, k, v, lts, lte, uts, ute)`` returns O and records a
backward that calls ``fm_attn_bwd`` with the forward's O and LSE, so the kernels
can sit inside a PyTorch training step.  Layouts as in the C ABI: q [B, n_q, H, D],
k / v [B, n_k, H_kv, D] (bf16, or fp32 with D = 64), mask vectors int32
[B, Hm, n_k] (None = the canonical empty stretch).  The tile metadata is built
once per call and reused by the backward.  The vectors are integer data and get
no gradient.
"""
from __future__ import annotations

import math

import torch

from . import fm_attn_bwd, fm_attn_fwd, fm_build_mask_meta


class FlashMaskAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, lts, lte, uts, ute, scale, deterministic):
        vecs = [lts, lte, uts, ute]
        meta = fm_build_mask_meta(*vecs, n_q=q.shape[1])
        o, lse = fm_attn_fwd(q, k, v, meta, vecs, scale)
        ctx.save_for_backward(q, k, v, o, lse, lts, lte, uts, ute)
        ctx.meta, ctx.scale, ctx.deterministic = meta, scale, deterministic
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, lts, lte, uts, ute = ctx.saved_tensors
        dq, dk, dv = fm_attn_bwd(q, k, v, o, lse, do.contiguous(), ctx.meta, [lts, lte, uts, ute], ctx.scale,
                                 deterministic=ctx.deterministic)
        return dq, dk, dv, None, None, None, None, None, None


def flashmask_attention(q, k, v, lts=None, lte=None, uts=None, ute=None, scale=None, deterministic=False):
    """Masked softmax attention with the four boundary vectors; differentiable in q, k and v.
    scale defaults to 1 / sqrt(D); deterministic selects the fixed-order dQ backward."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return FlashMaskAttention.apply(q, k, v, lts, lte, uts, ute, float(scale), bool(deterministic))
