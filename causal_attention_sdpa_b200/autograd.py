"""torch.autograd integration of the gpt_attn C ABI.

`gpt_attention(q, k, v)` is a drop-in for
`F.scaled_dot_product_attention(q, k, v, is_causal=True)` on bf16 CUDA tensors
[B, H, T, D] (heads as an extra batch dimension, as in the GPT-2 lecture's
attention module): the forward pass runs gpt_attn_fwd and keeps O and the
row log-sum-exp for the backward pass, which runs gpt_attn_bwd.  Argument
marshalling only; both passes run in the library's kernels.  The GPT-2
lecture's "Раздел 2" measures exactly this swap (switching the attention of a
GPT-2 training step to a fused kernel: same loss, shorter step).
"""
from __future__ import annotations

import math

import torch

from . import gpt_attn_bwd, gpt_attn_fwd


class GptAttnFunction(torch.autograd.Function):
    """O = softmax(scale * Q K^T, causal / windowed) V with its exact gradient."""

    @staticmethod
    def forward(ctx, q, k, v, scale, window):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = gpt_attn_fwd(q, k, v, scale=scale, window=window)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale = scale
        ctx.window = window
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = gpt_attn_bwd(q, k, v, o, lse, do.contiguous(), scale=ctx.scale, window=ctx.window)
        return dq, dk, dv, None, None


def gpt_attention(q, k, v, scale=None, window=0):
    """Causal (window <= 0) or sliding-window attention with autograd; q, k, v bf16 [B, H, T, D]."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return GptAttnFunction.apply(q, k, v, float(scale), int(window))
