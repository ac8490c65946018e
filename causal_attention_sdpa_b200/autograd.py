"""torch.autograd integration of the gpt_attn C ABI.

`gpt_attention(q, k, v)` is a drop-in for
`F.scaled_dot_product_attention(q, k, v, is_causal=True)` on bf16 CUDA tensors
[B, H, T, D] (heads as an extra batch dimension, as in the GPT-2 lecture's
attention module): the forward pass runs gpt_attn_fwd_ex and keeps O and the
row log-sum-exp for the backward pass, which runs gpt_attn_bwd_ex.  q, k and
v may be strided views (for instance the head views of a fused q/k/v
projection) as long as D is contiguous; nothing is copied into a
[B, H, T, D] layout first.  With out_layout="bthd" the result is returned as
[B, T, H, D], the layout the output projection reads, written there by the
kernel, and the gradients come back in that token-major layout too.
Argument marshalling only; both passes run in the library's kernels.  The
GPT-2 lecture's "Раздел 2" measures exactly this swap (switching the attention
of a GPT-2 training step to a fused kernel: same loss, shorter step).
"""
from __future__ import annotations

import math

import torch

from . import gpt_attn_bwd_ex, gpt_attn_fwd_ex


def _view_ok(t):
    return t.stride(-1) == 1 and all(s % 8 == 0 for s in t.stride()[:-1])


def _as_view(t):
    """t itself if the kernels can address it in place, else a contiguous copy."""
    return t if _view_ok(t) else t.contiguous()


class GptAttnFunction(torch.autograd.Function):
    """O = softmax(scale * Q K^T, causal / windowed) V with its exact gradient."""

    @staticmethod
    def forward(ctx, q, k, v, scale, window, token_major):
        q, k, v = _as_view(q), _as_view(k), _as_view(v)
        B, H, T, D = q.shape
        if token_major:
            out = torch.empty((B, T, H, D), dtype=q.dtype, device=q.device)
            o = out.permute(0, 2, 1, 3)
        else:
            out = o = torch.empty((B, H, T, D), dtype=q.dtype, device=q.device)
        _, lse = gpt_attn_fwd_ex(q, k, v, scale=scale, window=window, o=o)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale = scale
        ctx.window = window
        ctx.token_major = token_major
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse = ctx.saved_tensors
        B, H, T, D = q.shape
        do = dout.permute(0, 2, 1, 3) if ctx.token_major else dout
        do = _as_view(do)
        if ctx.token_major:
            bufs = [torch.empty((B, T, H, D), dtype=q.dtype, device=q.device).permute(0, 2, 1, 3) for _ in range(3)]
        else:
            bufs = [torch.empty((B, H, T, D), dtype=q.dtype, device=q.device) for _ in range(3)]
        dq, dk, dv = gpt_attn_bwd_ex(q, k, v, o, lse, do, scale=ctx.scale, window=ctx.window, dq=bufs[0],
                                     dk=bufs[1], dv=bufs[2])
        return dq, dk, dv, None, None, None


def gpt_attention(q, k, v, scale=None, window=0, out_layout="bhtd"):
    """Causal (window <= 0) or sliding-window attention with autograd.

    q, k, v: bf16 [B, H, T, D], any strides with contiguous D.  Returns O as [B, H, T, D]
    (out_layout="bhtd") or [B, T, H, D] (out_layout="bthd")."""
    if out_layout not in ("bhtd", "bthd"):
        raise ValueError("out_layout must be 'bhtd' or 'bthd'")
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return GptAttnFunction.apply(q, k, v, float(scale), int(window), out_layout == "bthd")
