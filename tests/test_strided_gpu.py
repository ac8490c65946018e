"""Strided layouts (gpt_attn_fwd_ex / gpt_attn_bwd_ex with tensor strides): attention read and
written in place inside a GPT-2 block's own buffers.

The GPT-2 lecture's attention module projects x to q, k, v in one matrix product, then treats heads
as a batch dimension by a view and a transpose; the library takes those views directly: q, k, v are
the three column blocks of a [B, T, 3, H, D] tensor, O is written into a [B, T, H, D] buffer (the
layout the output projection reads), and dQ, dK, dV go into one [B, T, 3, H, D] gradient buffer.
The results must equal those of contiguous tensors (forward, dK and dV bit for bit; dQ up to the
order of its fp32 sums) and match the fp64 oracle.  The CPU test checks the stride validation."""
import ctypes
import math

import numpy as np
import pytest
import torch

import causal_attention_sdpa_b200 as ga
import oracle
from workloads import make_inputs


def fused(q, k, v):
    """[B, H, T, D] q, k, v -> one [B, T, 3, H, D] tensor and its three [B, H, T, D] views."""
    B, H, T, D = q.shape
    qkv = torch.stack([q, k, v], dim=2).permute(0, 3, 2, 1, 4).contiguous()      # [B, T, 3, H, D]
    views = [qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3)]                   # [B, H, T, D] views
    return qkv, views


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,D,W", [(2, 12, 1000, 64, 0), (4, 6, 777, 64, 200), (1, 4, 700, 128, 0),
                                       (2, 3, 513, 128, 100)])
def test_strided_equals_contiguous_and_oracle(B, H, T, D, W):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    q, k, v, do = make_inputs(B, H, T, D, seed=B + T + D)
    s = 1.0 / math.sqrt(D)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    # contiguous reference run
    o_c, lse_c = ga.gpt_attn_fwd(qd, kd, vd, scale=s, window=W)
    dq_c, dk_c, dv_c = ga.gpt_attn_bwd(qd, kd, vd, o_c, lse_c, dod, scale=s, window=W)
    # strided run: inputs are views of a fused projection, outputs go into token-major buffers
    _, (qs, ks, vs) = fused(qd, kd, vd)
    y = torch.full((B, T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    o_s = y.permute(0, 2, 1, 3)
    dy = dod.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)                  # dO as a [B, T, H, D] view
    g = torch.full((B, T, 3, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dqs, dks, dvs = (g[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    assert not qs.is_contiguous() and not o_s.is_contiguous() and not dqs.is_contiguous()
    _, lse_s = ga.gpt_attn_fwd_ex(qs, ks, vs, scale=s, window=W, o=o_s)
    ga.gpt_attn_bwd_ex(qs, ks, vs, o_s, lse_s, dy, scale=s, window=W, dq=dqs, dk=dks, dv=dvs)
    assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
    assert torch.equal(o_s, o_c) and torch.equal(lse_s, lse_c)
    assert torch.equal(dks, dk_c) and torch.equal(dvs, dv_c)
    assert (dqs.float() - dq_c.float()).abs().max().item() <= 2 ** -6 * dq_c.float().abs().max().item()
    ro, _ = oracle.attn_fwd(q, k, v, s, W)
    rdq, rdk, rdv, _ = oracle.attn_bwd(q, k, v, do, s, W)
    for got, ref, tol in ((o_s, ro, 2e-2), (dqs, rdq, 5e-2), (dks, rdk, 5e-2), (dvs, rdv, 5e-2)):
        assert float(np.abs(got.float().cpu().double().numpy() - ref).max()) <= tol


def test_layout_validation():
    from causal_attention_sdpa_b200 import build
    build.build()
    L = ga.lib()
    vp = ctypes.c_void_p
    FAKE = 0x10000
    lay = ga.GptAttnLayout()
    for n in ("q", "k", "v", "o", "dO", "dq", "dk", "dv"):
        setattr(lay, n, ga.GptAttnStrides(12 * 64 * 64, 64 * 64, 64))
    ok = L.gpt_attn_fwd_ex(*[vp(FAKE)] * 5, 1, 12, 64, 64, ctypes.c_float(0.125), None, ctypes.byref(lay), vp(0))
    assert ok in (ga.GPT_ATTN_OK, ga.GPT_ATTN_ERR_CUDA)       # valid layout: any failure is past validation
    lay.k = ga.GptAttnStrides(12 * 64 * 64, 64 * 64, 68)       # token stride not a multiple of 8
    assert L.gpt_attn_fwd_ex(*[vp(FAKE)] * 5, 1, 12, 64, 64, ctypes.c_float(0.125), None, ctypes.byref(lay),
                             vp(0)) == ga.GPT_ATTN_ERR_ALIGN
    lay.k = ga.GptAttnStrides(-8, 64 * 64, 64)
    assert L.gpt_attn_fwd_ex(*[vp(FAKE)] * 5, 1, 12, 64, 64, ctypes.c_float(0.125), None, ctypes.byref(lay),
                             vp(0)) == ga.GPT_ATTN_ERR_SHAPE
