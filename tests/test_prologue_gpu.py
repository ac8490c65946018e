"""QK-Norm + rotary prologue kernels (gpt_attn_qk_prologue_fwd / _bwd) against the fp64 oracle.

The raw q and k come in as the column views of a fused [B, T, 3, H, D] projection (the layout of
the GPT-2 lecture's attention module, heads as a batch dimension without a copy); the prologue's
outputs feed gpt_attn_fwd, and its backward takes the attention's dQ, dK and writes the raw
gradients into the fused gradient buffer.  Each stage is compared with the oracle on the same
bf16 inputs; the CPU test checks argument validation."""
import ctypes
import math

import numpy as np
import pytest
import torch

import causal_attention_sdpa_b200 as ga
import oracle
from workloads import make_inputs


def _err(got, ref):
    g = got.float().cpu().double().numpy()
    r = np.asarray(ref, dtype=np.float64).reshape(g.shape)
    return float(np.abs(g - r).max()), float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))


@pytest.mark.gpu
@pytest.mark.parametrize("layout", ["fused", "bhtd"])
@pytest.mark.parametrize("B,H,T,D,norm,base", [(2, 12, 1000, 64, True, 10000.0), (1, 6, 8192, 128, True, 10000.0),
                                               (2, 4, 300, 64, False, 10000.0), (2, 4, 300, 128, True, 0.0)])
def test_prologue_then_attention_matches_oracle(B, H, T, D, norm, base, layout):
    """layout "fused": q, k as views of a [B, T, 3, H, D] projection (a token's heads adjacent: the
    kernels take a token at a time); "bhtd": contiguous [B, H, T, D] (the kernels take a row at a
    time)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    q, k, v, do = make_inputs(B, H, T, D, seed=T + D)
    if layout == "fused":
        qkv = torch.stack([q, k, v], dim=2).permute(0, 3, 2, 1, 4).contiguous().cuda()     # [B, T, 3, H, D]
        qr, kr, vr = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    else:
        qr, kr, vr = q.cuda(), k.cuda(), v.cuda()
    qn, kn = ga.gpt_attn_qk_prologue_fwd(qr, kr, qk_norm=norm, rope_base=base)
    # the prologue against the oracle on the same raw rows
    for got, raw in ((qn, q), (kn, k)):
        mx, fro = _err(got, oracle.qk_prologue_fwd(raw, norm, base))
        assert mx <= 2e-2 and fro <= 1e-2, (mx, fro)
    # attention on the prologue's outputs, then the prologue's backward into the fused buffer
    s = 1.0 / math.sqrt(D)
    o, lse = ga.gpt_attn_fwd(qn, kn, vr.contiguous(), scale=s)
    dq, dk, dv = ga.gpt_attn_bwd(qn, kn, vr.contiguous(), o, lse, do.cuda(), scale=s)
    if layout == "fused":
        g = torch.full((B, T, 3, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        dqr, dkr = (g[:, :, i].permute(0, 2, 1, 3) for i in range(2))
    else:
        dqr, dkr = (torch.full((B, H, T, D), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2))
    ga.gpt_attn_qk_prologue_bwd(qr, kr, dq, dk, qk_norm=norm, rope_base=base, dq_raw=dqr, dk_raw=dkr)
    assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
    for got, raw, dy in ((dqr, q, dq), (dkr, k, dk)):
        ref = oracle.qk_prologue_bwd(raw, dy.cpu(), norm, base)
        mx, fro = _err(got, ref)
        scale_ref = float(np.abs(ref).max())
        assert mx <= 5e-2 * max(1.0, scale_ref) and fro <= 1e-2, (mx, fro, scale_ref)


def test_prologue_argument_checks():
    from causal_attention_sdpa_b200 import build
    build.build()
    L = ga.lib()
    vp = ctypes.c_void_p
    FAKE = 0x10000
    assert L.gpt_attn_qk_prologue_fwd(vp(FAKE), vp(FAKE), vp(FAKE), vp(0), 1, 2, 8, 64, 1, ctypes.c_float(1e4),
                                      None, vp(0)) == ga.GPT_ATTN_ERR_NULL
    assert L.gpt_attn_qk_prologue_fwd(vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), 1, 2, 8, 48, 1, ctypes.c_float(1e4),
                                      None, vp(0)) == ga.GPT_ATTN_ERR_UNSUPPORTED_D
    bad = (ga.GptAttnStrides * 4)(*[ga.GptAttnStrides(2 * 8 * 64, 8 * 64, 60)] * 4)
    assert L.gpt_attn_qk_prologue_fwd(vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), 1, 2, 8, 64, 1, ctypes.c_float(1e4),
                                      bad, vp(0)) == ga.GPT_ATTN_ERR_ALIGN
    assert L.gpt_attn_qk_prologue_bwd(*[vp(FAKE)] * 5, vp(FAKE + 8), 1, 2, 8, 64, 1, ctypes.c_float(1e4), None,
                                      vp(0)) == ga.GPT_ATTN_ERR_ALIGN
