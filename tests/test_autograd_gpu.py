"""The torch.autograd wrapper of the C ABI (causal_attention_sdpa_b200.autograd) and its use
inside a GPT-2 model (bench_gpt2.py).

GPU: gradients that flow through `gpt_attention` are compared with the fp64 oracle at the parity
tolerances, and a small GPT-2 built with the gpt_attn arm matches the same model with the
attention written out (scores, causal mask, softmax, matmul) in loss and gradients: the GPT-2
lecture's "Раздел 2" point that switching to a fused attention changes the speed, not the loss.
CPU: the benchmark's model builds and runs its written-out arm.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import make_inputs

TOL_O, TOL_GRAD, TOL_FRO = 2e-2, 5e-2, 1e-2


def _cmp(name, got, ref, tol):
    g = got.detach().float().cpu().double().numpy()
    r = np.asarray(ref, dtype=np.float64).reshape(g.shape)
    err = float(np.abs(g - r).max())
    assert err <= tol, f"{name}: max |err| {err:.3e}"
    rn = float(np.linalg.norm(r))
    if rn > 1e-6 * math.sqrt(r.size):
        assert float(np.linalg.norm(g - r)) / rn <= TOL_FRO, name


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,D,W", [(2, 3, 300, 64, 0), (1, 2, 700, 128, 200), (4, 12, 1000, 64, 0)])
def test_autograd_matches_oracle(B, H, T, D, W):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    from causal_attention_sdpa_b200.autograd import gpt_attention
    q, k, v, do = make_inputs(B, H, T, D, seed=T + W)
    s = 1.0 / math.sqrt(D)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    o = gpt_attention(qd, kd, vd, window=W)
    o.backward(do.cuda())
    ro, _ = oracle.attn_fwd(q, k, v, s, W)
    rdq, rdk, rdv, _ = oracle.attn_bwd(q, k, v, do, s, W)
    _cmp("o", o, ro, TOL_O)
    _cmp("dq", qd.grad, rdq, TOL_GRAD)
    _cmp("dk", kd.grad, rdk, TOL_GRAD)
    _cmp("dv", vd.grad, rdv, TOL_GRAD)


@pytest.mark.gpu
def test_autograd_strided_inputs_and_token_major_output():
    """q, k, v as head views of a fused [B, T, 3, H, D] projection, O returned as [B, T, H, D]."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    from causal_attention_sdpa_b200.autograd import gpt_attention
    B, H, T, D = 2, 12, 500, 64
    q, k, v, do = make_inputs(B, H, T, D, seed=9)
    qkv = torch.stack([q, k, v], dim=2).permute(0, 3, 2, 1, 4).contiguous().cuda().requires_grad_(True)
    qs, ks, vs = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    y = gpt_attention(qs, ks, vs, out_layout="bthd")            # [B, T, H, D]
    assert tuple(y.shape) == (B, T, H, D)
    y.backward(do.permute(0, 2, 1, 3).cuda())
    s = 1.0 / math.sqrt(D)
    ro, _ = oracle.attn_fwd(q, k, v, s)
    rdq, rdk, rdv, _ = oracle.attn_bwd(q, k, v, do, s)
    _cmp("o", y.permute(0, 2, 1, 3), ro, TOL_O)
    g = qkv.grad
    for i, (name, ref) in enumerate((("dq", rdq), ("dk", rdk), ("dv", rdv))):
        _cmp(name, g[:, :, i].permute(0, 2, 1, 3), ref, TOL_GRAD)


@pytest.mark.gpu
def test_gpt2_arms_agree():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    import bench_gpt2
    torch.manual_seed(0)
    idx = torch.randint(0, 512, (2, 257))
    x, y = idx[:, :-1].cuda(), idx[:, 1:].cuda()
    out = {}
    for arm in ("naive", "gpt_attn"):
        m = bench_gpt2.build(arm, n_layer=2, n_head=2, d_model=128, block=256, vocab=512).cuda()
        with torch.autocast("cuda", dtype=torch.bfloat16):
            loss = m(x, y)
        loss.backward()
        out[arm] = (float(loss), {n: p.grad.float().clone() for n, p in m.named_parameters()})
    l0, g0 = out["naive"]
    l1, g1 = out["gpt_attn"]
    assert abs(l0 - l1) <= 1e-2 * abs(l0), (l0, l1)
    for n in g0:
        rel = float((g0[n] - g1[n]).norm() / g0[n].norm().clamp_min(1e-12))
        assert rel <= 5e-2, (n, rel)


def test_gpt2_model_runs_on_cpu():
    import bench_gpt2
    m = bench_gpt2.build("naive", n_layer=1, n_head=2, d_model=64, block=64, vocab=100)
    idx = torch.randint(0, 100, (2, 33))
    loss = m(idx[:, :-1], idx[:, 1:])
    assert torch.isfinite(loss) and abs(float(loss) - math.log(100)) < 0.5
