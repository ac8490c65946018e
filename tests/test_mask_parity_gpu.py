"""GPU parity of the masked entry points (gpt_attn_fwd_ex / gpt_attn_bwd_ex with a mask) against the
fp64 oracle's masked functions: per-head windows (the long/short sliding-window pattern) and
document starts (batches aligned to document ends), from the modded-nanogpt README's technique
list, on the same seeded inputs, element by element, at the parity tolerances.

Cases cover both head dimensions, ragged T, several work items per CTA in the persistent D = 64
kernels, windows and documents together, one-token documents, and the plain entry points'
equality with the masked ones under a single window.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import make_inputs

pytestmark = pytest.mark.gpu

TOL_O, TOL_GRAD, TOL_FRO, TOL_LSE = 2e-2, 5e-2, 1e-2, 1e-3


@pytest.fixture(scope="module")
def ga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import causal_attention_sdpa_b200 as m
    from causal_attention_sdpa_b200 import build
    build.build()
    m.lib()
    return m


def check(name, got, ref):
    g = got.float().cpu().double().numpy()
    r = np.asarray(ref, dtype=np.float64).reshape(g.shape)
    assert np.isfinite(g).all(), f"{name}: non-finite values"
    err = float(np.abs(g - r).max())
    if name == "lse":
        assert err <= TOL_LSE, f"lse: max |err| {err:.3e}"
        return
    tol = TOL_O if name == "o" else TOL_GRAD
    assert err <= tol, f"{name}: max |err| {err:.3e}"
    rn = float(np.linalg.norm(r))
    if rn > 1e-6 * math.sqrt(r.size):
        fro = float(np.linalg.norm(g - r)) / rn
        assert fro <= TOL_FRO, f"{name}: rel Frobenius {fro:.3e}"


CASES = [
    # (B, H, T, D, head_windows or None, window, max document length or None, scale)
    (2, 4, 1000, 64, [0, 1, 200, 700], 0, None, 0.125),        # per-head windows only
    (3, 2, 1024, 64, None, 0, 300, 0.125),                     # documents only
    (2, 2, 777, 64, [128, 0], 0, 250, 0.125),                  # both, ragged T
    (8, 12, 1000, 64, None, 256, 200, 0.125),                  # several items per CTA
    (1, 2, 1500, 128, [256, 0], 0, 400, 0.12),                 # D = 128, both
    (2, 3, 700, 128, None, 100, 90, 0.088),                    # D = 128, window + documents
    (1, 2, 640, 64, None, 0, 1, 0.125),                        # one-token documents
]


@pytest.mark.parametrize("B,H,T,D,hw,W,L,s", CASES,
                         ids=[f"B{c[0]}H{c[1]}T{c[2]}D{c[3]}{'hw' if c[4] else ''}W{c[5]}L{c[6]}" for c in CASES])
def test_masked_parity(ga, B, H, T, D, hw, W, L, s):
    q, k, v, do = make_inputs(B, H, T, D, seed=T + D + (L or 0))
    ds = workloads.make_doc_starts(B, T, seed=T, max_doc_len=L) if L else None
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    dsd = torch.from_numpy(ds).cuda() if ds is not None else None
    o, lse = ga.gpt_attn_fwd_ex(qd, kd, vd, scale=s, window=W, head_windows=hw, doc_start=dsd)
    dq, dk, dv = ga.gpt_attn_bwd_ex(qd, kd, vd, o, lse, dod, scale=s, window=W, head_windows=hw,
                                        doc_start=dsd)
    assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
    ro, rl = oracle.attn_fwd_masked(q, k, v, s, hw, W, ds)
    rdq, rdk, rdv, _ = oracle.attn_bwd_masked(q, k, v, do, s, hw, W, ds)
    for name, g, r in (("o", o, ro), ("lse", lse, rl), ("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        check(name, g, r)


def test_plain_entry_points_equal_masked_ones(ga):
    """gpt_attn_fwd/bwd(window) is gpt_attn_*_ex with {window, NULL, NULL} and no layout: same bits."""
    q, k, v, do = (t.cuda() for t in make_inputs(2, 3, 500, 64, seed=3))
    o1, l1 = ga.gpt_attn_fwd(q, k, v, window=100)
    o2, l2 = ga.gpt_attn_fwd_ex(q, k, v, window=100)
    dq1, dk1, dv1 = ga.gpt_attn_bwd(q, k, v, o1, l1, do, window=100)
    dq2, dk2, dv2 = ga.gpt_attn_bwd_ex(q, k, v, o1, l1, do, window=100)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert (dq1.float() - dq2.float()).abs().max().item() <= 2 ** -6 * dq1.float().abs().max().item()


def test_same_window_per_head_equals_scalar_window(ga):
    q, k, v, _ = (t.cuda() for t in make_inputs(1, 4, 600, 64, seed=4))
    o1, l1 = ga.gpt_attn_fwd(q, k, v, window=200)
    o2, l2 = ga.gpt_attn_fwd_ex(q, k, v, head_windows=[200] * 4)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
