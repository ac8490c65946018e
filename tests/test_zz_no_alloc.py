"""gpt_attn_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers run the backward pass where they may not allocate device memory
(an engine's enqueue step or a host callback, where cudaMalloc is not allowed,
or a process whose memory belongs to a pooling allocator).  For them the
library offers gpt_attn_bwd_noalloc, which uses a fixed 32 MiB scratch array
inside the library instead of a caller-supplied workspace.  These tests call
it through the C ABI and check it against gpt_attn_bwd, which takes its
workspace from the caller, and against the fp64 CPU oracle, on two calls in
a row: the second call reuses the scratch the first one left behind, with a
different shape.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import causal_attention_sdpa_b200 as ga
import oracle
from workloads import make_inputs

TOL_GRAD, TOL_FRO = 5e-2, 1e-2          # the gradient tolerances of the parity tests
FAKE = 0x10000


def _noalloc(L, t, scale, window, stream):
    q, k, v, o, lse, do, dq, dk, dv = t
    B, H, T, D = q.shape
    vp = ctypes.c_void_p
    return L.gpt_attn_bwd_noalloc(*[vp(x.data_ptr()) for x in t], B, H, T, D, ctypes.c_float(scale),
                                  int(window), vp(stream.cuda_stream))


def _close(name, got, ref):
    g = got.double().cpu()
    r = torch.as_tensor(np.asarray(ref, dtype=np.float64)) if not torch.is_tensor(ref) else ref.double().cpu()
    r = r.reshape(g.shape)
    err = (g - r).abs().max().item()
    assert err <= TOL_GRAD, f"{name}: max |err| {err:.3e}"
    rn = r.norm().item()
    if rn > 1e-6 * math.sqrt(r.numel()):
        fro = (g - r).norm().item() / rn
        assert fro <= TOL_FRO, f"{name}: rel Frobenius {fro:.3e}"


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    L = ga.lib()
    stream = torch.cuda.current_stream()
    cases = [  # (B, H, T, D, window, scale, seed): the first runs several work units per CTA on a
        # ragged T under a window; the second is smaller and uses D = 128
        (2, 48, 1000, 64, 200, 0.125, 11),
        (1, 2, 777, 128, 333, 0.12, 12),
    ]
    for B, H, T, D, W, s, seed in cases:
        q_h, k_h, v_h, do_h = make_inputs(B, H, T, D, seed=seed)
        q, k, v, do = (x.cuda() for x in (q_h, k_h, v_h, do_h))
        o, lse = ga.gpt_attn_fwd(q, k, v, scale=s, window=W)
        ref = ga.gpt_attn_bwd(q, k, v, o, lse, do, scale=s, window=W)
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        rc = _noalloc(L, [q, k, v, o, lse, do] + got, s, W, stream)
        assert rc == ga.GPT_ATTN_OK, ga.status_string(rc)
        assert ga.gpt_attn_check(stream) == ga.GPT_ATTN_OK
        exact = oracle.attn_bwd(q_h, k_h, v_h, do_h, s, W)[:3]
        for name, g_, r_, x_ in zip(("dq", "dk", "dv"), got, ref, exact):
            assert torch.isfinite(g_).all(), name
            _close(f"B{B}H{H}T{T}D{D} {name} vs gpt_attn_bwd", g_, r_)
            _close(f"B{B}H{H}T{T}D{D} {name} vs oracle", g_, x_)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """Validation happens before any device work, so this runs without a GPU."""
    from causal_attention_sdpa_b200 import build
    build.build()
    L = ga.lib()
    vp = ctypes.c_void_p
    args = [vp(FAKE)] * 9
    # B=64, H=12, T=1024, D=64 needs ~200 MB of workspace: more than the 32 MiB scratch
    assert ga.gpt_attn_bwd_workspace_bytes(64, 12, 1024, 64) > 32 << 20
    assert L.gpt_attn_bwd_noalloc(*args, 64, 12, 1024, 64, ctypes.c_float(0.125), 0, vp(0)) == \
        ga.GPT_ATTN_ERR_WORKSPACE
    assert L.gpt_attn_bwd_noalloc(*args[:8], vp(0), 1, 1, 8, 64, ctypes.c_float(0.125), 0, vp(0)) == \
        ga.GPT_ATTN_ERR_NULL
