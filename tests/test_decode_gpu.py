"""Decode attention (gpt_attn_decode): one new query per sequence against its key/value cache, the
step of the generation loop of "Un GPT desde cero + nanoGPT" (Laboratorio L2.1, generate).

GPU: compared with the fp64 oracle's decode function on the same seeded inputs at the parity
tolerances, over both head dimensions, one and many key splits, windows, ragged per-sequence
lengths (including an empty sequence and lengths past the cache) and long caches.  CPU: the
C ABI rejects bad arguments before any device work."""
import ctypes

import numpy as np
import pytest
import torch

import causal_attention_sdpa_b200 as ga
import oracle
from workloads import make_inputs

TOL_O, TOL_LSE = 2e-2, 1e-3


CASES = [
    # (B, H, T_max, D, window, lens, scale)
    (1, 12, 1024, 64, 0, [1024], 0.125),                 # GPT-2 124M, one sequence, full cache
    (4, 12, 1024, 64, 0, [1, 300, 777, 1024], 0.125),    # ragged lengths
    (8, 6, 256, 64, 0, [256, 5, 17, 128, 129, 200, 64, 1], 0.125),
    (2, 4, 8192, 128, 1024, [8192, 3000], 0.12),         # long cache, window
    (3, 2, 500, 128, 0, [0, 499, 10000], 0.088),         # empty sequence, length past the cache
    (64, 12, 1024, 64, 0, None, 0.125),                  # many heads: one split each
    (32, 12, 1024, 64, 0, None, 0.125),                  # two splits each
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,D,W,lens,s", CASES, ids=[f"B{c[0]}H{c[1]}T{c[2]}D{c[3]}W{c[4]}" for c in CASES])
def test_decode_parity(B, H, T, D, W, lens, s):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_sdpa_b200 import build
    build.build()
    q4, k, v, _ = make_inputs(B, H, T, D, seed=B * T + D + W)
    q = q4[:, :, -1].contiguous()                     # [B, H, D]
    if lens is None:
        lens = list(np.random.default_rng(B).integers(1, T + 1, size=B))
    ld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = ga.gpt_attn_decode(q.cuda(), k.cuda(), v.cuda(), ld, scale=s, window=W)
    assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
    ro, rl = oracle.attn_decode(q, k, v, lens, s, W)
    g = o.float().cpu().double().numpy()
    assert np.isfinite(g).all()
    assert float(np.abs(g - ro).max()) <= TOL_O
    gl = lse.cpu().double().numpy()
    empty = np.isneginf(rl)
    assert (np.isneginf(gl) == empty).all()
    assert float(np.abs(gl[~empty] - rl[~empty]).max(initial=0.0)) <= TOL_LSE
    rn = float(np.linalg.norm(ro))
    if rn > 0:
        assert float(np.linalg.norm(g - ro)) / rn <= 1e-2


FAKE = 0x10000


def test_decode_argument_checks():
    from causal_attention_sdpa_b200 import build
    build.build()
    L = ga.lib()
    vp = ctypes.c_void_p
    ws = ga.gpt_attn_decode_workspace_bytes(1, 12, 1024, 64, 0)
    assert ws > 16                                     # 12 heads split the keys over several CTAs
    assert ga.gpt_attn_decode_workspace_bytes(64, 12, 1024, 64, 0) == 16   # one split: no partials
    assert ga.gpt_attn_decode_workspace_bytes(1, 1, 8, 32, 0) == 0

    def call(ptrs=None, B=1, H=12, T=1024, D=64, w=FAKE, nbytes=ws):
        p = [FAKE] * 6 if ptrs is None else ptrs
        return L.gpt_attn_decode(*[vp(x) for x in p], B, H, T, D, ctypes.c_float(0.125), 0, vp(w), nbytes, vp(0))

    for i in range(6):
        p = [FAKE] * 6
        p[i] = 0
        assert call(p) == ga.GPT_ATTN_ERR_NULL
    assert call(D=96) == ga.GPT_ATTN_ERR_UNSUPPORTED_D
    assert call(T=0) == ga.GPT_ATTN_ERR_SHAPE
    assert call(nbytes=ws - 1) == ga.GPT_ATTN_ERR_WORKSPACE
    assert call(w=0) == ga.GPT_ATTN_ERR_WORKSPACE
    for i in range(6):
        p = [FAKE] * 6
        p[i] = FAKE + (2 if i in (3, 5) else 8)        # lens and lse need 4 bytes, the rest 16
        assert call(p) == ga.GPT_ATTN_ERR_ALIGN, i
