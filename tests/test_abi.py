"""Host-side checks of the C ABI: the library loads, exports every entry point
include/gpt_attn.h declares, and rejects bad arguments with the documented
status codes before touching the GPU (so these run without one)."""
import ctypes
import os
import re

import pytest

import causal_attention_sdpa_b200 as ga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from causal_attention_sdpa_b200 import build
    build.build()
    return ga.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gpt_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert set(names) == set(ga.EXPORTED), names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/gpt_attn.h but not exported"


def test_status_strings(L):
    for code in range(10):
        s = ga.status_string(code)
        assert s and s != "unknown status"
    assert ga.status_string(99) == "unknown status"


FAKE = 0x10000   # 16-byte aligned, never dereferenced: validation fails before any device work


def fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, T=8, D=64):
    vp = ctypes.c_void_p
    return L.gpt_attn_fwd(vp(q), vp(k), vp(v), vp(o), vp(lse), B, H, T, D, 0.125, 0, vp(0))


@pytest.mark.parametrize("which", range(5))
def test_fwd_null_pointers(L, which):
    args = [FAKE] * 5
    args[which] = 0
    assert fwd(L, *args) == ga.GPT_ATTN_ERR_NULL


@pytest.mark.parametrize("B,H,T", [(0, 1, 8), (1, 0, 8), (1, 1, 0), (-1, 1, 8), (1, 1, -5)])
def test_fwd_bad_shapes(L, B, H, T):
    assert fwd(L, B=B, H=H, T=T) == ga.GPT_ATTN_ERR_SHAPE


@pytest.mark.parametrize("D", [0, 16, 32, 63, 96, 256])
def test_fwd_unsupported_head_dim(L, D):
    assert fwd(L, D=D) == ga.GPT_ATTN_ERR_UNSUPPORTED_D


def test_fwd_overflowing_shape(L):
    assert fwd(L, B=2**30, H=2**30, T=2**30, D=64) == ga.GPT_ATTN_ERR_SHAPE


@pytest.mark.parametrize("which", range(5))
def test_fwd_misaligned(L, which):
    args = [FAKE] * 5
    args[which] = FAKE + 8
    assert fwd(L, *args) == ga.GPT_ATTN_ERR_ALIGN


def test_workspace_bytes(L):
    # fp32 dQ accumulator + three 32-bit rows per head padded to a multiple of 128 + one int per
    # (head, 128-key tile) + a 16-byte counter
    assert ga.gpt_attn_bwd_workspace_bytes(2, 3, 200, 64) == 4 * (6 * 200 * 64 + 3 * 6 * 256 + 6 * 2) + 16
    assert ga.gpt_attn_bwd_workspace_bytes(1, 1, 128, 128) == 4 * (128 * 128 + 3 * 128 + 1) + 16
    assert ga.gpt_attn_bwd_workspace_bytes(1, 1, 8, 32) == 0
    assert ga.gpt_attn_bwd_workspace_bytes(0, 1, 8, 64) == 0


def bwd(L, ptrs=None, B=1, H=1, T=8, D=64, ws=FAKE, ws_bytes=None):
    vp = ctypes.c_void_p
    p = [FAKE] * 9 if ptrs is None else ptrs
    if ws_bytes is None:
        ws_bytes = ga.gpt_attn_bwd_workspace_bytes(B, H, T, D)
    return L.gpt_attn_bwd(*[vp(x) for x in p], B, H, T, D, 0.125, 0, vp(ws), ws_bytes, vp(0))


@pytest.mark.parametrize("which", range(9))
def test_bwd_null_pointers(L, which):
    p = [FAKE] * 9
    p[which] = 0
    assert bwd(L, p) == ga.GPT_ATTN_ERR_NULL


def test_bwd_workspace_checks(L):
    assert bwd(L, ws=0) == ga.GPT_ATTN_ERR_WORKSPACE
    need = ga.gpt_attn_bwd_workspace_bytes(1, 1, 8, 64)
    assert bwd(L, ws_bytes=need - 1) == ga.GPT_ATTN_ERR_WORKSPACE


@pytest.mark.parametrize("which", range(9))
def test_bwd_misaligned(L, which):
    p = [FAKE] * 9
    p[which] = FAKE + 4
    assert bwd(L, p) == ga.GPT_ATTN_ERR_ALIGN


def test_bwd_bad_shape_and_d(L):
    assert bwd(L, T=0, ws_bytes=1 << 20) == ga.GPT_ATTN_ERR_SHAPE
    assert bwd(L, D=32, ws_bytes=1 << 20) == ga.GPT_ATTN_ERR_UNSUPPORTED_D


def test_debug_wait_rejects_bad_timeout(L):
    assert L.gpt_attn_debug_wait_timeout(0, ctypes.c_void_p(0)) == ga.GPT_ATTN_ERR_SHAPE
    assert L.gpt_attn_debug_wait_timeout(10**8, ctypes.c_void_p(0)) == ga.GPT_ATTN_ERR_SHAPE


def test_binding_has_no_oracle_dependency():
    """The product package must not reach the CPU oracle."""
    pkg = os.path.join(ROOT, "causal_attention_sdpa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle.c" not in text and "liboracle" not in text, f


def test_masked_entry_point_checks(L):
    """Mask validation runs before any device work."""
    vp = ctypes.c_void_p
    hw = (ctypes.c_int * 65)(*([1] * 65))
    m = ga.GptAttnMask(0, ctypes.cast(hw, ctypes.POINTER(ctypes.c_int)), None)
    p = [vp(FAKE)] * 5
    # per-head windows are limited to 64 heads
    assert L.gpt_attn_fwd_ex(*p, 1, 65, 8, 64, ctypes.c_float(0.125), ctypes.byref(m), None, vp(0)) == \
        ga.GPT_ATTN_ERR_SHAPE
    # document starts must be 4-byte aligned
    m2 = ga.GptAttnMask(0, None, FAKE + 2)
    assert L.gpt_attn_fwd_ex(*p, 1, 2, 8, 64, ctypes.c_float(0.125), ctypes.byref(m2), None, vp(0)) == \
        ga.GPT_ATTN_ERR_ALIGN
    ws = ga.gpt_attn_bwd_workspace_bytes(1, 2, 8, 64)
    q9 = [vp(FAKE)] * 9
    assert L.gpt_attn_bwd_ex(*q9, 1, 2, 8, 64, ctypes.c_float(0.125), ctypes.byref(m2), None, vp(FAKE), ws,
                             vp(0)) == ga.GPT_ATTN_ERR_ALIGN
    assert L.gpt_attn_bwd_ex(*q9[:8], vp(0), 1, 2, 8, 64, ctypes.c_float(0.125), None, None, vp(FAKE), ws,
                             vp(0)) == ga.GPT_ATTN_ERR_NULL
