"""Plain fp64 CPU oracle for causal scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library in
``causal_attention_sdpa_b200`` never does, and this package never imports it.

The arithmetic lives in ``oracle.c`` (plain row-by-row loops in double
precision, OpenMP over heads).  This module only compiles it with gcc and
marshals numpy arrays through ctypes.

Definition followed (restated, not copied): "NanoGPT Speedrun baseline",
section "El Mecanismo de Atencion" -- softmax(QK^T / sqrt(d_k)) V with
Attn_ij = 0 for j > i -- and, for the optional window, the long/short
sliding-window attention item of the modded-nanogpt README's technique list.
The backward pass is the exact gradient of sum(O * dO).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (-O2, OpenMP, strict IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        L = ctypes.c_long
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, L, L, L, ctypes.c_double, L,
                                        dp, dp, ctypes.c_int]
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, L, L, L, ctypes.c_double, L,
                                        dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lp = ctypes.POINTER(ctypes.c_long)
        lib.oracle_attn_fwd_masked.argtypes = [dp, dp, dp, L, L, L, L, ctypes.c_double, lp, L, lp,
                                               dp, dp, ctypes.c_int]
        lib.oracle_attn_fwd_masked.restype = ctypes.c_int
        lib.oracle_attn_bwd_masked.argtypes = [dp, dp, dp, dp, L, L, L, L, ctypes.c_double, lp, L, lp,
                                               dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_attn_bwd_masked.restype = ctypes.c_int
        lib.oracle_attn_decode.argtypes = [dp, dp, dp, lp, L, L, L, L, ctypes.c_double, L, dp, dp, ctypes.c_int]
        lib.oracle_attn_decode.restype = ctypes.c_int
        lib.oracle_qk_prologue_fwd.argtypes = [dp, L, L, L, ctypes.c_int, ctypes.c_double, dp]
        lib.oracle_qk_prologue_fwd.restype = ctypes.c_int
        lib.oracle_qk_prologue_bwd.argtypes = [dp, dp, L, L, L, ctypes.c_int, ctypes.c_double, dp]
        lib.oracle_qk_prologue_bwd.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _as_f64(x) -> np.ndarray:
    """Accept numpy arrays or torch CPU tensors (any float dtype) -> C-contiguous float64."""
    if hasattr(x, "detach"):  # torch tensor; bf16 widens exactly to fp32 and fp64
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def attn_fwd(q, k, v, scale: float, window: int = 0, nthreads: int = 0):
    """Forward pass.  q, k, v: [..., T, D].  Returns (O [..., T, D], lse [..., T]) in fp64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if not (q.shape == k.shape == v.shape) or q.ndim < 2:
        raise ValueError("q, k, v must share one shape [..., T, D]")
    *lead, T, D = q.shape
    NH = int(np.prod(lead)) if lead else 1
    o = np.zeros_like(q)
    lse = np.zeros(tuple(lead) + (T,), dtype=np.float64)
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), NH, T, D, float(scale),
                                 int(window), _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed with code {rc}")
    return o, lse


def attn_bwd(q, k, v, dO, scale: float, window: int = 0, nthreads: int = 0):
    """Backward pass of sum(O * dO).  Returns (dQ, dK, dV, Delta) in fp64."""
    q, k, v, dO = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dO)
    if not (q.shape == k.shape == v.shape == dO.shape) or q.ndim < 2:
        raise ValueError("q, k, v, dO must share one shape [..., T, D]")
    *lead, T, D = q.shape
    NH = int(np.prod(lead)) if lead else 1
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    delta = np.zeros(tuple(lead) + (T,), dtype=np.float64)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), NH, T, D,
                                 float(scale), int(window), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(delta), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv, delta



def _long_array(x, n=None):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int64).reshape(-1)).astype(ctypes.c_long)
    if n is not None and a.size != n:
        raise ValueError(f"expected {n} entries, got {a.size}")
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_long))


def attn_fwd_masked(q, k, v, scale: float, head_windows=None, window: int = 0, doc_start=None,
                    nthreads: int = 0):
    """Forward pass with a window per head and document boundaries.

    q, k, v: [B, H, T, D].  head_windows: H ints (window of head h in every batch row) or None
    for `window` everywhere.  doc_start: [B, T] ints, the first position of the document holding
    each token, or None for one document per row.  Returns (O [B,H,T,D], lse [B,H,T]) in fp64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if not (q.shape == k.shape == v.shape) or q.ndim != 4:
        raise ValueError("q, k, v must share one shape [B, H, T, D]")
    B, H, T, D = q.shape
    hw, hwp = _long_array(head_windows, H)
    ds, dsp = _long_array(doc_start, B * T)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, T), dtype=np.float64)
    rc = _load().oracle_attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), B, H, T, D, float(scale), hwp,
                                        int(window), dsp, _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_masked failed with code {rc}")
    return o, lse


def attn_bwd_masked(q, k, v, dO, scale: float, head_windows=None, window: int = 0, doc_start=None,
                    nthreads: int = 0):
    """Backward pass of sum(O * dO) under the mask of attn_fwd_masked.
    Returns (dQ, dK, dV, Delta) in fp64."""
    q, k, v, dO = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dO)
    if not (q.shape == k.shape == v.shape == dO.shape) or q.ndim != 4:
        raise ValueError("q, k, v, dO must share one shape [B, H, T, D]")
    B, H, T, D = q.shape
    hw, hwp = _long_array(head_windows, H)
    ds, dsp = _long_array(doc_start, B * T)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    delta = np.zeros((B, H, T), dtype=np.float64)
    rc = _load().oracle_attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), B, H, T, D, float(scale),
                                        hwp, int(window), dsp, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(delta),
                                        int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_masked failed with code {rc}")
    return dq, dk, dv, delta


def attn_decode(q, k_cache, v_cache, lens, scale: float, window: int = 0, nthreads: int = 0):
    """Decode: q [B, H, D] against cached keys/values [B, H, T_max, D]; sequence b has lens[b]
    tokens and its query is the last one.  Returns (O [B, H, D], lse [B, H]) in fp64."""
    q, k, v = _as_f64(q), _as_f64(k_cache), _as_f64(v_cache)
    if q.ndim != 3 or k.ndim != 4 or k.shape != v.shape or k.shape[:2] != q.shape[:2] or k.shape[3] != q.shape[2]:
        raise ValueError("q must be [B, H, D] and the caches [B, H, T_max, D]")
    B, H, T, D = k.shape
    ln, lnp = _long_array(lens, B)
    o = np.zeros_like(q)
    lse = np.zeros((B, H), dtype=np.float64)
    rc = _load().oracle_attn_decode(_ptr(q), _ptr(k), _ptr(v), lnp, B, H, T, D, float(scale), int(window),
                                    _ptr(o), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_decode failed with code {rc}")
    return o, lse


def qk_prologue_fwd(x, norm: bool = True, rope_base: float = 10000.0):
    """QK-Norm (unit L2 rows) then rotary embedding of half-split pairs by t * base^(-2i/D), on
    x [..., T, D] (token t = index along T).  rope_base <= 0: no rotation.  Returns fp64."""
    x = _as_f64(x)
    *lead, T, D = x.shape
    NH = int(np.prod(lead)) if lead else 1
    y = np.zeros_like(x)
    rc = _load().oracle_qk_prologue_fwd(_ptr(x), NH, T, D, int(bool(norm)), float(rope_base), _ptr(y))
    if rc != 0:
        raise RuntimeError(f"oracle_qk_prologue_fwd failed with code {rc}")
    return y


def qk_prologue_bwd(x, dy, norm: bool = True, rope_base: float = 10000.0):
    """Gradient of qk_prologue_fwd at x for the output gradient dy.  Returns fp64."""
    x, dy = _as_f64(x), _as_f64(dy)
    if x.shape != dy.shape:
        raise ValueError("x and dy must share one shape")
    *lead, T, D = x.shape
    NH = int(np.prod(lead)) if lead else 1
    dx = np.zeros_like(x)
    rc = _load().oracle_qk_prologue_bwd(_ptr(x), _ptr(dy), NH, T, D, int(bool(norm)), float(rope_base), _ptr(dx))
    if rc != 0:
        raise RuntimeError(f"oracle_qk_prologue_bwd failed with code {rc}")
    return dx
