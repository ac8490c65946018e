"""Python binding of the gpt_attn C ABI (libgpt_attn.so, built in-tree for sm_100a).

Argument marshalling only: every step of the attention computation runs in the
CUDA kernels behind the C ABI.  PyTorch supplies device memory and streams.
There is no CPU or library fallback: if the shared library is missing or
cannot be loaded, importing the functions raises.

Entry points (same names as the C ABI, see include/gpt_attn.h):
  gpt_attn_fwd(q, k, v, scale=None, window=0, o=None, lse=None, stream=None) -> (o, lse)
  gpt_attn_bwd(q, k, v, o, lse, dO, scale=None, window=0, dq=None, dk=None, dv=None,
               workspace=None, stream=None) -> (dq, dk, dv)
  gpt_attn_bwd_workspace_bytes(B, H, T, D) -> int
  gpt_attn_check(stream=None) -> int
  gpt_attn_status_string(status) -> str
Tensors are bf16 contiguous [B, H, T, D] on the GPU; lse is fp32 [B, H, T].
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt_attn.so")

GPT_ATTN_OK = 0
GPT_ATTN_ERR_NULL = 1
GPT_ATTN_ERR_SHAPE = 2
GPT_ATTN_ERR_UNSUPPORTED_D = 3
GPT_ATTN_ERR_ALIGN = 4
GPT_ATTN_ERR_CUDA = 5
GPT_ATTN_ERR_TIMEOUT = 6
GPT_ATTN_ERR_WORKSPACE = 7
GPT_ATTN_ERR_UNAVAILABLE = 8
GPT_ATTN_ERR_BOUNDS = 9

EXPORTED = ("gpt_attn_fwd", "gpt_attn_bwd", "gpt_attn_bwd_workspace_bytes", "gpt_attn_bwd_delta",
            "gpt_attn_bwd_grads", "gpt_attn_bwd_dq_convert", "gpt_attn_check", "gpt_attn_status_string",
            "gpt_attn_debug_wait_timeout", "gpt_attn_bwd_noalloc", "gpt_attn_tmap_cache_stats",
            "gpt_attn_fwd_ex", "gpt_attn_bwd_ex", "gpt_attn_decode", "gpt_attn_decode_workspace_bytes",
            "gpt_attn_debug_skip_load", "gpt_attn_qk_prologue_fwd", "gpt_attn_qk_prologue_bwd")


class GptAttnStrides(ctypes.Structure):
    """The C ABI's gpt_attn_strides: element strides (batch, head, token) of a [b, h, t, d] tensor."""
    _fields_ = [("batch", ctypes.c_longlong), ("head", ctypes.c_longlong), ("token", ctypes.c_longlong)]


class GptAttnLayout(ctypes.Structure):
    """The C ABI's gpt_attn_layout: strides of q, k, v, o, dO, dq, dk, dv."""
    _fields_ = [(n, GptAttnStrides) for n in ("q", "k", "v", "o", "dO", "dq", "dk", "dv")]


class GptAttnMask(ctypes.Structure):
    """The C ABI's gpt_attn_mask: a window for every head, or per-head windows (host ints), and
    optional document starts (device int32 [B, T])."""
    _fields_ = [("window", ctypes.c_int), ("head_windows", ctypes.POINTER(ctypes.c_int)),
                ("doc_start", ctypes.c_void_p)]

_lib = None


class GptAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libgpt_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m causal_attention_sdpa_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.gpt_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.gpt_attn_fwd.restype = i
        L.gpt_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.gpt_attn_bwd.restype = i
        L.gpt_attn_bwd_delta.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
        L.gpt_attn_bwd_delta.restype = i
        L.gpt_attn_bwd_grads.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.gpt_attn_bwd_grads.restype = i
        L.gpt_attn_bwd_dq_convert.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
        L.gpt_attn_bwd_dq_convert.restype = i
        L.gpt_attn_bwd_workspace_bytes.argtypes = [i, i, i, i]
        L.gpt_attn_bwd_workspace_bytes.restype = sz
        L.gpt_attn_check.argtypes = [vp]
        L.gpt_attn_check.restype = i
        L.gpt_attn_status_string.argtypes = [i]
        L.gpt_attn_status_string.restype = ctypes.c_char_p
        L.gpt_attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.gpt_attn_bwd_noalloc.restype = i
        L.gpt_attn_tmap_cache_stats.argtypes = [ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_longlong),
                                                 ctypes.POINTER(ctypes.c_int)]
        L.gpt_attn_tmap_cache_stats.restype = None
        mp = ctypes.POINTER(GptAttnMask)
        lp = ctypes.POINTER(GptAttnLayout)
        L.gpt_attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, mp, lp, vp]
        L.gpt_attn_fwd_ex.restype = i
        L.gpt_attn_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, mp, lp, vp, sz, vp]
        L.gpt_attn_bwd_ex.restype = i
        L.gpt_attn_decode_workspace_bytes.argtypes = [i, i, i, i, i]
        L.gpt_attn_decode_workspace_bytes.restype = sz
        L.gpt_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, sz, vp]
        L.gpt_attn_decode.restype = i
        spp = ctypes.POINTER(GptAttnStrides)
        L.gpt_attn_qk_prologue_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, spp, vp]
        L.gpt_attn_qk_prologue_fwd.restype = i
        L.gpt_attn_qk_prologue_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, spp, vp]
        L.gpt_attn_qk_prologue_bwd.restype = i
        L.gpt_attn_debug_skip_load.argtypes = [i]
        L.gpt_attn_debug_skip_load.restype = i
        L.gpt_attn_debug_wait_timeout.argtypes = [i, vp]
        L.gpt_attn_debug_wait_timeout.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gpt_attn_status_string(int(status)).decode()


gpt_attn_status_string = status_string


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    # A plain int: the c_void_p argtypes convert it (and None to NULL) without a wrapper object.
    return t.data_ptr() if t is not None else None


def _check_bf16(name, t, shape):
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(shape)}")


def gpt_attn_fwd(q, k, v, scale=None, window=0, o=None, lse=None, stream=None):
    """Forward pass; returns (o, lse).  Asynchronous on `stream` (default: current)."""
    import torch
    B, H, T, D = q.shape
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(n, t, q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check_bf16("o", o, q.shape)
    rc = lib().gpt_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, T, D, float(scale),
                            int(window), _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_fwd")
    return o, lse


def gpt_attn_bwd_workspace_bytes(B, H, T, D) -> int:
    return int(lib().gpt_attn_bwd_workspace_bytes(int(B), int(H), int(T), int(D)))


def gpt_attn_bwd(q, k, v, o, lse, dO, scale=None, window=0, dq=None, dk=None, dv=None, workspace=None,
                 stream=None):
    """Backward pass of sum(O * dO); returns (dq, dk, dv).  Asynchronous on `stream`."""
    import torch
    B, H, T, D = q.shape
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _check_bf16(n, t, q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = gpt_attn_bwd_workspace_bytes(B, H, T, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().gpt_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk),
                            _ptr(dv), B, H, T, D, float(scale), int(window), _ptr(workspace), ws_bytes,
                            _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd")
    return dq, dk, dv


def gpt_attn_bwd_noalloc(q, k, v, o, lse, dO, scale=None, window=0, dq=None, dk=None, dv=None, stream=None):
    """gpt_attn_bwd with the library's built-in 32 MiB scratch instead of a workspace argument.

    For callers that must not allocate device memory when the backward pass runs.  Pass
    dq, dk and dv to keep this wrapper itself allocation-free.  Calls that overlap on the
    GPU share the scratch and race; the first call on a device should precede any capture.
    """
    import torch
    B, H, T, D = q.shape
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _check_bf16(n, t, q.shape)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    rc = lib().gpt_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk),
                                    _ptr(dv), B, H, T, D, float(scale), int(window), _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd_noalloc")
    return dq, dk, dv


def _mask(H, window=0, head_windows=None, doc_start=None):
    """A GptAttnMask (and the host array it points at, which must outlive the call)."""
    import torch
    hw = None
    if head_windows is not None:
        hw = (ctypes.c_int * H)(*[int(x) for x in head_windows])
        if len(head_windows) != H:
            raise ValueError(f"head_windows needs {H} entries")
    if doc_start is not None:
        if doc_start.dtype != torch.int32 or not doc_start.is_cuda or not doc_start.is_contiguous():
            raise ValueError("doc_start must be a contiguous CUDA int32 tensor [B, T]")
    m = GptAttnMask(int(window), ctypes.cast(hw, ctypes.POINTER(ctypes.c_int)) if hw is not None else None,
                    doc_start.data_ptr() if doc_start is not None else None)
    return m, hw


def _check_view(name, t, shape):
    """A bf16 CUDA tensor of the given [B, H, T, D] shape whose last dimension is contiguous."""
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or tuple(t.shape) != tuple(shape) or t.stride(3) != 1:
        raise ValueError(f"{name} must be a CUDA bf16 [B, H, T, D] view of shape {tuple(shape)} with stride 1 in D")


def _strides(t):
    return GptAttnStrides(t.stride(0), t.stride(1), t.stride(2))


_STRIDES24 = ctypes.c_longlong * 24


def _layout(**tensors):
    """A GptAttnLayout of the tensors' strides (given in the struct's order q, k, v, o, dO, dq, dk,
    dv), or None when they are all contiguous [B, H, T, D] (the C default)."""
    ts = list(tensors.values())
    if all(t.is_contiguous() for t in ts):
        return None
    v = []
    for t in ts:
        st = t.stride()
        v += (st[0], st[1], st[2])
    return GptAttnLayout.from_buffer(_STRIDES24(*v))     # one flat copy; the struct keeps it alive


def _byref(x):
    return ctypes.byref(x) if x is not None else None


def gpt_attn_fwd_ex(q, k, v, scale=None, window=0, head_windows=None, doc_start=None, o=None, lse=None,
                    stream=None):
    """Forward pass with per-head windows and/or document starts, on any [B, H, T, D] views whose D
    dimension is contiguous (e.g. the q, k, v columns of a fused [B, T, 3, H, D] projection, and an
    o that is a view of a [B, T, H, D] buffer); returns (o, lse)."""
    import torch
    B, H, T, D = q.shape
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_view(n, t, q.shape)
    if doc_start is not None and tuple(doc_start.shape) != (B, T):
        raise ValueError(f"doc_start must have shape {(B, T)}")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty((B, H, T, D), dtype=q.dtype, device=q.device) if o is None else o
    _check_view("o", o, q.shape)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
    m, keep = _mask(H, window, head_windows, doc_start)
    lay = _layout(q=q, k=k, v=v, o=o, dO=o, dq=o, dk=o, dv=o)
    rc = lib().gpt_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, T, D, float(scale),
                               ctypes.byref(m), _byref(lay), _stream_handle(stream))
    del keep
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_fwd_ex")
    return o, lse


def gpt_attn_bwd_ex(q, k, v, o, lse, dO, scale=None, window=0, head_windows=None, doc_start=None, dq=None,
                    dk=None, dv=None, workspace=None, stream=None):
    """Backward pass under the same mask as gpt_attn_fwd_ex, on [B, H, T, D] views with contiguous D
    (dq, dk, dv may be views into one [B, T, 3, H, D] gradient buffer); returns (dq, dk, dv)."""
    import torch
    B, H, T, D = q.shape
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _check_view(n, t, q.shape)
    if doc_start is not None and tuple(doc_start.shape) != (B, T):
        raise ValueError(f"doc_start must have shape {(B, T)}")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    mk = lambda: torch.empty((B, H, T, D), dtype=q.dtype, device=q.device)
    dq = mk() if dq is None else dq
    dk = mk() if dk is None else dk
    dv = mk() if dv is None else dv
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_view(n, t, q.shape)
    ws, nbytes = _ws(workspace, q)
    m, keep = _mask(H, window, head_windows, doc_start)
    lay = _layout(q=q, k=k, v=v, o=o, dO=dO, dq=dq, dk=dk, dv=dv)
    rc = lib().gpt_attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, H, T, D, float(scale), ctypes.byref(m), _byref(lay), _ptr(ws),
                               nbytes, _stream_handle(stream))
    del keep
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd_ex")
    return dq, dk, dv


def _ws(workspace, q):
    import torch
    B, H, T, D = q.shape
    if workspace is None:
        workspace = torch.empty(max(gpt_attn_bwd_workspace_bytes(B, H, T, D), 16), dtype=torch.uint8,
                                device=q.device)
    return workspace, workspace.numel() * workspace.element_size()


def gpt_attn_bwd_delta(o, lse, dO, workspace, stream=None):
    """Stage 1 of the backward pass (Delta, scaled lse, zeroed dQ accumulator)."""
    B, H, T, D = o.shape
    ws, nbytes = _ws(workspace, o)
    rc = lib().gpt_attn_bwd_delta(_ptr(o), _ptr(lse), _ptr(dO), B, H, T, D, _ptr(ws), nbytes,
                                  _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd_delta")
    return ws


def gpt_attn_bwd_grads(q, k, v, dO, dk, dv, workspace, scale=None, window=0, stream=None):
    """Stage 2 of the backward pass (dK, dV written; dQ accumulated in the workspace)."""
    B, H, T, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    ws, nbytes = _ws(workspace, q)
    rc = lib().gpt_attn_bwd_grads(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dk), _ptr(dv), B, H, T, D,
                                  float(scale), int(window), _ptr(ws), nbytes, _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd_grads")


def gpt_attn_bwd_dq_convert(dq, workspace, scale=None, stream=None):
    """Stage 3 of the backward pass (bf16 dQ = scale * the fp32 accumulator)."""
    B, H, T, D = dq.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    ws, nbytes = _ws(workspace, dq)
    rc = lib().gpt_attn_bwd_dq_convert(_ptr(dq), B, H, T, D, float(scale), _ptr(ws), nbytes,
                                       _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_bwd_dq_convert")


def gpt_attn_decode_workspace_bytes(B, H, T_max, D, window=0) -> int:
    return int(lib().gpt_attn_decode_workspace_bytes(int(B), int(H), int(T_max), int(D), int(window)))


def gpt_attn_decode(q, k_cache, v_cache, seq_lens, scale=None, window=0, o=None, lse=None, workspace=None,
                    stream=None):
    """Decode: q bf16 [B, H, D] against caches bf16 [B, H, T_max, D]; seq_lens int32 [B] on the
    device.  Returns (o [B, H, D], lse [B, H])."""
    import torch
    B, H, T, D = k_cache.shape
    _check_bf16("k_cache", k_cache, (B, H, T, D))
    _check_bf16("v_cache", v_cache, (B, H, T, D))
    _check_bf16("q", q, (B, H, D))
    if seq_lens.dtype != torch.int32 or not seq_lens.is_cuda or tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be a CUDA int32 tensor [B]")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    need = gpt_attn_decode_workspace_bytes(B, H, T, D, window)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = lib().gpt_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), _ptr(o), _ptr(lse), B, H,
                               T, D, float(scale), int(window), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_decode")
    return o, lse


def gpt_attn_qk_prologue_fwd(q_raw, k_raw, qk_norm=True, rope_base=10000.0, q_out=None, k_out=None, stream=None):
    """QK-Norm + rotary prologue: returns (q, k) bf16 [B, H, T, D] (contiguous unless q_out/k_out are
    given); q_raw, k_raw may be strided views (e.g. of a fused [B, T, 3, H, D] projection)."""
    import torch
    B, H, T, D = q_raw.shape
    mk = lambda: torch.empty((B, H, T, D), dtype=torch.bfloat16, device=q_raw.device)
    q_out = mk() if q_out is None else q_out
    k_out = mk() if k_out is None else k_out
    ts = [q_raw, k_raw, q_out, k_out]
    for n, t in zip(("q_raw", "k_raw", "q_out", "k_out"), ts):
        _check_view(n, t, q_raw.shape)
    arr = (GptAttnStrides * 4)(*[_strides(t) for t in ts])
    rc = lib().gpt_attn_qk_prologue_fwd(*[_ptr(t) for t in ts], B, H, T, D, int(bool(qk_norm)), float(rope_base),
                                        arr, _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_qk_prologue_fwd")
    return q_out, k_out


def gpt_attn_qk_prologue_bwd(q_raw, k_raw, dq_out, dk_out, qk_norm=True, rope_base=10000.0, dq_raw=None,
                             dk_raw=None, stream=None):
    """Gradient of the prologue: returns (dq_raw, dk_raw)."""
    import torch
    B, H, T, D = q_raw.shape
    mk = lambda: torch.empty((B, H, T, D), dtype=torch.bfloat16, device=q_raw.device)
    dq_raw = mk() if dq_raw is None else dq_raw
    dk_raw = mk() if dk_raw is None else dk_raw
    ts = [q_raw, k_raw, dq_out, dk_out, dq_raw, dk_raw]
    for n, t in zip(("q_raw", "k_raw", "dq_out", "dk_out", "dq_raw", "dk_raw"), ts):
        _check_view(n, t, q_raw.shape)
    arr = (GptAttnStrides * 6)(*[_strides(t) for t in ts])
    rc = lib().gpt_attn_qk_prologue_bwd(*[_ptr(t) for t in ts], B, H, T, D, int(bool(qk_norm)), float(rope_base),
                                        arr, _stream_handle(stream))
    if rc != GPT_ATTN_OK:
        raise GptAttnError(rc, "gpt_attn_qk_prologue_bwd")
    return dq_raw, dk_raw


def gpt_attn_check(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib().gpt_attn_check(_stream_handle(stream)))


def gpt_attn_tmap_cache_stats():
    """(hits, misses, entries) of the library's host-side tensor-map cache."""
    h, m, u = ctypes.c_longlong(0), ctypes.c_longlong(0), ctypes.c_int(0)
    lib().gpt_attn_tmap_cache_stats(ctypes.byref(h), ctypes.byref(m), ctypes.byref(u))
    return h.value, m.value, u.value


def gpt_attn_debug_wait_timeout(timeout_us: int, stream=None) -> int:
    return int(lib().gpt_attn_debug_wait_timeout(int(timeout_us), _stream_handle(stream)))
