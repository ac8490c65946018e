"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module holds only input recipes and bookkeeping (shapes, seeds, flop and
byte counts).  It holds none of the attention arithmetic, so both the CUDA
library and the CPU oracle can be fed from it without sharing any of the
method's code.

Shapes stand in for the pages' workloads (no dataset or trained weights are
used; activations are N(0,1)):
  * tiny char-GPT (d_model 384, 6 heads, block 256) from "Un GPT desde cero +
    nanoGPT", Laboratorio L2.2;
  * GPT-2 124M (12 heads, head dim 64, context 1024) at micro-batch 8 and 64,
    from the GPT-2 lecture ("Раздел 2" uses 16x1024, the DDP section 64x1024);
  * GPT-2 large width (20 heads of 64) from the nanoGPT skill card's size table;
  * the modded-nanogpt README's sliding-window attention with QK-Norm
    (window 1024 on an 8192-token sequence, head dim 128, Q/K rows
    L2-normalised, scale 0.12).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int          # 1-based configuration number
    name: str
    B: int
    H: int
    T: int
    D: int
    scale: float
    window: int = 0     # <= 0: plain causal; W >= 1: key j visible iff i - W < j <= i
    qk_norm: bool = False

    @property
    def seed(self) -> int:
        return 1234 + self.index

    @property
    def shape(self):
        return (self.B, self.H, self.T, self.D)

    def describe(self) -> str:
        w = f", window {self.window}" if self.window > 0 else ""
        n = ", QK-normed" if self.qk_norm else ""
        return (f"{self.name}: B={self.B} H={self.H} T={self.T} D={self.D}, causal{w}, "
                f"scale {self.scale:g}{n}")


WORKLOADS = [
    Workload(1, "tiny char-GPT attention", 1, 6, 256, 64, 1.0 / 8),
    Workload(2, "GPT-2 124M attention, micro-batch 8", 8, 12, 1024, 64, 1.0 / 8),
    Workload(3, "GPT-2 124M attention, micro-batch 64", 64, 12, 1024, 64, 1.0 / 8),
    Workload(4, "GPT-2 large-width attention", 16, 20, 1024, 64, 1.0 / 8),
    Workload(5, "long-context sliding-window attention", 4, 6, 8192, 128, 0.12,
             window=1024, qk_norm=True),
]
BY_INDEX = {w.index: w for w in WORKLOADS}
HEADLINE = BY_INDEX[3]


def make_inputs(B, H, T, D, seed, qk_norm=False, device="cpu"):
    """Q, K, V, dO as contiguous bf16 [B, H, T, D].

    Drawn in that order from one CPU torch.Generator seeded with `seed`, as
    fp32 N(0,1), then rounded to bf16.  With qk_norm, Q and K rows are
    L2-normalised in fp32 before the rounding (input preparation for the
    QK-Norm workload; gradients then flow to the normalised Q and K).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, T, D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_norm:
        q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    out = [t.to(torch.bfloat16).contiguous() for t in (q, k, v, do)]
    if device != "cpu":
        out = [t.to(device) for t in out]
    return out


def workload_inputs(w: Workload, device="cpu"):
    return make_inputs(w.B, w.H, w.T, w.D, w.seed, w.qk_norm, device)


def visible_pairs(T: int, window: int = 0) -> int:
    """Number of (query, key) pairs with key j visible to query i, per head."""
    if window <= 0 or window >= T:
        return T * (T + 1) // 2
    W = window
    return W * (W + 1) // 2 + (T - W) * W


def fwd_flops(B, H, T, D, window=0) -> float:
    """Forward flops.  Plain causal: 2*B*H*T^2*D (the usual causal count).
    Windowed: the algorithmic count 4*D per visible pair (QK^T and PV)."""
    if window <= 0 or window >= T:
        return 2.0 * B * H * T * T * D
    return 4.0 * B * H * D * visible_pairs(T, window)


def fwd_bwd_flops(B, H, T, D, window=0) -> float:
    """Forward + backward flops: the backward counts 2.5x the forward."""
    return 3.5 * fwd_flops(B, H, T, D, window)


def min_bytes(B, H, T, D):
    """Minimum HBM bytes per pass (bf16 tensors, fp32 row statistics)."""
    n = B * H * T * D
    rows = B * H * T
    fwd = 2 * n * 4 + 4 * rows                 # read q,k,v ; write o ; write lse
    pre = 2 * n * 2 + 4 * rows                 # read o,dO ; write Delta
    bwd = 2 * n * 4 + 2 * n * 3 + 8 * rows     # read q,k,v,dO ; write dq,dk,dv ; read lse,Delta
    return fwd, pre, bwd


def sample_heads(B, H, n, seed=0):
    """A deterministic spread of n (b, h) pairs, always including the first and last head."""
    total = B * H
    if n >= total:
        return [(b, h) for b in range(B) for h in range(H)]
    idx = {0, total - 1}
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(total, generator=g).tolist()
    for p in perm:
        if len(idx) >= n:
            break
        idx.add(p)
    return [(i // H, i % H) for i in sorted(idx)]


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def doc_starts_from_lengths(lengths, T):
    """[T] int32: for each position, the first position of the document holding it, for documents
    of the given lengths laid end to end (the last one is cut at T)."""
    import numpy as np
    out = np.zeros(T, dtype=np.int32)
    pos = 0
    for n in lengths:
        if pos >= T:
            break
        n = int(n)
        if n < 1:
            raise ValueError("document lengths must be >= 1")
        out[pos:pos + n] = pos
        pos += n
    if pos < T:
        out[pos:] = pos
    return out


def make_doc_starts(B, T, seed, max_doc_len, min_doc_len=1):
    """[B, T] int32 document starts for B rows of T tokens packed with documents whose lengths are
    drawn uniformly from [min_doc_len, max_doc_len] (one CPU torch.Generator seeded with `seed`).
    Stands in for training batches aligned to end-of-document tokens with a maximum document
    length (the modded-nanogpt README's technique list); no text is involved."""
    import numpy as np
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    rows = []
    for _ in range(B):
        n = torch.randint(min_doc_len, max_doc_len + 1, (T,), generator=g).tolist()
        rows.append(doc_starts_from_lengths(n, T))
    return np.stack(rows).astype(np.int32)
