#!/usr/bin/env python
"""GPT-2 124M training step on one B200 with three attention implementations.

The GPT-2 lecture's "Раздел 2" step-time table times one training step of GPT-2
124M (micro-batch 16 x 1024, bf16 autocast) on an A100 and reports 130 ms with
the attention written out (scores, causal mask, softmax, matmul) against 96 ms
with F.scaled_dot_product_attention(is_causal=True): same loss, shorter step.
This script redoes that comparison on B200 with a third arm, the gpt_attn
kernels through their autograd wrapper:

  naive     att = softmax(mask(q k^T / sqrt(d))) v, the T x T matrix materialised
  sdpa      torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
  gpt_attn  causal_attention_sdpa_b200.autograd.gpt_attention(q, k, v, out_layout="bthd"): the
            kernels read q, k, v as strided views of the fused projection and write O in the
            [B, T, H, D] layout the output projection reads (no transposes)

The model is a plain GPT-2 124M written here (12 layers, 12 heads, d_model 768,
context 1024, vocabulary padded to 50304, tied embedding and output head, GELU
tanh MLP), random-initialised, trained on seeded random token ids (no dataset).
One step = forward under bf16 autocast, cross-entropy loss, backward, fused
AdamW update.  Everything but the attention call is identical across arms; all
run eagerly (no torch.compile).

  python bench_gpt2.py [--steps K] [--warmup W] [--batch B] [--arms naive,sdpa,gpt_attn]

Prints one JSON line: median ms per step and tokens/s per arm, and the loss of
the first step per arm (identical inputs and initial weights).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import torch
import torch.nn as nn
import torch.nn.functional as F

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)


class Attention(nn.Module):
    def __init__(self, d_model, n_head, arm):
        super().__init__()
        self.n_head = n_head
        self.c_attn = nn.Linear(d_model, 3 * d_model)
        self.c_proj = nn.Linear(d_model, d_model)
        self.arm = arm

    def forward(self, x):
        B, T, C = x.shape
        H, D = self.n_head, C // self.n_head
        q, k, v = self.c_attn(x).split(C, dim=2)
        # heads become an extra batch dimension: [B, H, T, D]
        q, k, v = (t.view(B, T, H, D).transpose(1, 2) for t in (q, k, v))
        if self.arm == "naive":
            att = (q @ k.transpose(-2, -1)) * (1.0 / math.sqrt(D))
            blocked = torch.ones(T, T, dtype=torch.bool, device=x.device).triu(1)
            att = att.masked_fill(blocked, float("-inf")).softmax(dim=-1)
            y = att @ v
        elif self.arm == "sdpa":
            y = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        else:
            # the head views of the fused projection go in as they are; O comes back token-major
            from causal_attention_sdpa_b200.autograd import gpt_attention
            return self.c_proj(gpt_attention(q, k, v, out_layout="bthd").reshape(B, T, C))
        return self.c_proj(y.transpose(1, 2).reshape(B, T, C))


class Block(nn.Module):
    def __init__(self, d_model, n_head, arm):
        super().__init__()
        self.ln_1 = nn.LayerNorm(d_model)
        self.attn = Attention(d_model, n_head, arm)
        self.ln_2 = nn.LayerNorm(d_model)
        self.c_fc = nn.Linear(d_model, 4 * d_model)
        self.c_proj = nn.Linear(4 * d_model, d_model)

    def forward(self, x):
        x = x + self.attn(self.ln_1(x))
        return x + self.c_proj(F.gelu(self.c_fc(self.ln_2(x)), approximate="tanh"))


class GPT(nn.Module):
    def __init__(self, arm, n_layer=12, n_head=12, d_model=768, block=1024, vocab=50304):
        super().__init__()
        self.wte = nn.Embedding(vocab, d_model)
        self.wpe = nn.Embedding(block, d_model)
        self.blocks = nn.ModuleList(Block(d_model, n_head, arm) for _ in range(n_layer))
        self.ln_f = nn.LayerNorm(d_model)
        self.lm_head = nn.Linear(d_model, vocab, bias=False)
        self.lm_head.weight = self.wte.weight

    def forward(self, idx, targets):
        T = idx.shape[1]
        x = self.wte(idx) + self.wpe(torch.arange(T, device=idx.device))
        for b in self.blocks:
            x = b(x)
        logits = self.lm_head(self.ln_f(x))
        return F.cross_entropy(logits.float().reshape(-1, logits.shape[-1]), targets.reshape(-1))


def build(arm, seed=0, **kw):
    torch.manual_seed(seed)
    m = GPT(arm, **kw)
    for n, p in m.named_parameters():
        if p.dim() >= 2:
            nn.init.normal_(p, mean=0.0, std=0.02)
        elif n.endswith("bias"):
            nn.init.zeros_(p)
    return m


def time_arm(arm, args, idx, tgt):
    model = build(arm).cuda()
    opt = torch.optim.AdamW(model.parameters(), lr=6e-4, fused=True)

    def step():
        with torch.autocast("cuda", dtype=torch.bfloat16):
            loss = model(idx, tgt)
        loss.backward()
        opt.step()
        opt.zero_grad(set_to_none=True)
        return loss

    first = float(step().item())
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs:
        e0.record()
        step()
        e1.record()
    torch.cuda.synchronize()
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
    med = ms[len(ms) // 2]
    del model, opt
    torch.cuda.empty_cache()
    return {"ms_per_step": med, "tokens_per_s": idx.numel() / (med / 1e3), "first_loss": first}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--seq", type=int, default=1024)
    ap.add_argument("--arms", default="naive,sdpa,gpt_attn")
    args = ap.parse_args()
    g = torch.Generator().manual_seed(1234)
    idx = torch.randint(0, 50257, (args.batch, args.seq + 1), generator=g)
    x, y = idx[:, :-1].contiguous().cuda(), idx[:, 1:].contiguous().cuda()
    res = {a: time_arm(a, args, x, y) for a in args.arms.split(",")}
    line = {"metric": "GPT-2 124M training step (fwd+bwd+AdamW, bf16 autocast, eager) ms on 1 B200",
            "unit": "ms", "higher_is_better": False, "data": "synthetic token ids",
            "config": {"model": "GPT-2 124M (12 layers, 12 heads, d_model 768)", "batch": args.batch,
                       "seq_len": args.seq, "steps": args.steps, "warmup": args.warmup},
            "arms": res}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
