"""The attention kernels' own abort path, exercised without a fault (debug build).

In libgpt_attn_debug.so the producer of CTA 0 can be told to skip one load: it neither issues the
copy nor announces it to its barrier, so nothing is in flight for it.  The consumer's bounded wait
then runs out, the CTA's roles leave their loops, the producer drains the loads it did issue, TMEM
is released, and gpt_attn_check reports GPT_ATTN_ERR_TIMEOUT.  The test then checks that the same
process still computes correct results (against the fp64 oracle), for the forward and the backward
kernel.  It runs in a fresh process with a short wait limit (GPT_ATTN_WAIT_TIMEOUT_MS), which the
library reads once per process.  The release library refuses the skip hook on the CPU."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
sys.path.insert(0, ROOT)
import numpy as np
import torch
import causal_attention_sdpa_b200 as ga
from causal_attention_sdpa_b200 import build
import oracle
from workloads import make_inputs

ga.LIB_PATH = build.build(debug=True)
L = ga.lib()

def parity(B, H, T, D, W, seed):
    q, k, v, do = make_inputs(B, H, T, D, seed=seed)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = ga.gpt_attn_fwd(qd, kd, vd, window=W)
    dq, dk, dv = ga.gpt_attn_bwd(qd, kd, vd, o, lse, dod, window=W)
    assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
    s = 1.0 / np.sqrt(D)
    ro, _ = oracle.attn_fwd(q, k, v, s, W)
    rdq, rdk, rdv, _ = oracle.attn_bwd(q, k, v, do, s, W)
    for g, r, tol in ((o, ro, 2e-2), (dq, rdq, 5e-2), (dk, rdk, 5e-2), (dv, rdv, 5e-2)):
        assert float(np.abs(g.float().cpu().double().numpy() - r).max()) <= tol

assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
parity(2, 3, 700, 64, 0, 1)                     # the debug build's checks stay quiet on valid work

q, k, v, do = (t.cuda() for t in make_inputs(4, 12, 1024, 64, seed=2))
assert L.gpt_attn_debug_skip_load(1) == ga.GPT_ATTN_OK
ga.gpt_attn_fwd(q, k, v)
assert ga.gpt_attn_check() == ga.GPT_ATTN_ERR_TIMEOUT
assert L.gpt_attn_debug_skip_load(0) == ga.GPT_ATTN_OK
parity(2, 12, 1000, 64, 200, 3)                 # same process, after the aborted launch

o, lse = ga.gpt_attn_fwd(q, k, v)
assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
assert L.gpt_attn_debug_skip_load(2) == ga.GPT_ATTN_OK
ga.gpt_attn_bwd(q, k, v, o, lse, do)
assert ga.gpt_attn_check() == ga.GPT_ATTN_ERR_TIMEOUT
assert L.gpt_attn_debug_skip_load(0) == ga.GPT_ATTN_OK
parity(2, 12, 1000, 64, 0, 4)
print("ABORT_PATH_OK")
'''


@pytest.mark.gpu
def test_skipped_load_times_out_and_context_survives():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, GPT_ATTN_WAIT_TIMEOUT_MS="200")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "ABORT_PATH_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


def test_release_library_refuses_the_skip_hook():
    import causal_attention_sdpa_b200 as ga
    from causal_attention_sdpa_b200 import build
    build.build()
    assert ga.lib().gpt_attn_debug_skip_load(1) == ga.GPT_ATTN_ERR_UNAVAILABLE
