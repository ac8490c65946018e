"""Host logic of bench.py that needs no GPU: the flop counts behind the metric, the workload
description, and when a recorded ncu DRAM-traffic figure may be reported."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench      # noqa: E402
import workloads  # noqa: E402


def test_flop_counts():
    # causal: fwd 2*B*H*T^2*D, fwd+bwd 3.5x that (bwd 2.5x)
    assert workloads.fwd_flops(64, 12, 1024, 64) == pytest.approx(2 * 64 * 12 * 1024 ** 2 * 64)
    assert workloads.fwd_bwd_flops(64, 12, 1024, 64) == pytest.approx(7 * 64 * 12 * 1024 ** 2 * 64)
    # windowed: 4*D per visible pair; T=8192, W=1024 has sum_i min(i+1, W) visible pairs per head
    pairs = sum(min(i + 1, 1024) for i in range(8192))
    assert workloads.fwd_flops(4, 6, 8192, 128, 1024) == pytest.approx(4 * 128 * pairs * 24)
    assert workloads.fwd_bwd_flops(4, 6, 8192, 128, 1024) / 1e9 == pytest.approx(338.3, rel=1e-3)


def test_l2_note_tells_resident_from_streamed_inputs():
    assert "larger than L2" in bench.l2_note(workloads.BY_INDEX[3])
    assert "fit in L2" in bench.l2_note(workloads.BY_INDEX[1])


def test_workload_config_names_the_workload():
    c = bench.workload_config(workloads.HEADLINE)
    for key in ("workload", "B", "H", "T", "D", "window", "scale", "seed", "l2", "flop_count"):
        assert key in c
    assert c["workload"] and "model" not in c


def test_recorded_traffic_is_gated_by_source_hash_and_shape(tmp_path, monkeypatch):
    w3 = workloads.BY_INDEX[3]
    rec = {"attn_bwd_kernel": {"source_hash": bench.kernel_source_hash(), "dram_bytes": 768e6, "units": 768,
                               "T": w3.T, "D": w3.D, "window": w3.window}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: rec["attn_bwd_kernel"]["source_hash"])
    assert bench.recorded_traffic("attn_bwd_kernel", w3) == pytest.approx(768e6)
    # same T, D, window, fewer heads: scaled by B*H
    assert bench.recorded_traffic("attn_bwd_kernel", workloads.BY_INDEX[2]) == pytest.approx(768e6 * 96 / 768)
    # another shape, another kernel, or changed sources: nothing reported
    assert bench.recorded_traffic("attn_bwd_kernel", workloads.BY_INDEX[5]) is None
    assert bench.recorded_traffic("attn_fwd_kernel", w3) is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0" * 16)
    assert bench.recorded_traffic("attn_bwd_kernel", w3) is None



def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    import shutil
    src = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc")
    dst = tmp_path / "causal_attention_sdpa_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = {k: bench.kernel_source_hash(k) for k in bench.KERNEL_SOURCES}
    f = dst / "schedule.h"
    text = f.read_text()
    f.write_text(text.replace("// Key tiles [lo, hi]", "// (reworded)  Key tiles [lo, hi]") + "\n/* note */\n")
    assert {k: bench.kernel_source_hash(k) for k in bench.KERNEL_SOURCES} == h0
    f.write_text(text.replace("constexpr int kTile = 128;", "constexpr int kTile = 64;"))
    for k in bench.KERNEL_SOURCES:
        assert bench.kernel_source_hash(k) != h0[k]
    # a change confined to another kernel's file leaves this kernel's key alone
    f.write_text(text)
    g = dst / "attn_bwd_d64.cuh"
    g.write_text(g.read_text().replace("namespace gpt_attn {", "namespace gpt_attn {\nconstexpr int kUnused = 1;", 1))
    assert bench.kernel_source_hash("attn_fwd_kernel") == h0["attn_fwd_kernel"]
    assert bench.kernel_source_hash("attn_bwd_kernel") != h0["attn_bwd_kernel"]


def test_kernel_sources_cover_the_kernels_includes():
    """Every csrc/ header that a profiled kernel's files include is part of its hash key."""
    import re
    csrc = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc")
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            text = open(os.path.join(csrc, f), encoding="utf-8").read()
            for inc in re.findall(r'#include "([^"]+)"', text):
                if os.path.exists(os.path.join(csrc, inc)):
                    assert inc in files, (kernel, f, inc)
