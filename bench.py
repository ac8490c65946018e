#!/usr/bin/env python
"""Benchmark: causal attention forward + backward TFLOP/s on B200.

One step = one forward pass (gpt_attn_fwd) and one backward pass
(gpt_attn_bwd_delta -> gpt_attn_bwd_grads -> gpt_attn_bwd_dq_convert) over
one batch of the GPT-2 124M attention workload at micro-batch 64
(B=64, H=12, T=1024, D=64, causal, scale 1/8), seeded N(0,1) bf16 inputs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  `value` counts 7*B*H*T^2*D flops per step
(forward 2*B*H*T^2*D, backward 2.5x that) on every rank, divided by the
slowest rank's device time for the K timed steps.  Under torchrun each rank
drives one GPU with its own copy of the workload (weak scaling; attention has
no exchange step).  `--impl reference` times the fp64 CPU oracle on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402


METRIC = "causal attention fwd+bwd TFLOP/s on 1 B200 and % of dense bf16 peak"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=workloads.HEADLINE.index,
                    help="workload number (1-5); the default is the headline shape")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size B (smaller cases for profiler captures)")
    ap.add_argument("--decode", action="store_true",
                    help="time decode attention instead (one new query per sequence against a K/V cache; "
                         "GB/s of cache read against the HBM peak) and print its own JSON line")
    ap.add_argument("--prologue", action="store_true",
                    help="time the QK-Norm + rotary prologue (forward and backward) on q and k read from a "
                         "fused [B, T, 3, H, D] projection and print its own JSON line (GB/s against the HBM peak)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer, then read another, between timed steps (outside their "
                         "events) and sum the per-step times: a cold-L2 figure for workloads whose "
                         "inputs fit in L2")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(src: str) -> str:
    """Source text without comments and whitespace: what the compiler turns into kernels."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return re.sub(r"\s+", "", src)


# Device sources that define each profiled kernel (the file with its body and every header it
# includes from csrc/).  Host-side launch code is not part of the key; the committed summary
# records the launch configuration it was captured with.
KERNEL_SOURCES = {
    "attn_fwd_kernel": ("attn_fwd.cuh", "schedule.h", "sm100.cuh"),
    "attn_bwd_kernel": ("attn_bwd_d64.cuh", "attn_bwd.cuh", "attn_fwd.cuh", "schedule.h", "sm100.cuh"),
}


def kernel_source_hash(kernel: str = "attn_bwd_kernel") -> str:
    """Hash of the code (comments and layout excluded) of the device sources that define `kernel`,
    keying recorded ncu data: it changes exactly when that kernel's device code does."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, w):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current kernel
    source and on a workload of the same T, D and window (bytes scale with B*H)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or kernel not in KERNEL_SOURCES or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    if (e.get("T"), e.get("D"), e.get("window")) != (w.T, w.D, w.window):
        return None
    return e["dram_bytes"] * (w.B * w.H) / e["units"]


class NvmlClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML about every 2 ms while
    running, so that even a timed region of a few milliseconds is sampled from inside."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4))

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def __enter__(self):
        try:
            import threading

            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nvml = pynvml
            pr = torch.cuda.get_device_properties(self.device)
            h = pynvml.nvmlDeviceGetHandleByPciBusId(
                "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except Exception:
                        return
                    self._stop.wait(0.002)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2.0)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
        return False

    def summary(self):
        if not self.samples:
            return None
        bits = {name: getattr(self._nvml, attr, default) for name, attr, default in self.REASONS}
        reasons = sorted({name for _, r in self.samples for name, b in bits.items() if r & b})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, inside the timed region"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running (used when NVML
    cannot be read)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.samples = []
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8:
                self.samples.append(parts)
        return False

    def summary(self):
        if not getattr(self, "samples", None):
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [float(p[1]) for p in self.samples if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for p in self.samples if p[2].replace(".", "").isdigit()]
        reasons = sorted({names[i] for p in self.samples for i in range(4) if p[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """A per-rank time reduced to the job's: the slowest rank decides (every rank gets it)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step: float, world: int, steps: int, ms: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the max-over-ranks time (replicas, weak scaling)."""
    return flops_per_rank_step * world * steps / (ms / 1e3) / 1e12


def oracle_sample(w, q, k, v, do, n_heads):
    import oracle
    heads = workloads.sample_heads(w.B, w.H, n_heads, seed=1)
    sel = lambda t: __import__("torch").stack([t[b, h] for b, h in heads])
    qs, ks, vs, dos = sel(q), sel(k), sel(v), sel(do)
    t0 = time.perf_counter()
    oracle.attn_fwd(qs, ks, vs, w.scale, w.window)
    oracle.attn_bwd(qs, ks, vs, dos, w.scale, w.window)
    dt = time.perf_counter() - t0
    flops = workloads.fwd_bwd_flops(1, len(heads), w.T, w.D, w.window)
    return flops, dt, len(heads), oracle.max_threads()


def run_reference(args, w, rank):
    """The CPU oracle, timed on the host cores on a bounded sample of the workload."""
    if rank != 0:
        return
    import oracle
    q, k, v, do = workloads.workload_inputs(w)
    cores = oracle.max_threads()
    n = min(w.B * w.H, max(1, cores) * 4)
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, do, n)
    tot_f, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        f, t, nh, cores = oracle_sample(w, q, k, v, do, n)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = (f"{nh} of {w.B * w.H} heads (b,h) of the workload per step, fwd+bwd, fp64 oracle "
              f"(OpenMP over heads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def l2_note(w):
    mb = w.B * w.H * w.T * w.D * 2 / 1e6
    if 4 * mb > 126:
        return "inputs larger than L2 (4 x %.0f MB bf16 > 126 MB), no flush" % mb
    return "inputs fit in L2 (4 x %.1f MB bf16), no flush: warm-L2 timing" % mb


def workload_config(w):
    return {"workload": w.describe(), "B": w.B, "H": w.H, "T": w.T, "D": w.D, "window": w.window,
            "scale": w.scale, "qk_norm": w.qk_norm, "seed": w.seed,
            "l2": l2_note(w),
            "flop_count": ("7*B*H*T^2*D (fwd 2*B*H*T^2*D, bwd 2.5x)" if w.window <= 0 or w.window >= w.T
                           else "algorithmic: 4*D per visible pair fwd, 10*D bwd")}


class L2Flush:
    """Between timed calls: 256 MB written (a buffer larger than the 126 MB L2), then another
    256 MB read.  The read evicts the written lines, so their write-back to HBM happens here,
    outside the timed events, instead of inside the next timed call, which then starts with its
    data in HBM and a clean L2."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def run_decode(args):
    """Decode attention for generation: B sequences of a GPT-2 124M-shaped K/V cache (H=12, D=64,
    T_max=1024), each at full length, one new query each.  Memory-bound: reports the K/V bytes read
    per call over the call's device time against the HBM peak."""
    import torch
    import causal_attention_sdpa_b200 as ga
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    lines = []
    for B, H, T, D in ((64, 12, 1024, 64), (1, 12, 1024, 64), (16, 6, 8192, 128)):
        q4, k, v, _ = workloads.make_inputs(B, H, T, D, seed=77, device=dev)
        q = q4[:, :, -1].contiguous()
        lens = torch.full((B,), T, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, ga.gpt_attn_decode_workspace_bytes(B, H, T, D)), dtype=torch.uint8, device=dev)
        flush = L2Flush(dev)
        for _ in range(args.warmup):
            ga.gpt_attn_decode(q, k, v, lens, o=o, lse=lse, workspace=ws)
        assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
        times = []
        for _ in range(args.steps):
            flush()                              # cold L2: the caches come from HBM, as in generation
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ga.gpt_attn_decode(q, k, v, lens, o=o, lse=lse, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        nbytes = 2 * B * H * T * D * 2 + 2 * B * H * D * 2 + B * H * 4
        lines.append({"B": B, "H": H, "T_max": T, "D": D, "ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9,
                      "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]})
    print(json.dumps({"metric": "decode attention K/V-cache read bandwidth on 1 B200", "unit": "GB/s",
                      "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "l2": "256 MB written, then 256 MB read, between calls (outside the events)",
                      "steps": args.steps,
                      "warmup": args.warmup, "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"],
                      "cases": lines}), flush=True)


def run_prologue(args):
    """QK-Norm + rotary prologue of q and k (modded-nanogpt's modernised-architecture item) on the
    long-context shape (B=4 H=6 T=8192 D=128) and on the GPT-2 124M micro-batch-64 shape, inputs
    read in place from a fused [B, T, 3, H, D] projection.  Memory-bound: bytes that must move per
    call (forward: q, k read and written; backward: raw q, k and their output gradients read, the
    raw gradients written) over the call's device time against the HBM peak."""
    import torch
    import causal_attention_sdpa_b200 as ga
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    lines = []
    flush = L2Flush(dev)
    for B, H, T, D in ((4, 6, 8192, 128), (64, 12, 1024, 64)):
        g = torch.Generator(device=dev)
        g.manual_seed(99)
        qkv = torch.randn((B, T, 3, H, D), generator=g, device=dev).to(torch.bfloat16)
        qr, kr = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(2))
        qn, kn = (torch.empty((B, H, T, D), dtype=torch.bfloat16, device=dev) for _ in range(2))
        dq, dk = (torch.randn((B, H, T, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(2))
        grad = torch.empty_like(qkv)
        dqr, dkr = (grad[:, :, i].permute(0, 2, 1, 3) for i in range(2))
        row_bytes = B * H * T * D * 2
        calls = {
            "fwd": (lambda: ga.gpt_attn_qk_prologue_fwd(qr, kr, q_out=qn, k_out=kn), 2 * 2 * row_bytes),
            "bwd": (lambda: ga.gpt_attn_qk_prologue_bwd(qr, kr, dq, dk, dq_raw=dqr, dk_raw=dkr), 2 * 3 * row_bytes),
        }
        case = {"B": B, "H": H, "T": T, "D": D}
        for name, (fn, nbytes) in calls.items():
            for _ in range(args.warmup):
                fn()
            assert ga.gpt_attn_check() == ga.GPT_ATTN_OK
            times = []
            for _ in range(args.steps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            gbs = nbytes / (ms / 1e3) / 1e9
            case[name] = {"ms": ms, "bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        lines.append(case)
    print(json.dumps({"metric": "QK-Norm + rotary prologue bandwidth on 1 B200", "unit": "GB/s",
                      "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "l2": "256 MB written, then 256 MB read, between calls (outside the events)",
                      "steps": args.steps,
                      "warmup": args.warmup, "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"],
                      "cases": lines}), flush=True)


def main():
    args = parse_args()
    if args.decode:
        return run_decode(args)
    if args.prologue:
        return run_prologue(args)
    w = workloads.BY_INDEX[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, w, rank)

    import torch
    import causal_attention_sdpa_b200 as ga

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    ga.lib()

    # Host copies (pinned) for the end-to-end leg; device copies for the kernel leg.
    q_h, k_h, v_h, do_h = workloads.workload_inputs(w)
    q_h, k_h, v_h, do_h = (t.pin_memory() for t in (q_h, k_h, v_h, do_h))
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    B, H, T, D = w.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(ga.gpt_attn_bwd_workspace_bytes(B, H, T, D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ga.gpt_attn_fwd(q, k, v, scale=w.scale, window=w.window, o=o, lse=lse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        ga.gpt_attn_bwd_delta(o, lse, do, ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        ga.gpt_attn_bwd_grads(q, k, v, do, dk, dv, ws, scale=w.scale, window=w.window, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        ga.gpt_attn_bwd_dq_convert(dq, ws, scale=w.scale, stream=stream)
        if ev is not None:
            ev[4].record(stream)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    status = ga.gpt_attn_check(stream)
    if status != ga.GPT_ATTN_OK:
        raise RuntimeError(f"warm-up failed: {ga.status_string(status)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    flush = L2Flush(dev) if args.flush_l2 else None
    barrier()
    with ClockSampler(local) as clk:
        time.sleep(0.25)   # let the sampler start before the timed region
        barrier()
        with NvmlClockSampler(dev) as nclk:
            host_s = 0.0
            for i in range(args.steps):
                if flush is not None:
                    flush()
                h0 = time.perf_counter()
                step(evs[i])
                host_s += time.perf_counter() - h0
            barrier()
    status = ga.gpt_attn_check(stream)
    if status != ga.GPT_ATTN_OK:
        raise RuntimeError(f"timed steps failed: {ga.status_string(status)}")
    if flush is None:
        total_ms = evs[0][0].elapsed_time(evs[-1][4])
    else:   # the flushes between steps are not part of the work
        total_ms = sum(e[0].elapsed_time(e[4]) for e in evs)
    per_kernel = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
                  for i, name in enumerate(("attn_fwd_kernel", "attn_bwd_prep_kernel", "attn_bwd_kernel",
                                            "attn_dq_convert_kernel"))}
    step_median_ms = max_over_ranks(statistics.median(e[0].elapsed_time(e[4]) for e in evs), dist, dev)
    total_ms = max_over_ranks(total_ms, dist, dev)

    flops_step = workloads.fwd_bwd_flops(B, H, T, D, w.window)
    value = job_throughput(flops_step, world, args.steps, total_ms)

    # ---- end to end: pinned host buffers in and out through the public API, copies timed
    e2e = None
    if not args.no_e2e:
        # Every step copies its inputs in from pinned host memory and its results (O, lse, dQ, dK,
        # dV) back out.  Consecutive steps run on two streams with two sets of device and host
        # buffers, so the upload of step k+1 overlaps the compute and download of step k (PCIe
        # moves both directions at once); a user streaming batches through the library would do
        # the same.
        lanes = []
        for ln in range(2):
            if ln == 0:
                bufs = dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)
            else:
                bufs = dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                            do=torch.empty_like(do), o=torch.empty_like(o), lse=torch.empty_like(lse),
                            dq=torch.empty_like(dq), dk=torch.empty_like(dk), dv=torch.empty_like(dv),
                            ws=torch.empty_like(ws))
            bufs["host_out"] = [torch.empty_like(t, device="cpu").pin_memory()
                                for t in (o, lse, dq, dk, dv)]
            bufs["stream"] = torch.cuda.Stream(dev)
            lanes.append(bufs)
        e_steps = max(2, min(args.steps, 8))

        def e2e_step(i):
            b = lanes[i % 2]
            st = b["stream"]
            with torch.cuda.stream(st):
                for d_, h_ in ((b["q"], q_h), (b["k"], k_h), (b["v"], v_h), (b["do"], do_h)):
                    d_.copy_(h_, non_blocking=True)
                ga.gpt_attn_fwd(b["q"], b["k"], b["v"], scale=w.scale, window=w.window, o=b["o"],
                                lse=b["lse"], stream=st)
                ga.gpt_attn_bwd(b["q"], b["k"], b["v"], b["o"], b["lse"], b["do"], scale=w.scale,
                                window=w.window, dq=b["dq"], dk=b["dk"], dv=b["dv"], workspace=b["ws"],
                                stream=st)
                for h_, d_ in zip(b["host_out"], (b["o"], b["lse"], b["dq"], b["dk"], b["dv"])):
                    h_.copy_(d_, non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e0.record(lanes[0]["stream"])
        lanes[1]["stream"].wait_event(e0)
        for i in range(e_steps):
            e2e_step(i)
        for ln in range(2):
            ends[ln].record(lanes[ln]["stream"])
        barrier()
        e_ms = max_over_ranks(max(e0.elapsed_time(ev) for ev in ends), dist, dev)
        n_el = B * H * T * D
        e2e = {"value": job_throughput(flops_step, world, e_steps, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 4 * n_el * 2, "d2h_bytes_per_step": 4 * n_el * 2 + B * H * T * 4,
               "steps": e_steps, "pipelined": "two streams and buffer sets: the upload of step k+1 "
                                             "overlaps the compute and download of step k"}
        for ln in range(2):
            status = ga.gpt_attn_check(lanes[ln]["stream"])
            if status != ga.GPT_ATTN_OK:
                raise RuntimeError(f"end-to-end steps failed: {ga.status_string(status)}")
        del lanes

    if rank != 0:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    fwd_f = workloads.fwd_flops(B, H, T, D, w.window)
    bwd_f = flops_step - fwd_f
    kflops = {"attn_fwd_kernel": fwd_f, "attn_bwd_kernel": bwd_f}
    dominant = max(kflops, key=lambda n: per_kernel[n])
    achieved = kflops[dominant] / (per_kernel[dominant] / 1e3) / 1e12
    roofline = {"kernel": dominant, "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "peak_source": f"{peaks['source']} burst dense bf16",
                "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                      if peaks.get("bf16_tflops_sustained") else None),
                "traffic": recorded_traffic(dominant, w)}
    n_el = B * H * T * D
    prep_bytes = 2 * n_el * 2 + 4 * n_el + B * H * T * 4 * 3
    kernels = {n: {"ms": per_kernel[n]} for n in per_kernel}
    kernels["attn_fwd_kernel"]["tflops"] = fwd_f / (per_kernel["attn_fwd_kernel"] / 1e3) / 1e12
    kernels["attn_bwd_kernel"]["tflops"] = bwd_f / (per_kernel["attn_bwd_kernel"] / 1e3) / 1e12
    kernels["attn_bwd_prep_kernel"]["gbs"] = prep_bytes / (per_kernel["attn_bwd_prep_kernel"] / 1e3) / 1e9

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        import oracle  # the CPU baseline leg: oracle only
        cores = oracle.max_threads()
        f, t, nh, cores = oracle_sample(w, q_h, k_h, v_h, do_h, min(B * H, max(1, cores) * 24))
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{nh} of {B * H} heads (b,h) of the workload, fwd+bwd, fp64, {t:.1f} s wall"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "ms_per_step_median": step_median_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(workload_config(w), **({"l2": "L2 flushed between steps (256 MB "
                                                                    "written, then 256 MB read, outside "
                                                                    "the step events), sum of per-step "
                                                                    "times"}
                                                                    if flush is not None else {})),
        "pct_of_peak": value / world / peaks["bf16_tflops"],
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": 4 * args.steps, "clocks": nclk.summary() or clk.summary(),
        # CPU time to issue one step's four library calls (binding, C entry points, launches;
        # the CUDA event records in between included)
        "host_us_per_step": host_s / args.steps * 1e6,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
