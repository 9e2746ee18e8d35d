#!/usr/bin/env python
"""Benchmark of the 4-bit MoE layer on B200: prefill T=4096 tokens/s (the
reported value), decode T=1 us/token, both against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|zipf] [--no-cpu-baseline]

One step = one call of the layer (router, top-k, histogram/scan/permute,
gate/up GEMM with SwiGLU, down GEMM, shared expert, combine) over T=4096
tokens with weights and inputs resident in HBM.  Weights and activations are
drawn on the device from the synthetic recipe (bit_quantized_expert_route_b200
.synth); four layers and four activation sets are cycled so that nothing a
step reads is still in the 126 MB L2 from the previous step.

N > 1 (torchrun): every rank runs an independent replica of the layer on its
own GPU ("replicas only": the layer has no exchange step); the timed region is
bracketed by a barrier and a device synchronisation, and the slowest rank's
time is reported.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

T_PREFILL = 4096
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_LAUNCHES_PER_STEP = 7     # router, hist, scan, scatter, gate/up, down, combine
DECODE_LAUNCHES_PER_STEP = 6      # router, hist, scan, scatter, gate/up GEMV, down GEMV+combine
COMPUTE_DTYPE = "bf16"            # grouped GEMM operands (FP32 accumulation in tensor memory)
DOMINANT_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/gemm_tc.cu"
DOMINANT_KERNEL = "grouped_gemm_tc_kernel<true>"
DECODE_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/decode.cu"
DECODE_KERNEL = "decode_gateup_kernel"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("prefill", "zipf"), default="prefill")
    ap.add_argument("--decode-steps", type=int, default=400)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    return ap.parse_args(argv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def file_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_traffic(kernel: str, src_rel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged since."""
    sha = file_sha(src_rel)
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    pat = re.compile(r"^traffic_bytes_per_launch:\s+(\S+)\s+(\d+)\s+src_sha=(\w+)\s+workload=(\S+)", re.M)
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, name)) as f:
            for m in pat.finditer(f.read()):
                if m.group(1) == kernel and m.group(3) == sha:
                    return int(m.group(2)), m.group(4)
    return None


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu_index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in getattr(self, "lines", []):
            p = [v.strip() for v in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- helpers ---

def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(world):
    import torch
    import torch.distributed as dist
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_loop(fn, steps, world):
    """Device time of `steps` calls of fn(i) on the current stream, max over ranks (ms)."""
    import torch
    s = torch.cuda.current_stream()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier_sync(world)
    start.record(s)
    for i in range(steps):
        fn(i)
    stop.record(s)
    barrier_sync(world)
    return max_over_ranks(start.elapsed_time(stop), world)


# --------------------------------------------------------------- our arm ---

def run_ours(a):
    import torch
    from bit_quantized_expert_route_b200 import moe, synth

    world, rank, local = dist_setup(a.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    dims = synth.Dims()
    zipf = a.workload == "zipf"
    peaks, peak_src = load_peaks()

    # ---- prefill: 4 layers + 4 activation sets cycled (1.9 GB > L2) ----
    NL = 4
    layers = [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(1000 * rank + 1 + i, i, dims, dev, zipf))
              for i in range(NL)]
    xs = [synth.make_x_on_device(1000 * rank + 11 + i, T_PREFILL, dims.H, dev) for i in range(NL)]
    out = torch.empty_like(xs[0])
    ws = moe.alloc_workspace(layers[0], T_PREFILL, dev)

    def step(i):
        moe.moe_forward(layers[i % NL], xs[i % NL], out, ws)

    for i in range(a.warmup):
        step(i)
    with ClockSampler(torch.cuda.current_device()) as clk:
        total_ms = timed_loop(step, a.steps, world)
    clocks = clk.summary()
    ms_per_step = total_ms / a.steps
    value = world * T_PREFILL * a.steps / (total_ms / 1e3)

    # per-stage device times over the same workload (events between stages)
    stages = {}
    for i in range(a.steps):
        st = moe.moe_forward_profiled(layers[i % NL], xs[i % NL], out, ws)
        for k_, v in st.items():
            stages.setdefault(k_, []).append(v)
    stage_ms = {k_: statistics.mean(v) for k_, v in stages.items()}
    assert moe.moe_get_status(ws) == 0

    rows = T_PREFILL * dims.k + T_PREFILL
    flop_gateup = rows * 2 * 2 * dims.H * dims.I
    flop_layer = T_PREFILL * (dims.k + 1) * 6 * dims.H * dims.I + 2 * T_PREFILL * dims.H * dims.E
    achieved = flop_gateup / (stage_ms["gateup"] / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    tr = committed_traffic(DOMINANT_KERNEL, DOMINANT_KERNEL_SRC)
    roofline = {"kernel": DOMINANT_KERNEL, "bound": "tensor", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16 sustained",
                "algorithmic_per_launch": flop_gateup,
                "traffic": tr[0] if tr else None,
                "layer_frac": round(flop_layer / (ms_per_step / 1e3) / 1e12 / peak, 4)}

    # ---- e2e: the same call with host (pinned) buffers, copies inside ----
    xh = [xs[i].cpu().pin_memory() for i in range(NL)]
    oh = torch.empty_like(xh[0]).pin_memory()
    ws_h = ws

    def step_host(i):
        moe.moe_forward_host(layers[i % NL], xh[i % NL], oh, ws_h)

    for i in range(2):
        step_host(i)
    e2e_ms = timed_loop(step_host, a.steps, world)
    e2e = {"value": round(world * T_PREFILL * a.steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": T_PREFILL * dims.H * 2, "d2h_bytes_per_step": T_PREFILL * dims.H * 2}

    # ---- decode T=1: 40 resident layers cycled ----
    decode = None
    if not a.no_decode:
        del layers, xs
        torch.cuda.empty_cache()
        NLD = 40
        dl = [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(5000 * rank + l, l, dims, dev, False))
              for l in range(NLD)]
        dx = synth.make_x_on_device(7000 + rank, 64, dims.H, dev)
        dout = torch.empty((1, dims.H), dtype=torch.bfloat16, device=dev)
        dws = moe.alloc_workspace(dl[0], 1, dev)

        def dstep(i):
            moe.moe_forward(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws)

        for i in range(max(a.warmup, 40)):
            dstep(i)
        d_ms = timed_loop(dstep, a.decode_steps, world)
        us_tok = d_ms * 1e3 / a.decode_steps
        dst = {}
        for i in range(min(a.decode_steps, 200)):
            st = moe.moe_forward_profiled(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws)
            for k_, v in st.items():
                dst.setdefault(k_, []).append(v)
        dstage = {k_: statistics.median(v) for k_, v in dst.items()}
        expert_bytes = dims.I * dims.H // 2 + dims.I * (dims.H // 64) * 4          # one q-matrix [I,H]
        gateup_bytes = (dims.k + 1) * 2 * expert_bytes
        active_bytes = (dims.k + 1) * 3 * expert_bytes
        ach = gateup_bytes / (dstage["gateup"] / 1e3) / 1e9
        trd = committed_traffic(DECODE_KERNEL, DECODE_KERNEL_SRC)
        decode = {"workload": "decode T=1, 40 resident layers cycled (18.2 GB)", "us_per_token": round(us_tok, 3),
                  "active_expert_bytes": active_bytes,
                  "active_bytes_GBps": round(active_bytes / (us_tok / 1e6) / 1e9, 1),
                  "hbm_frac_active_bytes": round(active_bytes / (us_tok / 1e6) / 1e9 / peaks["hbm_gbs"], 4),
                  "stage_us": {k_: round(v * 1e3, 2) for k_, v in dstage.items()},
                  "roofline": {"kernel": DECODE_KERNEL, "bound": "hbm", "achieved": round(ach, 1),
                               "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                               "peak_source": f"{peak_src} HBM copy", "algorithmic_per_launch": gateup_bytes,
                               "traffic": trd[0] if trd else None},
                  "gpu_launches": DECODE_LAUNCHES_PER_STEP * a.decode_steps}
        del dl

    # ---- CPU baseline: the oracle on a bounded sample, rank 0 at N=1 ----
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline_sample(n_tokens=48, zipf=zipf)

    if rank == 0:
        line = {
            "metric": "MoE-layer tokens/s (prefill T=4096)",
            "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": COMPUTE_DTYPE, "data": "synthetic",
            "config": {"workload": f"prefill T=4096 {'zipf(1.2) router bias' if zipf else 'uniform routing'}",
                       "T": T_PREFILL, "H": dims.H, "E": dims.E, "k": dims.k, "I": dims.I, "I_shared": dims.I_s,
                       "quant": "affine 4-bit, group 64, bf16 scale/bias",
                       "l2": "4 layers + 4 activation sets cycled (1.9 GB read per cycle) > 126 MB L2",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": roofline,
            "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": PREFILL_LAUNCHES_PER_STEP * a.steps,
            "clocks": clocks,
            "decode": decode,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def cpu_baseline_sample(n_tokens: int, zipf: bool, seed: int = 0):
    """The CPU oracle (float64 NumPy, as it stands) on n_tokens of the prefill workload."""
    import numpy as np
    from bit_quantized_expert_route_b200 import synth
    from oracle import moe_ref
    dims = synth.Dims()
    lay = synth.make_layer(seed, 0, dims, zipf=zipf)
    x = synth.make_x(seed, T_PREFILL, dims.H)
    toks = np.arange(n_tokens)
    t0 = time.perf_counter()
    moe_ref.moe_layer(x, lay, dims.k, tokens=toks)
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": round(n_tokens / dt, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_tokens} of the 4096 prefill tokens (routing for all 4096, expert MLPs for the sample), "
                      f"NumPy float64, BLAS threads = {cores}", "seconds": round(dt, 2)}


# --------------------------------------------------------- reference arm ---

def run_reference(a):
    """The oracle as the reference arm: rank 0 only, a bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from bit_quantized_expert_route_b200 import synth
    from oracle import moe_ref
    dims = synth.Dims()
    zipf = a.workload == "zipf"
    lay = synth.make_layer(0, 0, dims, zipf=zipf)
    x = synth.make_x(0, T_PREFILL, dims.H)
    per_step = 4
    times = []
    for i in range(a.warmup + a.steps):
        toks = (np.arange(per_step) + per_step * i) % T_PREFILL
        t0 = time.perf_counter()
        moe_ref.moe_layer(x, lay, dims.k, tokens=toks)
        dt = time.perf_counter() - t0
        if i >= a.warmup:
            times.append(dt)
    total = sum(times)
    value = per_step * len(times) / total
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference",
        "metric": "MoE-layer tokens/s (prefill T=4096)", "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(total / len(times) * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"prefill T=4096 {'zipf(1.2) router bias' if zipf else 'uniform routing'}",
                   "T": T_PREFILL, "H": dims.H, "E": dims.E, "k": dims.k, "I": dims.I},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} tokens per step of the 4096 prefill tokens, NumPy float64"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    a = parse_args(argv)
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
    return 0


if __name__ == "__main__":
    sys.exit(main())
