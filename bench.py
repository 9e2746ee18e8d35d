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
PREFILL_LAUNCHES_PER_STEP = 7     # router (+ segment counts), scan, scatter, gather, gate/up, down, combine
NOMINAL_BF16_TFLOPS = 2250.0      # B200 dense bf16 datasheet figure (context)
NOMINAL_HBM_GBS = 8000.0          # B200 HBM3e nominal bandwidth (context)
DECODE_LAUNCHES_PER_STEP = 3      # unfused: routing (router+top-k+sort), gate/up GEMV, down GEMV+combine
FUSED_DECODE_LAUNCHES_PER_STEP = 1   # T <= 2: the whole layer in one cooperative launch
COMPUTE_DTYPE = "bf16"            # grouped GEMM operands (FP32 accumulation in tensor memory)
DOMINANT_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/gemm_tc.cu"
DOMINANT_KERNEL = "grouped_gemm_tc_kernel<true>"
DECODE_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/decode.cu"
DECODE_KERNEL = "decode_gateup_kernel"
FUSED_DECODE_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/decode_fused.cu"
FUSED_DECODE_KERNEL = "decode_fused_kernel<1>"


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
    ap.add_argument("--decode-only", action="store_true", help="only the decode measurement (profiling)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass (profiling)")
    ap.add_argument("--no-stages", action="store_true", help="skip the per-stage traced pass (profiling)")
    ap.add_argument("--layers", type=int, default=4, help="prefill layers cycled")
    ap.add_argument("--decode-layers", type=int, default=40, help="decode layers cycled")
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

def dist_setup(n_gpus, backend: str = "nccl"):
    """One process per GPU: rank/world from the launcher's environment; the process group only
    carries the barriers and the max-over-ranks timing (replicas exchange no data)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(world, cuda: bool = True):
    import torch
    import torch.distributed as dist
    if cuda:
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def replica_seeds(rank: int, n_layers: int):
    """Each replica draws its own layers and inputs: (layer seeds, activation seeds)."""
    return [1000 * rank + 1 + i for i in range(n_layers)], [1000 * rank + 11 + i for i in range(n_layers)]


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
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

def prefill_phase(a, world, rank, dev, dims, zipf, peaks, peak_src):
    """K timed steps of the whole layer at T=4096, then per-stage times and e2e."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    NL = a.layers
    lseeds, xseeds = replica_seeds(rank, NL)
    layers = [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(lseeds[i], i, dims, dev, zipf))
              for i in range(NL)]
    xs = [synth.make_x_on_device(xseeds[i], T_PREFILL, dims.H, dev) for i in range(NL)]
    out = torch.empty_like(xs[0])
    ws = moe.alloc_workspace(layers[0], T_PREFILL, dev)

    def step(i):
        moe.moe_forward(layers[i % NL], xs[i % NL], out, ws)

    for i in range(a.warmup):
        step(i)
    total_ms = timed_loop(step, a.steps, world)
    res = {"ms_per_step": total_ms / a.steps, "value": whole_job_rate(T_PREFILL * a.steps, world, total_ms)}

    if not a.no_stages:
        # per-stage device times over the same workload (events between stages)
        stages = {}
        for i in range(a.steps):
            for k_, v in moe.moe_forward_profiled(layers[i % NL], xs[i % NL], out, ws).items():
                stages.setdefault(k_, []).append(v)
        stage_ms = {k_: statistics.mean(v) for k_, v in stages.items()}
        rows = T_PREFILL * dims.k + T_PREFILL
        flop_gateup = rows * 2 * 2 * dims.H * dims.I
        flop_layer = T_PREFILL * (dims.k + 1) * 6 * dims.H * dims.I + 2 * T_PREFILL * dims.H * dims.E
        # the "gateup" stage is the GEMM launch alone (the gather pass is its own stage)
        achieved = flop_gateup / (stage_ms["gateup"] / 1e3) / 1e12
        # the stage is one launch inside a sub-millisecond layer call, timed at full SM clock
        # (no power-cap reason in the clock samples): the burst figure is the fair peak
        peak = peaks["bf16_tflops"]
        tr = committed_traffic(DOMINANT_KERNEL, DOMINANT_KERNEL_SRC)
        res["roofline"] = {"kernel": DOMINANT_KERNEL, "bound": "tensor", "achieved": round(achieved, 2),
                           "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                           "peak_source": f"{peak_src} bf16 burst",
                           "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                           "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
                           "algorithmic_per_launch": flop_gateup,
                           "traffic": tr[0] if tr else None,
                           "layer_frac": round(flop_layer / (res["ms_per_step"] / 1e3) / 1e12 / peak, 4)}
        res["stage_ms"] = {k_: round(v, 4) for k_, v in stage_ms.items()}
    assert moe.moe_get_status(ws) == 0

    if not a.no_e2e:
        # the same call with host (pinned) buffers, copies inside the timed region
        xh = [xs[i].cpu().pin_memory() for i in range(NL)]
        oh = torch.empty_like(xh[0]).pin_memory()

        def step_host(i):
            moe.moe_forward_host(layers[i % NL], xh[i % NL], oh, ws)

        for i in range(2):
            step_host(i)
        sync_ms = timed_loop(step_host, a.steps, world)
        # streaming use: consecutive calls alternate two streams (each with its
        # own workspace and output buffer), so one call's host<->device copies
        # overlap the other's kernels; every step still copies its x in and
        # its result out inside the timed region
        ws2 = [ws, moe.alloc_workspace(layers[0], T_PREFILL, dev)]
        oh2 = [oh, torch.empty_like(oh).pin_memory()]
        streams = [torch.cuda.Stream(), torch.cuda.Stream()]

        def run_pipelined(n):
            cur = torch.cuda.current_stream()
            start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier_sync(world)
            start.record(cur)
            for st in streams:
                st.wait_stream(cur)
            for i in range(n):
                moe.moe_forward_host_async(layers[i % NL], xh[i % NL], oh2[i % 2], ws2[i % 2], stream=streams[i % 2])
            for st in streams:
                cur.wait_stream(st)
            stop.record(cur)
            barrier_sync(world)
            return max_over_ranks(start.elapsed_time(stop), world)

        run_pipelined(4)
        e2e_ms = run_pipelined(a.steps)
        for w_ in ws2:
            assert moe.moe_get_status(w_) == 0
        res["e2e"] = {"value": round(whole_job_rate(T_PREFILL * a.steps, world, e2e_ms), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": T_PREFILL * dims.H * 2, "d2h_bytes_per_step": T_PREFILL * dims.H * 2,
                      "how": "moe_forward_host_async, two streams alternating (copies overlap kernels)",
                      "blocking_call_value": round(whole_job_rate(T_PREFILL * a.steps, world, sync_ms), 1)}
    del layers, xs
    torch.cuda.empty_cache()
    return res


def decode_phase(a, world, rank, dev, dims, peaks, peak_src):
    """Decode T=1 through `decode_layers` resident layers, cycled (stream-launched and as a CUDA graph)."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    NLD = a.decode_layers
    dl = [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(5000 * rank + l, l, dims, dev, False))
          for l in range(NLD)]
    dx = synth.make_x_on_device(7000 + rank, 64, dims.H, dev)
    dout = torch.empty((1, dims.H), dtype=torch.bfloat16, device=dev)
    dws = moe.alloc_workspace(dl[0], 1, dev)

    def dstep(i):
        moe.moe_forward(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws)

    for i in range(max(a.warmup, NLD)):
        dstep(i)
    # one traced call tells which decode path runs (one fused launch or three)
    fused = len(moe.moe_forward_profiled(dl[0], dx[0:1], dout, dws)) == 1
    per_step = FUSED_DECODE_LAUNCHES_PER_STEP if fused else DECODE_LAUNCHES_PER_STEP
    d_ms = timed_loop(dstep, a.decode_steps, world)
    us_tok_stream = d_ms * 1e3 / a.decode_steps
    # the same layer calls captured once as a CUDA graph and replayed
    gstream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    gstream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(gstream):
        for l in range(NLD):
            dstep(l)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=gstream):
            for l in range(NLD):
                dstep(l)
    torch.cuda.synchronize()
    reps = max(1, a.decode_steps // NLD)
    for _ in range(2):
        graph.replay()
    g_ms = timed_loop(lambda i: graph.replay(), reps, world)
    us_tok = g_ms * 1e3 / (reps * NLD)
    del graph
    expert_bytes = dims.I * dims.H // 2 + dims.I * (dims.H // 64) * 4          # one q-matrix [I,H]
    gateup_bytes = (dims.k + 1) * 2 * expert_bytes
    active_bytes = (dims.k + 1) * 3 * expert_bytes
    res = {"workload": f"decode T=1, {NLD} resident layers cycled ({NLD * 0.456:.1f} GB)",
           "us_per_token": round(us_tok, 3), "us_per_token_stream_launched": round(us_tok_stream, 3),
           "timing": "us_per_token: the layer sequence as one CUDA graph, replayed; "
                     "stream-launched: one moe_forward call per layer",
           "active_expert_bytes": active_bytes,
           "active_bytes_GBps": round(active_bytes / (us_tok / 1e6) / 1e9, 1),
           "hbm_frac_active_bytes": round(active_bytes / (us_tok / 1e6) / 1e9 / peaks["hbm_gbs"], 4),
           "gpu_launches": per_step * reps * NLD}
    if not a.no_stages:
        dst = {}
        for i in range(min(a.decode_steps, 200)):
            for k_, v in moe.moe_forward_profiled(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws).items():
                dst.setdefault(k_, []).append(v)
        dstage = {k_: statistics.median(v) for k_, v in dst.items()}
        if fused:
            # the one launch moves the active experts' weights (and the router matrix)
            kern, src, alg, t_ms = FUSED_DECODE_KERNEL, FUSED_DECODE_KERNEL_SRC, active_bytes, dstage["decode_fused"]
        else:
            kern, src, alg, t_ms = DECODE_KERNEL, DECODE_KERNEL_SRC, gateup_bytes, dstage["gateup"]
        ach = alg / (t_ms / 1e3) / 1e9
        trd = committed_traffic(kern, src)
        res["stage_us"] = {k_: round(v * 1e3, 2) for k_, v in dstage.items()}
        res["roofline"] = {"kernel": kern, "bound": "hbm", "achieved": round(ach, 1),
                           "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                           "peak_source": f"{peak_src} HBM copy",
                           "frac_of_nominal": round(ach / NOMINAL_HBM_GBS, 4), "algorithmic_per_launch": alg,
                           "traffic": trd[0] if trd else None}
    del dl
    torch.cuda.empty_cache()
    return res


def run_ours(a):
    import torch
    from bit_quantized_expert_route_b200 import synth

    world, rank, local = dist_setup(a.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    dims = synth.Dims()
    zipf = a.workload == "zipf"
    peaks, peak_src = load_peaks()

    clk = ClockSampler(torch.cuda.current_device()).__enter__()   # sampled across every timed phase
    pre = {} if a.decode_only else prefill_phase(a, world, rank, dev, dims, zipf, peaks, peak_src)
    decode = None if a.no_decode else decode_phase(a, world, rank, dev, dims, peaks, peak_src)
    clk.__exit__(None, None, None)
    clocks = clk.summary()

    # ---- CPU baseline: the oracle on a bounded sample, rank 0 at N=1 ----
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline_sample(n_tokens=48, zipf=zipf)

    if rank == 0:
        line = {
            "metric": "MoE-layer tokens/s (prefill T=4096)",
            "value": round(pre["value"], 1) if pre else None, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(pre["ms_per_step"], 4) if pre else None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": COMPUTE_DTYPE, "data": "synthetic",
            "config": {"workload": f"prefill T=4096 {'zipf(1.2) router bias' if zipf else 'uniform routing'}",
                       "T": T_PREFILL, "H": dims.H, "E": dims.E, "k": dims.k, "I": dims.I, "I_shared": dims.I_s,
                       "quant": "affine 4-bit, group 64, bf16 scale/bias",
                       "l2": f"{a.layers} layers + {a.layers} activation sets cycled "
                             f"({a.layers * 0.47:.1f} GB read per cycle) > 126 MB L2",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": pre.get("roofline"),
            "stage_ms": pre.get("stage_ms"),
            "cpu_baseline": cpu,
            "e2e": pre.get("e2e"),
            "gpu_launches": PREFILL_LAUNCHES_PER_STEP * a.steps if pre else 0,
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
