#!/usr/bin/env python
"""Benchmark of the 4-bit MoE layer on B200 over the five synthetic workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|zipf] [--no-cpu-baseline] [--no-sweep] ...

The headline (the JSON line's "value") is prefill at T=4096 tokens with
uniform routing: one step = one call of the whole layer (router, top-k,
histogram/scan/permute, gate/up GEMM with SwiGLU, down GEMM, shared expert,
combine) with weights and inputs resident in HBM; four layers and four
activation sets are cycled so that nothing a step reads is still in the
126 MB L2 from the previous step.  The same line carries every other
workload under "workloads":

  tiny    T=16, H=256, E=16, k=2, I=128 (launch-latency bound)
  decode  T=1, H=2048, E=256, k=8, I=512, 40 resident layers cycled (HBM bound)
  prefill T=4096 uniform routing (the headline) and Zipf(1.2) skewed routing
  sweep   T in {1, 8, 64, 512, 4096, 16384} over a 40-layer stack joined by
          RMSNorm (moe_forward_stack), uniform and Zipf routing

each with tokens/s, us/token and the fraction of the roofline that bounds it,
and the float64 CPU oracle timed on the same host (full inputs; single-core
runs for the small workloads).

N > 1 (torchrun): every rank runs an independent replica on its own GPU
("replicas only": the layer has no exchange step); timed regions are
bracketed by a barrier and a device synchronisation, and the slowest rank's
time is reported.  Only rank 0 at N=1 runs the CPU oracle.
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
SWEEP_T = (1, 8, 64, 512, 4096, 16384)
ATTN_L = (4096, 32768, 131072)    # decode-attention context lengths (one sequence, 16 Q heads, 2 KV heads, D=256)
GDN_B = (1, 8, 64)                # recurrence batch sizes (16 key heads, 32 value heads, 128 x 128 FP32 state)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_LAUNCHES_PER_STEP = 7     # router (+ segment counts), scan, scatter, gather, gate/up, down, combine
UNFUSED_DECODE_LAUNCHES = 4       # routing (router+top-k+sort), gate/up GEMV, down GEMV, combine
FUSED_DECODE_LAUNCHES = 1         # T <= 3 (single layer): the whole layer in one cooperative launch
NOMINAL_BF16_TFLOPS = 2250.0      # B200 dense bf16 datasheet figure (context)
NOMINAL_HBM_GBS = 8000.0          # B200 HBM3e nominal bandwidth (context)
COMPUTE_DTYPE = "bf16"            # grouped GEMM operands (FP32 accumulation in tensor memory)
GEMM_SRC = "bit_quantized_expert_route_b200/csrc/gemm_tc.cu"
GATEUP_KERNEL = "grouped_gemm_tc_kernel<true>"
DOWN_KERNEL = "grouped_gemm_tc_kernel<false>"
DECODE_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/decode.cu"
DECODE_KERNEL = "mid_gateup_kernel"
FUSED_DECODE_KERNEL_SRC = "bit_quantized_expert_route_b200/csrc/decode_fused.cu"
FUSED_DECODE_KERNEL = "decode_fused_kernel<1>"
ATTN_SRC = "bit_quantized_expert_route_b200/csrc/attn.cu"
EPS = 1e-6


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("prefill", "zipf"), default="prefill",
                    help="routing of the headline prefill workload")
    ap.add_argument("--decode-steps", type=int, default=400)
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip every CPU-oracle timing")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-tiny", action="store_true")
    ap.add_argument("--no-attn", action="store_true", help="skip the decode-attention workload")
    ap.add_argument("--attn-L", type=str, default=",".join(str(n) for n in ATTN_L))
    ap.add_argument("--attn-reps", type=int, default=30, help="timed launches per attention point")
    ap.add_argument("--no-zipf-prefill", action="store_true", help="skip the skewed prefill workload")
    ap.add_argument("--decode-only", action="store_true", help="only the decode measurement (profiling)")
    ap.add_argument("--attn-only", action="store_true", help="only the decode-attention measurement (profiling)")
    ap.add_argument("--no-gdn", action="store_true", help="skip the Gated DeltaNet recurrence workload")
    ap.add_argument("--gdn-only", action="store_true", help="only the recurrence measurement (profiling)")
    ap.add_argument("--gdn-B", type=str, default=",".join(str(n) for n in GDN_B))
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass (profiling)")
    ap.add_argument("--e2e-streams", type=int, default=4,
                    help="streams (each with its own workspace and output buffer) that consecutive "
                         "host-buffer calls rotate over")
    ap.add_argument("--no-stages", action="store_true", help="skip the per-stage traced pass (profiling)")
    ap.add_argument("--layers", type=int, default=4, help="prefill layers cycled")
    ap.add_argument("--decode-layers", type=int, default=40, help="resident layers of the decode and sweep stacks")
    ap.add_argument("--sweep-T", type=str, default=",".join(str(t) for t in SWEEP_T))
    ap.add_argument("--sweep-reps", type=int, default=3, help="timed stack calls per sweep point")
    ap.add_argument("--no-mid", action="store_true", help="skip the single-layer mid-size decode workload")
    ap.add_argument("--mid-T", type=str, default="16,64", help="token counts of the mid-size decode workload")
    ap.add_argument("--oracle-sweep-T", type=str, default=",".join(str(t) for t in SWEEP_T),
                    help="sweep points at which the CPU oracle is timed (layer 0)")
    ap.add_argument("--probe-T", type=int, default=0,
                    help="profiling probe: only `--probe-calls` moe_forward calls of T tokens on two resident "
                         "layers (~0.9 GB), no timing, no JSON line")
    ap.add_argument("--probe-calls", type=int, default=4)
    ap.add_argument("--probe-stack", type=int, default=0,
                    help="with --probe-T: call moe_forward_stack on this many resident layers instead")
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


def committed_traffic(kernel: str, src_rel: str, workload: str | None = None):
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
                if m.group(1) == kernel and m.group(3) == sha and (workload is None or m.group(4) == workload):
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
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu_index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
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
        for ln in self.lines:
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


def capture_graph(fn):
    """fn() captured once into a CUDA graph on a side stream (after one eager call there)."""
    import torch
    gstream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    gstream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(gstream):
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=gstream):
            fn()
    torch.cuda.synchronize()
    return graph


def layer_flops(dims, T: int) -> int:
    """Algorithmic FLOPs of one layer call: (k + 1) SwiGLU experts per token plus the router
    and the shared-gate row."""
    return T * (dims.k + 1) * 6 * dims.H * dims.I + 2 * T * dims.H * (dims.E + 1)


def expert_bytes(dims) -> int:
    """Packed codes plus bf16 scales and biases of one expert's three q-matrices."""
    one = dims.I * dims.H // 2 + dims.I * (dims.H // 64) * 4      # one q-matrix [I, H] (or [H, I])
    return 3 * one


def tensor_roofline(kernel, flop, ms, peaks, peak_src, sustained: bool, traffic=None):
    achieved = flop / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    return {"kernel": kernel, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'}",
            "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
            "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "algorithmic_per_launch": int(flop), "traffic": traffic}


def hbm_roofline(kernel, nbytes, ms, peaks, peak_src, traffic=None):
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} HBM copy",
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4), "algorithmic_per_launch": int(nbytes),
            "traffic": traffic}


# ---------------------------------------------------- prefill (CFG2, CFG3) ---

def prefill_phase(a, world, rank, dev, dims, zipf, peaks, peak_src, e2e: bool):
    """K timed steps of the whole layer at T=4096, then per-stage times and (optionally) e2e."""
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
    res = {"workload": f"prefill T={T_PREFILL}, {'Zipf(1.2) router bias' if zipf else 'uniform routing'}, "
                       f"{NL} layers + activation sets cycled",
           "ms_per_step": round(total_ms / a.steps, 4),
           "value": whole_job_rate(T_PREFILL * a.steps, world, total_ms),
           "us_per_token": round(total_ms / a.steps * 1e3 / T_PREFILL, 5)}
    flop_layer = layer_flops(dims, T_PREFILL)
    res["layer_roofline"] = tensor_roofline("whole layer (7 launches)", flop_layer, total_ms / a.steps, peaks,
                                            peak_src, sustained=False)
    if not a.no_stages:
        stages = {}
        for i in range(a.steps):
            for k_, v in moe.moe_forward_profiled(layers[i % NL], xs[i % NL], out, ws).items():
                stages.setdefault(k_, []).append(v)
        stage_ms = {k_: statistics.mean(v) for k_, v in stages.items()}
        rows = T_PREFILL * dims.k + T_PREFILL
        flop_gateup = rows * 2 * 2 * dims.H * dims.I
        flop_down = rows * 2 * dims.H * dims.I
        wl = "prefill_T4096_zipf" if zipf else "prefill_T4096_uniform"
        tr_g = committed_traffic(GATEUP_KERNEL, GEMM_SRC, wl)
        tr_d = committed_traffic(DOWN_KERNEL, GEMM_SRC, wl)
        # each GEMM stage is one launch inside a sub-millisecond layer call, timed at full SM
        # clock: the burst figure is the fair peak
        res["roofline"] = tensor_roofline(GATEUP_KERNEL, flop_gateup, stage_ms["gateup"], peaks, peak_src,
                                          sustained=False, traffic=tr_g[0] if tr_g else None)
        res["down_roofline"] = tensor_roofline(DOWN_KERNEL, flop_down, stage_ms["down"], peaks, peak_src,
                                               sustained=False, traffic=tr_d[0] if tr_d else None)
        res["stage_ms"] = {k_: round(v, 4) for k_, v in stage_ms.items()}
    assert moe.moe_get_status(ws) == 0

    if e2e and not a.no_e2e:
        # the same call with host (pinned) buffers, copies inside the timed region
        xh = [xs[i].cpu().pin_memory() for i in range(NL)]
        oh = torch.empty_like(xh[0]).pin_memory()

        def step_host(i):
            moe.moe_forward_host(layers[i % NL], xh[i % NL], oh, ws)

        for i in range(2):
            step_host(i)
        sync_ms = timed_loop(step_host, a.steps, world)
        # streaming use: consecutive calls rotate over S streams (each with its
        # own workspace and output buffer), so one call's host<->device copies
        # overlap the others' kernels; every step still copies its x in and
        # its result out inside the timed region.  One stream runs its call's
        # copy in, layer and copy out in order (~0.33 + 0.43 + 0.33 ms at
        # T=4096), so S = 2 holds a step to about half of that chain; from
        # S = 3 the copies hide behind the kernels (S = 1, 2, 3, 4, 6: 1.06,
        # 0.578, 0.459, 0.450, 0.459 ms per step against 0.425 device-only).
        S = max(1, a.e2e_streams)
        ws2 = [ws] + [moe.alloc_workspace(layers[0], T_PREFILL, dev) for _ in range(S - 1)]
        oh2 = [oh] + [torch.empty_like(oh).pin_memory() for _ in range(S - 1)]
        streams = [torch.cuda.Stream() for _ in range(S)]

        def run_pipelined(n):
            cur = torch.cuda.current_stream()
            start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier_sync(world)
            start.record(cur)
            for st in streams:
                st.wait_stream(cur)
            for i in range(n):
                moe.moe_forward_host_async(layers[i % NL], xh[i % NL], oh2[i % S], ws2[i % S], stream=streams[i % S])
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
                      "how": f"moe_forward_host_async, {S} streams in rotation (copies overlap kernels)",
                      "blocking_call_value": round(whole_job_rate(T_PREFILL * a.steps, world, sync_ms), 1)}
    del layers, xs
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------- decode (CFG1) ---

def make_stack_layers(a, rank, dev, dims):
    """The 40 resident layers (uniform routing) shared by the decode and sweep workloads."""
    from bit_quantized_expert_route_b200 import moe, synth
    return [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(5000 * rank + l, l, dims, dev, False))
            for l in range(a.decode_layers)]


def decode_phase(a, world, rank, dev, dims, peaks, peak_src, dl):
    """Decode T=1 through the resident layers, cycled (stream-launched and as a CUDA graph)."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    NLD = len(dl)
    dx = synth.make_x_on_device(7000 + rank, 64, dims.H, dev)
    dout = torch.empty((1, dims.H), dtype=torch.bfloat16, device=dev)
    dws = moe.alloc_workspace(dl[0], 1, dev)

    def dstep(i):
        moe.moe_forward(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws)

    for i in range(max(a.warmup, NLD)):
        dstep(i)
    fused = len(moe.moe_forward_profiled(dl[0], dx[0:1], dout, dws)) == 1
    per_step = FUSED_DECODE_LAUNCHES if fused else UNFUSED_DECODE_LAUNCHES
    d_ms = timed_loop(dstep, a.decode_steps, world)
    us_tok_stream = d_ms * 1e3 / a.decode_steps
    graph = capture_graph(lambda: [dstep(l) for l in range(NLD)])
    reps = max(1, a.decode_steps // NLD)
    for _ in range(2):
        graph.replay()
    g_ms = timed_loop(lambda i: graph.replay(), reps, world)
    us_tok = g_ms * 1e3 / (reps * NLD)
    del graph
    active = (dims.k + 1) * expert_bytes(dims)
    res = {"workload": f"decode T=1, {NLD} resident layers cycled ({NLD * 0.456:.1f} GB)",
           "us_per_token": round(us_tok, 3), "tokens_per_s": round(1e6 / us_tok, 1),
           "us_per_token_stream_launched": round(us_tok_stream, 3),
           "timing": "us_per_token: the layer sequence as one CUDA graph, replayed; "
                     "stream-launched: one moe_forward call per layer",
           "active_expert_bytes": active,
           "active_bytes_GBps": round(active / (us_tok / 1e6) / 1e9, 1),
           "hbm_frac_active_bytes": round(active / (us_tok / 1e6) / 1e9 / peaks["hbm_gbs"], 4),
           "gpu_launches": per_step * reps * NLD}
    if not a.no_stages:
        dst = {}
        for i in range(min(a.decode_steps, 200)):
            for k_, v in moe.moe_forward_profiled(dl[i % NLD], dx[i % 64:i % 64 + 1], dout, dws).items():
                dst.setdefault(k_, []).append(v)
        dstage = {k_: statistics.median(v) for k_, v in dst.items()}
        if fused:
            kern, src, alg, t_ms = FUSED_DECODE_KERNEL, FUSED_DECODE_KERNEL_SRC, active, dstage["decode_fused"]
        else:
            kern, src, alg, t_ms = DECODE_KERNEL, DECODE_KERNEL_SRC, (dims.k + 1) * expert_bytes(dims) * 2 // 3, \
                dstage["gateup"]
        trd = committed_traffic(kern, src)
        res["stage_us"] = {k_: round(v * 1e3, 2) for k_, v in dstage.items()}
        res["roofline"] = hbm_roofline(kern, alg, t_ms, peaks, peak_src, traffic=trd[0] if trd else None)
    assert moe.moe_get_status(dws) == 0
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------- mid-size decode (single layers) ---

def decode_mid_phase(a, world, rank, dev, dims, peaks, peak_src, dl):
    """Single-layer calls at 4 <= T <= 128 (the mid-size decode path) through the resident layers, as a CUDA
    graph of one call per layer; HBM roofline over the distinct experts each call's routing touches."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    NL = len(dl)
    out_rows = {}
    for T in [int(t) for t in a.mid_T.split(",") if t]:
        x = synth.make_x_on_device(9000 + 10 * T + rank, T, dims.H, dev)
        out = torch.empty_like(x)
        ws = moe.alloc_workspace(dl[0], T, dev)
        stages = moe.moe_forward_profiled(dl[0], x, out, ws)
        graph = capture_graph(lambda: [moe.moe_forward(dl[l], x, out, ws) for l in range(NL)])
        graph.replay()
        reps = max(1, a.sweep_reps)
        g_ms = timed_loop(lambda i: graph.replay(), reps, world) / reps
        del graph
        # the distinct experts of each layer's routing of x (+ the shared expert)
        r = moe.Routing(T, dims.E, dims.k, dev)
        distinct = 0
        for l in range(NL):
            moe.moe_route(dl[l], x, r, ws)
            distinct += int((r.counts > 0).sum().item()) + 1
        assert moe.moe_get_status(ws) == 0
        layer_ms = g_ms / NL
        out_rows[str(T)] = {
            "layer_us": round(layer_ms * 1e3, 3), "us_per_token": round(layer_ms * 1e3 / T, 4),
            "tokens_per_s": round(whole_job_rate(T, world, layer_ms), 1),
            "kernel_set": "mid-size decode" if len(stages) == len(moe.MID_DECODE_STAGES) else
                          ("fused decode" if len(stages) == 1 else "tensor-core"),
            "distinct_experts_per_layer": round(distinct / NL, 2),
            "roofline": hbm_roofline("whole layer (router, gate/up, down, combine)", distinct * expert_bytes(dims),
                                     g_ms, peaks, peak_src)}
    torch.cuda.empty_cache()
    return {"workload": f"single-layer calls (moe_forward), {NL} distinct resident layers, random inputs "
                        f"(uniform routing), H={dims.H}, E={dims.E}, k={dims.k}, I={dims.I}",
            "timing": "one call per layer captured as one CUDA graph and replayed; per-layer time = graph time / layers",
            "roofline_note": "HBM bytes = the distinct experts each call's routing touches (routed + shared) x "
                             "1,769,472 B, over the whole layer's time",
            "points": out_rows}


# ------------------------------------------------------------ sweep (CFG4) ---

def sweep_phase(a, world, rank, dev, dims, peaks, peak_src, dl):
    """40-layer stacks (moe_forward_stack: layers joined by RMSNorm) at every T, uniform routing on
    even seeds and the Zipf(1.2) bias on odd seeds; stream-launched and CUDA-graph timings."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    NL = len(dl)
    Ts = [int(t) for t in a.sweep_T.split(",") if t]
    zl = [moe.MoELayer.from_tensors(dims, {**L.tensors,
                                           "router_bias": synth.zipf_bias_on_device(5000 * rank + l, l, dims, dev)})
          for l, L in enumerate(dl)]
    stacks = {"uniform": moe.LayerStack(dl), "zipf": moe.LayerStack(zl)}
    ws = moe.alloc_workspace(dl[0], max(Ts), dev)
    out_rows = {}
    for T in Ts:
        row = {}
        for seed, (kind, stack) in enumerate(stacks.items()):
            x = synth.make_x_on_device(8000 + 10 * T + seed, T, dims.H, dev)
            out = torch.empty_like(x)

            def call():
                moe.moe_forward_stack(stack, x, out, ws, eps=EPS)

            call()
            reps = a.sweep_reps if T >= 512 else 4 * a.sweep_reps
            s_ms = timed_loop(lambda i: call(), reps, world) / reps
            graph = capture_graph(call)
            graph.replay()
            g_ms = timed_loop(lambda i: graph.replay(), reps, world) / reps
            del graph
            assert moe.moe_get_status(ws) == 0
            layer_ms = g_ms / NL
            ent = {"seed": seed, "stack_ms": round(g_ms, 4), "stack_ms_stream_launched": round(s_ms, 4),
                   "layer_us": round(layer_ms * 1e3, 3), "us_per_token_per_layer": round(layer_ms * 1e3 / T, 5),
                   "tokens_per_s_per_layer": round(whole_job_rate(T, world, layer_ms), 1),
                   "tokens_per_s_stack": round(whole_job_rate(T, world, g_ms), 1)}
            if T <= 64:
                # HBM bound: the distinct experts each layer touches (routing of the stack's own
                # activations, read back from a traced run)
                trace = torch.empty((NL, 2, T, dims.H), dtype=torch.bfloat16, device=dev)
                moe.moe_forward_stack(stack, x, out, ws, trace=trace, eps=EPS)
                r = moe.Routing(T, dims.E, dims.k, dev)
                rws = moe.alloc_workspace(dl[0], T, dev)
                distinct = []
                for l in range(NL):
                    moe.moe_route(stack.layers[l], trace[l, 0].contiguous(), r, rws)
                    distinct.append(int((r.counts > 0).sum().item()) + 1)     # + the shared expert
                nbytes = sum(distinct) * expert_bytes(dims)
                ent["distinct_experts_per_layer"] = round(sum(distinct) / NL, 2)
                ent["roofline"] = hbm_roofline("40-layer stack", nbytes, g_ms, peaks, peak_src)
                del trace
            else:
                ent["roofline"] = tensor_roofline("40-layer stack", NL * layer_flops(dims, T), g_ms, peaks,
                                                  peak_src, sustained=True)
            row[kind] = ent
        out_rows[str(T)] = row
    torch.cuda.empty_cache()
    return {"workload": f"{NL}-layer stack joined by RMSNorm (moe_forward_stack), H={dims.H}, E={dims.E}, "
                        f"k={dims.k}, I={dims.I}; seed 0 uniform routing, seed 1 Zipf(1.2) router bias",
            "timing": "stack_ms: one stack call captured as a CUDA graph and replayed; stream-launched alongside; "
                      "18.2 GB of resident weights, so nothing is L2-resident between calls",
            "roofline_note": "T <= 64: HBM bytes = distinct experts per layer (routed + shared) x 1,769,472 B; "
                             "T >= 512: layer FLOPs vs the sustained bf16 peak (a stack call is a long step)",
            "points": out_rows}


# ------------------------------------------------------------- tiny (CFG0) ---

def tiny_phase(a, world, dev):
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    dims = synth.Dims.tiny()
    T = 16
    L = moe.MoELayer.from_synth(synth.make_layer(0, 0, dims), dev)
    x = moe._bits_tensor(synth.make_x(0, T, dims.H), dev)
    out = torch.empty_like(x)
    ws = moe.alloc_workspace(L, T, dev)
    n = 100
    graph = capture_graph(lambda: [moe.moe_forward(L, x, out, ws) for _ in range(n)])
    graph.replay()
    g_ms = timed_loop(lambda i: graph.replay(), 5, world) / (5 * n)
    s_ms = timed_loop(lambda i: moe.moe_forward(L, x, out, ws), 200, world) / 200
    del graph
    assert moe.moe_get_status(ws) == 0
    return {"workload": "tiny layer T=16, H=256, E=16, k=2, I=I_s=128 (mid-size decode path)",
            "layer_us": round(g_ms * 1e3, 3), "layer_us_stream_launched": round(s_ms * 1e3, 3),
            "tokens_per_s": round(whole_job_rate(T, world, g_ms), 1),
            "bound": "launch latency (4 dependent launches: router, gate/up, down, combine; ~1 MB of weights)"}


# --------------------------------------------------- decode attention ---

CYCLE_BYTES = 320 << 20   # distinct inputs cycled per timed pass: > 2.5 x the 126 MB L2


def attention_phase(a, world, rank, dev, peaks, peak_src):
    """One decode step of GQA attention over a fixed-block KV cache (attn_decode) for one sequence
    of L positions: 16 query heads, 2 KV heads, D=256, blocks of 64 rows in a shuffled block table.
    Distinct caches (together > 320 MB, so none is L2-resident when it is read again) are cycled in
    a CUDA graph of calls; the per-call time is the graph's time over its calls."""
    import torch
    from bit_quantized_expert_route_b200 import attn, moe, synth
    pts = {}
    for L in [int(n) for n in a.attn_L.split(",") if n]:
        kv = L * 2 * 256 * 2 * 2                      # keys + values of both KV heads, bf16
        n_cases = max(2, -(-CYCLE_BYTES // kv))
        cases = [synth.make_attention_case_on_device(900 + 97 * rank + i, [L], dev) for i in range(n_cases)]
        outs = [torch.empty_like(c.q) for c in cases]
        mb = cases[0].block_table.shape[1]
        ws = attn.alloc_workspace(1, 2, 256, 64, mb, dev)
        calls = n_cases * max(1, 32 // n_cases)

        def run_all():
            for i in range(calls):
                c = cases[i % n_cases]
                attn.attn_decode(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len, outs[i % n_cases], ws)

        for _ in range(max(3, a.warmup)):
            run_all()
        graph = capture_graph(run_all)
        graph.replay()
        reps = max(1, a.attn_reps // 10)
        ms = timed_loop(lambda i: graph.replay(), reps, world) / (reps * calls)
        del graph
        assert moe.moe_get_status(ws) == 0
        n_split, cps = attn.plan(1, 2, 64, mb)
        trd = committed_traffic("attn_decode_kernel<256>", ATTN_SRC, f"attn_L{L}")   # main kernel, per launch
        overhead = (n_split * 2 * 8 * (256 + 2) * 4 * 2) if n_split > 1 else 0   # partials written + read
        pts[str(L)] = {"us": round(ms * 1e3, 3), "steps_per_s": round(whole_job_rate(1, world, ms), 1),
                       "kv_bytes": kv, "split_partial_bytes": overhead, "n_split": n_split, "chunks_per_split": cps,
                       "launches_per_step": 2 if n_split > 1 else 1, "distinct_caches_cycled": n_cases,
                       "roofline": hbm_roofline("attn_decode_kernel<256> + attn_combine_kernel<256>", kv, ms, peaks,
                                                peak_src, traffic=trd[0] if trd else None)}
        del cases, outs, ws
        torch.cuda.empty_cache()
    return {"workload": "decode attention, 1 sequence, 16 Q heads / 2 KV heads (GQA groups of 8), D=256, "
                        "fixed blocks of 64 rows, shuffled block table, bf16 K/V ~ N(0,1)",
            "timing": "CUDA graph of back-to-back calls cycling distinct caches (> 320 MB together, so every "
                      "call reads its cache from HBM); per-call time = graph time / calls",
            "roofline_note": "algorithmic bytes = L x 2 KV heads x (K + V) x 256 x 2 B; the split partials "
                             "(split_partial_bytes) are overhead on top; the time covers both kernels",
            "points": pts}


def gdn_phase(a, world, rank, dev, peaks, peak_src):
    """One Gated DeltaNet decode step (gdn_decode_step) for B sequences: 16 key heads, 32 value heads,
    128 x 128 FP32 state per value head, updated in place.  Distinct states (together > 320 MB, as
    the model's 30 recurrence layers each keep their own) are cycled in a CUDA graph of calls."""
    import torch
    from bit_quantized_expert_route_b200 import deltanet
    Hk, Hv, dk, dv = 16, 32, 128, 128
    pts = {}
    for B in [int(n) for n in a.gdn_B.split(",") if n]:
        gen = torch.Generator(device=dev)
        gen.manual_seed(910 + 31 * rank + B)
        sb = B * Hv * dv * dk * 4
        n_st = max(2, -(-CYCLE_BYTES // sb))
        q = torch.randn((B, Hk, dk), generator=gen, device=dev).to(torch.bfloat16)
        k = torch.randn((B, Hk, dk), generator=gen, device=dev).to(torch.bfloat16)
        v = torch.randn((B, Hv, dv), generator=gen, device=dev).to(torch.bfloat16)
        g = torch.log(torch.rand((B, Hv), generator=gen, device=dev) * 0.149 + 0.85)
        beta = torch.rand((B, Hv), generator=gen, device=dev) * 0.9 + 0.05
        states = [torch.randn((B, Hv, dv, dk), generator=gen, device=dev) * 0.05 for _ in range(n_st)]
        out = torch.empty_like(v)
        calls = n_st * max(1, 64 // n_st)

        def run_all():
            for i in range(calls):
                deltanet.gdn_decode_step(q, k, v, g, beta, states[i % n_st], out)

        for _ in range(max(3, a.warmup)):
            run_all()
        graph = capture_graph(run_all)
        graph.replay()
        reps = max(1, a.attn_reps // 10)
        ms = timed_loop(lambda i: graph.replay(), reps, world) / (reps * calls)
        del graph
        nb = sb * 2 + B * (2 * Hk * dk + 2 * Hv * dv) * 2 + B * Hv * 8
        pts[str(B)] = {"us": round(ms * 1e3, 3), "tokens_per_s": round(whole_job_rate(B, world, ms), 1),
                       "bytes": nb, "launches_per_step": 1, "distinct_states_cycled": n_st,
                       "roofline": hbm_roofline("gdn_step_kernel<128>", nb, ms, peaks, peak_src)}
        del q, k, v, g, beta, states, out
        torch.cuda.empty_cache()
    return {"workload": "Gated DeltaNet decode step, 16 key heads / 32 value heads, 128 x 128 FP32 state per value "
                        "head, q, k, v ~ N(0,1) bf16, alpha ~ U(0.85, 0.999), beta ~ U(0.05, 0.95)",
            "timing": "CUDA graph of back-to-back steps cycling distinct states (> 320 MB together, so every "
                      "step reads its state from HBM); per-step time = graph time / steps",
            "roofline_note": "algorithmic bytes = the state read and written (B x 32 x 128 x 128 x 4 B x 2) "
                             "+ q, k, v, out, g, beta",
            "points": pts}


def gdn_oracle_times():
    """The float64 recurrence oracle on this host for every batch size of the workload."""
    from bit_quantized_expert_route_b200 import synth
    from oracle import deltanet_ref
    res = {}
    for B in GDN_B:
        c = synth.make_deltanet_case(910, B)
        t0 = time.perf_counter()
        deltanet_ref.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
        res[str(B)] = {"seconds": round(time.perf_counter() - t0, 3)}
    return res


def attention_oracle_times():
    """The float64 attention oracle on this host for every context length of the workload."""
    from bit_quantized_expert_route_b200 import synth
    from oracle import attn_ref
    res = {}
    for L in ATTN_L:
        c = synth.make_attention_case(900, [L])
        t0 = time.perf_counter()
        attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
        res[str(L)] = {"seconds": round(time.perf_counter() - t0, 3)}
    return res


# ------------------------------------------------------------ CPU oracle ---

def _oracle_time(fn, single_core: bool = False):
    from threadpoolctl import threadpool_limits
    if single_core:
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            fn()
            return time.perf_counter() - t0
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def oracle_full_cfg2():
    """The float64 oracle, as it stands, on the whole prefill input (4096 tokens): the
    cpu_baseline of the headline and the reference arm's step."""
    from bit_quantized_expert_route_b200 import synth
    from oracle import moe_ref
    dims = synth.Dims()
    lay = synth.make_layer(0, 0, dims)
    x = synth.make_x(0, T_PREFILL, dims.H)
    return lambda: moe_ref.moe_layer(x, lay, dims.k), lay, x


def oracle_phase(a):
    """Oracle timings on this host for every workload (rank 0 at N=1 only)."""
    from bit_quantized_expert_route_b200 import synth
    from oracle import moe_ref
    cores = len(os.sched_getaffinity(0))
    res = {"cores": cores, "kind": "oracle", "note": "NumPy float64; BLAS threads = cores unless single_core"}
    dims = synth.Dims()
    full, lay, x = oracle_full_cfg2()
    dt = _oracle_time(full)
    res["prefill_uniform"] = {"seconds": round(dt, 2), "tokens_per_s": round(T_PREFILL / dt, 2),
                              "sample": "all 4096 tokens of the uniform prefill input"}
    lay3 = synth.make_layer(1, 0, dims, zipf=True)
    x3 = synth.make_x(1, T_PREFILL, dims.H)
    dt3 = _oracle_time(lambda: moe_ref.moe_layer(x3, lay3, dims.k))
    res["prefill_zipf"] = {"seconds": round(dt3, 2), "tokens_per_s": round(T_PREFILL / dt3, 2),
                           "sample": "all 4096 tokens of the Zipf prefill input"}
    d1 = _oracle_time(lambda: moe_ref.moe_layer(x[:1], lay, dims.k))
    d1s = _oracle_time(lambda: moe_ref.moe_layer(x[:1], lay, dims.k), single_core=True)
    res["decode_T1"] = {"seconds": round(d1, 3), "seconds_single_core": round(d1s, 3),
                        "us_per_token": round(d1 * 1e6, 1), "us_per_token_single_core": round(d1s * 1e6, 1)}
    td = synth.Dims.tiny()
    lt, xt = synth.make_layer(0, 0, td), synth.make_x(0, 16, td.H)
    t0 = _oracle_time(lambda: moe_ref.moe_layer(xt, lt, td.k))
    t0s = _oracle_time(lambda: moe_ref.moe_layer(xt, lt, td.k), single_core=True)
    res["tiny_T16"] = {"seconds": round(t0, 4), "seconds_single_core": round(t0s, 4),
                       "tokens_per_s": round(16 / t0, 1), "tokens_per_s_single_core": round(16 / t0s, 1)}
    sw = {}
    for T in [int(t) for t in a.oracle_sweep_T.split(",") if t]:
        xs = synth.make_x(2, T, dims.H)
        dt_ = _oracle_time(lambda: moe_ref.moe_layer(xs, lay, dims.k))
        sw[str(T)] = {"seconds": round(dt_, 3), "tokens_per_s": round(T / dt_, 2)}
    res["sweep_layer0"] = sw
    if not a.no_attn:
        res["attention"] = attention_oracle_times()
    if not a.no_gdn:
        res["gated_deltanet"] = gdn_oracle_times()
    cpu_baseline = {"value": res["prefill_uniform"]["tokens_per_s"], "unit": "tokens/s", "cores": cores,
                    "kind": "oracle", "sample": "the whole uniform prefill input (4096 tokens), one call, "
                                                "NumPy float64, BLAS threads = cores",
                    "seconds": res["prefill_uniform"]["seconds"]}
    return cpu_baseline, res


# --------------------------------------------------------------- our arm ---

def run_ours(a):
    import torch
    from bit_quantized_expert_route_b200 import synth

    world, rank, local = dist_setup(a.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    dims = synth.Dims()
    zipf = a.workload == "zipf"
    peaks, peak_src = load_peaks()
    workloads = {}

    clk = ClockSampler(torch.cuda.current_device()).__enter__()   # sampled across every timed phase
    pre = {}
    if a.attn_only or a.gdn_only:
        a.decode_only, a.no_decode = True, True
        if a.attn_only:
            workloads["attention"] = attention_phase(a, world, rank, dev, peaks, peak_src)
        if a.gdn_only:
            workloads["gated_deltanet"] = gdn_phase(a, world, rank, dev, peaks, peak_src)
    if not a.decode_only:
        pre = prefill_phase(a, world, rank, dev, dims, zipf, peaks, peak_src, e2e=True)
        if not a.no_zipf_prefill and not zipf:
            workloads["prefill_zipf"] = prefill_phase(a, world, rank, dev, dims, True, peaks, peak_src, e2e=False)
    dl = None
    if not a.no_decode or (not a.no_sweep and not a.decode_only):
        dl = make_stack_layers(a, rank, dev, dims)
    if not a.no_decode:
        workloads["decode"] = decode_phase(a, world, rank, dev, dims, peaks, peak_src, dl)
    if not a.no_sweep and not a.decode_only:
        workloads["sweep"] = sweep_phase(a, world, rank, dev, dims, peaks, peak_src, dl)
    if not a.no_mid and not a.decode_only and dl is not None:
        workloads["decode_mid"] = decode_mid_phase(a, world, rank, dev, dims, peaks, peak_src, dl)
    del dl
    torch.cuda.empty_cache()
    if not a.no_tiny and not a.decode_only:
        workloads["tiny"] = tiny_phase(a, world, dev)
    if not a.no_attn and not a.decode_only:
        workloads["attention"] = attention_phase(a, world, rank, dev, peaks, peak_src)
    if not a.no_gdn and not a.decode_only:
        workloads["gated_deltanet"] = gdn_phase(a, world, rank, dev, peaks, peak_src)
    clk.__exit__(None, None, None)
    clocks = clk.summary()

    cpu, oracle_times = None, None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu, oracle_times = oracle_phase(a)

    if rank == 0:
        line = {
            "metric": "MoE-layer tokens/s (prefill T=4096)",
            "value": round(pre["value"], 1) if pre else None, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": pre.get("ms_per_step"), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": COMPUTE_DTYPE, "data": "synthetic",
            "config": {"workload": f"prefill T=4096 {'zipf(1.2) router bias' if zipf else 'uniform routing'}",
                       "T": T_PREFILL, "H": dims.H, "E": dims.E, "k": dims.k, "I": dims.I, "I_shared": dims.I_s,
                       "quant": "affine 4-bit, group 64, bf16 scale/bias",
                       "l2": f"{a.layers} layers + {a.layers} activation sets cycled "
                             f"({a.layers * 0.47:.1f} GB read per cycle) > 126 MB L2",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": pre.get("roofline"),
            "down_roofline": pre.get("down_roofline"),
            "layer_roofline": pre.get("layer_roofline"),
            "stage_ms": pre.get("stage_ms"),
            "cpu_baseline": cpu,
            "e2e": pre.get("e2e"),
            "gpu_launches": PREFILL_LAUNCHES_PER_STEP * a.steps if pre else 0,
            "clocks": clocks,
            "workloads": workloads,
            "oracle": oracle_times,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------- reference arm ---

def run_reference(a):
    """The oracle as the reference arm: rank 0 only.  Every timed step is one oracle call on the
    whole uniform prefill input (4096 tokens); warm-up steps run it on 16 of those tokens (the
    oracle has no state to warm, so they only page the code and data in)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from bit_quantized_expert_route_b200 import synth
    from oracle import moe_ref
    dims = synth.Dims()
    full, lay, x = oracle_full_cfg2()
    for _ in range(a.warmup):
        moe_ref.moe_layer(x[:16], lay, dims.k)
    times = []
    for _ in range(a.steps):
        t0 = time.perf_counter()
        full()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = T_PREFILL * len(times) / total
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference",
        "metric": "MoE-layer tokens/s (prefill T=4096)", "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(total / len(times) * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill T=4096 uniform routing", "T": T_PREFILL, "H": dims.H, "E": dims.E,
                   "k": dims.k, "I": dims.I, "I_shared": dims.I_s, "quant": "affine 4-bit, group 64, bf16 scale/bias",
                   "parallelism": "single process (CPU)"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "every timed step: the whole 4096-token uniform prefill input, NumPy float64, "
                                   "BLAS threads = cores; warm-up steps: 16 of those tokens"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_probe(a):
    """A small, fixed sequence of layer calls for ncu captures (one GPU)."""
    import torch
    from bit_quantized_expert_route_b200 import moe, synth
    dev = torch.device("cuda", 0)
    dims = synth.Dims()
    n_layers = a.probe_stack if a.probe_stack else 2
    layers = [moe.MoELayer.from_tensors(dims, synth.make_layer_on_device(300 + l, l, dims, dev, False))
              for l in range(n_layers)]
    x = synth.make_x_on_device(7, a.probe_T, dims.H, dev)
    out = torch.empty_like(x)
    ws = moe.alloc_workspace(layers[0], a.probe_T, dev)
    stack = moe.LayerStack(layers)
    for i in range(a.probe_calls):
        if a.probe_stack:
            moe.moe_forward_stack(stack, x, out, ws, eps=EPS)
        else:
            moe.moe_forward(layers[i % 2], x, out, ws)
    torch.cuda.synchronize()
    st = moe.moe_get_status(ws)
    print(f"probe T={a.probe_T} calls={a.probe_calls} status={st}")
    return 0 if st == 0 else 1


def main(argv=None):
    a = parse_args(argv)
    if a.probe_T:
        return run_probe(a)
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
    return 0


if __name__ == "__main__":
    sys.exit(main())
