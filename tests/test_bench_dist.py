"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The layer shards as independent replicas (no exchange step), so what N > 1
adds is host logic: one process per rank, rank-distinct seeds, barriers, the
max-over-ranks timing and the whole-job rate, and a reference arm that runs
on rank 0 only.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo")
    bench.barrier_sync(w, cuda=False)
    slow = bench.max_over_ranks(10.0 * (r + 1), w, device="cpu")   # rank r "took" 10(r+1) ms
    seeds = bench.replica_seeds(r, 2)
    bench.barrier_sync(w, cuda=False)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "max_ms": slow, "seeds": seeds}, f)
    dist.destroy_process_group()


def test_two_rank_timing_and_seeds(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(x["world"] == world for x in res)
    assert [x["max_ms"] for x in res] == [20.0, 20.0]           # every rank reports the slowest
    assert res[0]["seeds"] != res[1]["seeds"]                   # replicas draw distinct data


def test_whole_job_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(4096 * 10, 1, 1000.0) == pytest.approx(40960.0)
    assert bench.whole_job_rate(4096 * 10, 4, 1000.0) == pytest.approx(4 * 40960.0)


def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_committed_traffic_needs_the_same_source_and_workload(tmp_path, monkeypatch):
    """The roofline's `traffic` comes from a committed ncu summary only while the kernel's source
    file is byte-identical to the one profiled, and only for the workload it was captured on."""
    sys.path.insert(0, ROOT)
    import hashlib
    import bench
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.md").write_text(
        f"traffic_bytes_per_launch: k<true> 1234 src_sha={sha} workload=wl_a\n"
        f"traffic_bytes_per_launch: k<true> 999 src_sha=0000000000000000 workload=wl_b\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.committed_traffic("k<true>", "k.cu", "wl_a") == (1234, "wl_a")
    assert bench.committed_traffic("k<true>", "k.cu", "wl_b") is None       # captured on an older source
    assert bench.committed_traffic("k<false>", "k.cu", "wl_a") is None      # another kernel
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench.committed_traffic("k<true>", "k.cu", "wl_a") is None       # source changed since
