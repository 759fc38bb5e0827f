"""Multi-rank plumbing of bench.py on CPU: gloo, world size 2 (the GPU path uses NCCL the same way)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.rank_barrier(world)
        mx = bench.reduce_over_ranks([1.0 + rank, 10.0 - rank, 3.5], world, "cpu", "max")
        sm = bench.reduce_over_ranks([100.0 * (rank + 1)], world, "cpu", "sum")
        out[rank] = (mx, sm)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()   # no fork of this (threaded) process
    out = manager.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in (0, 1):
        mx, sm = out[rank]
        assert mx == [2.0, 10.0, 3.5]          # max over ranks, element by element
        assert sm == [300.0]                   # bytes of all ranks


def test_whole_job_value():
    sys.path.insert(0, ROOT)
    import bench

    # two replicas moving 4 GB each in a slowest-rank step of 2 ms: 4 TB/s whole-job
    assert bench.whole_job_gbs(8e9, 2.0) == pytest.approx(4000.0)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny",
           "--cpu-sample-tokens", "16"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_reports_our_config_and_a_pinned_full_pass():
    """The reference arm names the same config dict as our arm and times the whole workload on one core."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "1",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "1", "--steps", "2", "--warmup", "3", "--workload", "tiny"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads([l for l in res.stdout.splitlines() if l.startswith("{")][0])
    sys.path.insert(0, ROOT)
    import bench
    from combine_get_dispatch_histogram_b200 import inputs

    assert line["config"] == bench.config_of(inputs.tiny(), 1)
    cb = line["cpu_baseline"]
    assert cb["cores"] == 1 and cb["pinned_core"] is not None
    assert cb["sample"].startswith("the whole workload")
    assert set(cb["stage_seconds"]) == {"layout", "dispatch", "combine"}


def test_kernel_time_statistics():
    sys.path.insert(0, ROOT)
    import bench

    st = bench.stats_ms([3.0, 1.0, 2.0, 10.0, 2.5])
    assert st == {"median": 2.5, "min": 1.0, "max": 10.0}


def test_l2_flush_only_for_steps_whose_rows_could_stay_cached():
    """Prefill's token rows (470 MB) outgrow L2 and go unflushed; decode (15 MB), the sweeps and the
    replica workload (134 MB) write a buffer larger than L2 before each timed step, and say so."""
    sys.path.insert(0, ROOT)
    import bench
    from combine_get_dispatch_histogram_b200 import inputs

    assert bench.L2_FLUSH_BYTES > bench.L2_BYTES
    assert not bench.needs_l2_flush(inputs.named("prefill"))
    assert bench.config_of(inputs.named("prefill"), 1)["l2"].startswith("no flush")
    for name in ("tiny", "decode", "sweep_T16", "sweep_T512", "sweep_T64_mask5", "replica"):
        w = inputs.named(name)
        assert bench.needs_l2_flush(w), name
        assert bench.config_of(w, 1)["l2"].startswith("flushed"), name
