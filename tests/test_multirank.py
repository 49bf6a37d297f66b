"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, no GPU.

Sequences are independent, so the ranks share no data; what must hold is that every rank runs the
same shapes on its own seed, that the job time is the slowest rank's, that the job's value counts
every rank's units, and that the reference arm runs on rank 0 only.
"""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        wl = bench.rank_workload("ctx1m_fp8_b32", r)
        slow = bench.max_over_ranks(10.0 + 5.0 * r, w, torch.device("cpu"))  # rank 1 is the slow one
        dist.barrier()
        value = bench.job_throughput(w, wl.L * wl.total_S, 4, slow)
        out.put((r, w, local, wl.seed, wl.B, wl.total_S, slow, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, seed0, B0, T0, slow0, v0), (r1, w1, l1, seed1, B1, T1, slow1, v1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == world and (l0, l1) == (0, 1)
    assert seed0 != seed1 and (B0, T0) == (B1, T1)           # own seed, same shapes
    assert slow0 == slow1 == 15.0                             # the slowest rank's time on every rank
    assert v0 == v1 == pytest.approx(world * 3 * T0 * 4 / 15e-3)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_matches_the_gpu_arm():
    """Rank 0 prints one JSON line with the GPU arm's metric, unit and config (the oracle timed on
    a bounded sample of the same workload) and an e2e with no host-device bytes."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    import synth
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--cpu-sample", "512"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC and out["unit"] == bench.UNIT
    assert out["higher_is_better"] is True and out["n_gpus"] == 1 and out["value"] > 0
    assert out["config"] == bench.workload_config(synth.workload(bench.DEFAULT_WORKLOAD), 0.5, 1)
    assert out["e2e"] == {"value": out["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == out["value"] and cb["cores"] >= 1 and "512" in cb["sample"]
