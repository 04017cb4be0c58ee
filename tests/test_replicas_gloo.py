"""The multi-GPU form of this path is replicas (every (batch, KV head) unit is
independent; no collective on the data path).  bench.py's only cross-rank steps
are a barrier and the max over ranks of the timed duration, from which the
whole-job throughput follows.  Checked here with two gloo ranks on the CPU."""
import datetime
import os
import socket
import subprocess
import sys

import pytest

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        ms = 10.0 + 5.0 * rank  # each replica's own timed duration
        dist.barrier()
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        q.put((rank, w, r, local, slowest, bench.job_throughput(w, 100, slowest / 1e3)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_duration():
    import torch.multiprocessing as mp

    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    for rank, (r_, w, r, local, slowest, value) in enumerate(res):
        assert (r_, w, r, local) == (rank, 2, rank, rank)
        assert slowest == 15.0
        assert value == pytest.approx(2 * 100 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_throughput(1, 10, 0.5) == 20.0


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun every rank but 0 leaves the reference arm at once with status 0."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_f32_4k"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_json_contract():
    """The reference arm (the CPU oracle timed on the host) prints one JSON line with the
    bench contract's keys, its own impl tag, a cpu_baseline and a zero-byte e2e."""
    import json

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_f32_4k"], capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "steps/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny_f32_4k"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"]


def test_cpu_baseline_uses_every_host_core():
    """The benchmark's CPU baseline times whole decode steps of the oracle on every core
    this process may run on, and a bounded one-thread sample beside it."""
    sys.path.insert(0, ROOT)
    import bench
    from hata_inputs import WORKLOADS, make_inputs

    wl = WORKLOADS["tiny_f32_4k"]
    cb = bench.cpu_baseline(wl, make_inputs(wl, seed=0), budget_s=0.5)
    assert cb["kind"] == "oracle" and cb["unit"] == "steps/s" and cb["value"] > 0
    assert cb["cores"] == bench.host_cores()
    assert cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0
