"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1).
Weak scaling: every rank runs the same workload and the job takes as long as
its slowest rank; no data-path collective exists (the path shards by
independent sequences / query rows)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = [12.5, 17.0][rank]               # this rank's step time
        ms_max = bench.max_over_ranks(world, ms)
        value = bench.job_throughput(world, 131072, ms_max)
        bench.barrier(world)
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, value in got:
        assert ms_max == 17.0                      # max over ranks, on every rank
        assert value == pytest.approx(2 * 131072 / 17.0e-3)


def test_single_rank_paths_need_no_process_group():
    assert bench.max_over_ranks(1, 3.25) == 3.25
    assert bench.job_throughput(1, 100, 10.0) == pytest.approx(1e4)


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", str(world), "--steps", "1", "--warmup", "0", "--prefill", "tiny"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_runs_on_rank0_only():
    other = _run_reference(1, 2)
    assert other.returncode == 0 and other.stdout.strip() == ""
    first = _run_reference(0, 2)
    assert first.returncode == 0, first.stderr
    line = json.loads(first.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
