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


# ------------------------------------------------ shard plan (no exchange)

def _shard_main(rank, world, port, q):
    """Each rank computes its own part of the 128K prefill and of a decode
    batch from the library's host-only partition; rank 0 gathers them."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = bench.shard_prefill_rows(world, rank, 131072, 131072, 2048, 8, 128, 128, 576, 512)
        ctx = [8192 + (b * 7919) % 122880 for b in range(64)]
        dec = bench.shard_decode_seqs(world, rank, ctx, 2048, 128, 576)
        parts = [None] * world
        dist.all_gather_object(parts, (rank, mine, dec))
        q.put(parts)
    finally:
        dist.destroy_process_group()


def _row_cost(t, S=131072, T=131072, k=2048):
    n = t + S - T + 1
    return (n * 2 * 8 * 128 / 2 if n > k else 0) + min(n, k) * 2 * 128 * (576 + 512)


def test_two_gloo_ranks_split_rows_and_sequences_once_with_balanced_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert got[0] == got[1]                      # every rank sees the same plan
    parts = sorted(got[0])
    rows = [pr for _, pr, _ in parts]
    seqs = [ds for _, _, ds in parts]
    # contiguous ranges covering every row / sequence exactly once
    assert rows[0][0] == 0 and rows[-1][1] == 131072 and rows[0][1] == rows[1][0]
    assert seqs[0][0] == 0 and seqs[-1][1] == 64 and seqs[0][1] == seqs[1][0]
    # balanced modelled work: the split row sits where the cost halves
    costs = [sum(_row_cost(t) for t in range(a, b)) for a, b in rows]
    assert abs(costs[0] - costs[1]) <= 2 * max(_row_cost(t) for t in range(131072))
    # the later rows cost more (causal indexer term): rank 0 takes more rows
    assert rows[0][1] - rows[0][0] > rows[1][1] - rows[1][0]


def test_partition_edge_cases_on_the_host():
    import sparse_attention_20_b200 as dsa
    # more ranks than rows: some ranges are empty, all rows covered once
    b = dsa.partition_prefill_rows(5, 5, 2048, 8, 128, 128, 576, 512, 8)
    assert b[0] == 0 and b[-1] == 5 and all(x <= y for x, y in zip(b, b[1:]))
    # one rank: everything
    assert dsa.partition_prefill_rows(1000, 4000, 64, 4, 32, 4, 80, 64, 1) == [0, 1000]
    # a tail prefill (T < S): costs start high, ranges stay contiguous and balanced
    b = dsa.partition_prefill_rows(4096, 131072, 2048, 8, 128, 128, 576, 512, 4)
    assert b[0] == 0 and b[-1] == 4096 and len(b) == 5
    sizes = [y - x for x, y in zip(b, b[1:])]
    assert max(sizes) - min(sizes) <= 0.01 * 1024          # costs there differ by ~3%
    assert sizes == sorted(sizes, reverse=True)            # later rows cost more
    # decode: equal contexts split evenly; one huge sequence gets a rank alone
    assert dsa.partition_decode_seqs([1000] * 8, 2048, 128, 576, 4) == [0, 2, 4, 6, 8]
    b = dsa.partition_decode_seqs([100000, 10, 10, 10], 2048, 128, 576, 2)
    assert b == [0, 1, 4]
    # argument errors are reported, not launched
    with pytest.raises(dsa.DSAError):
        dsa.partition_prefill_rows(10, 5, 2048, 8, 128, 128, 576, 512, 2)
    with pytest.raises(dsa.DSAError):
        dsa.partition_decode_seqs([10, -1], 2048, 128, 576, 2)
