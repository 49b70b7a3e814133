"""Benchmark of the DSA hot path on B200: one JSON line on stdout (rank 0).

A step is one pass of the whole hot path over one batch of synthetic inputs:
the 128K-token causal prefill (lightning indexer + Top-k selector + sparse MQA
attention over 2048 selected latent rows per token) followed by one decode
step of 64 sequences (contexts uniform in [8K, 128K]). `value` is prefill
tokens/s over the whole job (all ranks); decode seqs/s is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs the same independent workload (weak
scaling, no collective on the data path); the step time is the max over ranks.
Inputs (19 GB of queries) are far larger than L2, so no flush is needed
between steps. `--impl reference` times the CPU oracle on bounded samples of
the same workload.
"""
from __future__ import annotations

import argparse
import json
import re
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "DSA prefill tokens/s & decode seqs/s at 128K ctx; % of FP8/BF16 TC / HBM roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill", default="prefill128k")
    ap.add_argument("--decode", default="decode")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override L of the prefill workload (smaller cases for profiling)")
    ap.add_argument("--varlen", default=None,
                    help="comma-separated sequence lengths: time a packed batch of causal prefills "
                         "(varlen indexer + attention) instead of the default step")
    ap.add_argument("--decode-page-size", type=int, default=None,
                    help="run the decode step over paged caches (block table, pages of this size)")
    ap.add_argument("--rows", type=int, default=None,
                    help="prefill only the last ROWS tokens of the sequence (long rows, small "
                         "footprint: profiling)")
    ap.add_argument("--bwd", nargs="?", const="prefill32k", default=None,
                    help="time the sparse attention backward on this prefill workload "
                         "(default prefill32k) instead of the default step")
    ap.add_argument("--kl", nargs="?", const="prefill32k", default=None,
                    help="time the indexer KL loss and its gradient on this prefill workload "
                         "(default prefill32k) instead of the default step")
    ap.add_argument("--mha", nargs="?", const="mha_short", default=None,
                    help="time MLA MHA-mode dense causal attention (short prefill, default "
                         "mha_short: 2048 tokens, 128 heads, d_h 192, d_hv 128) instead of the default step")
    ap.add_argument("--replicas", action="store_true",
                    help="with several ranks, run the whole workload on every rank (weak scaling) "
                         "instead of splitting its query rows and sequences between them")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args()


# ------------------------------------------------------------- distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    """The largest x over all ranks (the step time of the slowest GPU)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_prefill_rows(world: int, rank: int, T: int, S: int, k: int, H_I: int, d_I: int, Hq: int,
                       d_qk: int, d_v: int):
    """This rank's query rows [t0, t1) of one causal prefill: contiguous ranges of
    equal modelled work from the library's partition (host-only call)."""
    import sparse_attention_20_b200 as dsa
    b = dsa.partition_prefill_rows(T, S, k, H_I, d_I, Hq, d_qk, d_v, world)
    return b[rank], b[rank + 1]


def shard_decode_seqs(world: int, rank: int, ctx, k: int, d_I: int, d_qk: int):
    """This rank's decode sequences [b0, b1) (contiguous, equal modelled bytes)."""
    import sparse_attention_20_b200 as dsa
    b = dsa.partition_decode_seqs(ctx, k, d_I, d_qk, world)
    return b[rank], b[rank + 1]


def shard_inputs(x, world: int, rank: int):
    """The part of batch x this rank runs. A causal prefill (pos / k_base NULL)
    keeps rows [t0, t1) as the tail prefill of its first t1 + S - T tokens (the
    row slices of q_idx, w, q and a prefix of the caches); a decode batch keeps
    sequences [b0, b1) with their pos / k_base over the whole caches."""
    import synth
    H_I, d_I = x.q_idx.shape[1], x.q_idx.shape[2]
    Hq, d_qk = x.q.shape[1], x.q.shape[2]
    if x.pos is None and x.k_base is None:
        t0, t1 = shard_prefill_rows(world, rank, x.T, x.S, x.k, H_I, d_I, Hq, d_qk, x.d_v)
        s1 = t1 + x.S - x.T
        return synth.DSAInputs(x.config, x.q_idx[t0:t1], x.w[t0:t1], x.k_idx[:s1], x.q[t0:t1], x.kv[:s1],
                               None, None, x.k, x.scale, x.d_v, dict(x.meta, rows=(t0, t1)))
    ctx = (x.positions() + 1).cpu().tolist()
    b0, b1 = shard_decode_seqs(world, rank, ctx, x.k, d_I, d_qk)
    # pos / k_base slices are copied: the library wants 16-byte aligned arrays
    return synth.DSAInputs(x.config, x.q_idx[b0:b1], x.w[b0:b1], x.k_idx, x.q[b0:b1], x.kv,
                           x.positions()[b0:b1].clone(), x.bases()[b0:b1].clone(), x.k, x.scale, x.d_v,
                           dict(x.meta, rows=(b0, b1)))


def job_throughput(world: int, units_per_rank: int, ms_max: float) -> float:
    """Whole-job units/s for weak scaling: every rank processes units_per_rank,
    the job takes as long as its slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v for v in vis.split(",") if v.strip()]
        self.index = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.index, f"--query-gpu={self.FIELDS}", "--format=csv",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or not parts[1].split()[0].isdigit():
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [int(r[1].split()[0]) for r in rows]
        mx = max(int(r[2].split()[0]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(sm)}


# ------------------------------------------------------------- workloads

def algorithmic_work(x):
    """Per-launch algorithmic work of one forward over batch x (units in the docstrings)."""
    pos = x.positions().cpu().long()
    n = pos + 1
    H_I, d_I = x.q_idx.shape[1], x.q_idx.shape[2]
    Hq, d_qk = x.q.shape[1], x.q.shape[2]
    d_v, k = x.d_v, x.k
    sel = torch.clamp(n, max=k)
    # indexer: FP8 flops of q.k over the causal pairs of rows that need scoring (n > k)
    scored = n[n > k]
    idx_flops = float(scored.sum().item()) * 2 * H_I * d_I
    # attention: bf16 flops of q.c (d_qk) and p.v (d_v) per (row, selected entry, head)
    attn_flops = float(sel.sum().item()) * Hq * 2 * (d_qk + d_v)
    # bytes a perfect implementation moves: every key of every row's range read once
    # (decode), the selected latent rows gathered once per row, q read, out/lse written
    idx_bytes = float(n.sum().item()) * d_I + x.T * (H_I * d_I + 4 * H_I + 4 * k)
    attn_bytes = (float(sel.sum().item()) * d_qk * 2 + x.T * Hq * (d_qk * 2 + d_v * 2 + 4)
                  + x.T * k * 4)
    return dict(idx_flops=idx_flops, attn_flops=attn_flops, idx_bytes=idx_bytes,
                attn_bytes=attn_bytes)


def prefill_kw(args):
    kw = {}
    if args.seq_len:
        kw["L"] = args.seq_len
    if args.rows:
        kw["T"] = args.rows
    return kw


def sharded(args, world) -> bool:
    """Several ranks split one workload (strong scaling) unless --replicas."""
    return world > 1 and not getattr(args, "replicas", False)


def workload_config(args, xp, world):
    """The `config` of the JSON line, the same for both arms."""
    H_I, d_I = xp.q_idx.shape[1], xp.q_idx.shape[2]
    Hq, d_qk = xp.q.shape[1], xp.q.shape[2]
    dc = synth.CONFIGS[args.decode]
    decode = (f"{dc['B']} seqs, ctx U[{dc['ctx_lo']},{dc['ctx_hi']}]" if dc["kind"] == "decode"
              else f"{dc['L']} rows")
    if getattr(args, "decode_page_size", None):
        decode += f", paged caches of {args.decode_page_size}-row pages"
    rows = f"L={xp.T}" if xp.T == xp.S else f"last {xp.T} of L={xp.S}"
    return {"workload": f"{args.prefill} causal prefill ({rows}, H_I={H_I}, d_I={d_I}, k={xp.k}, "
                        f"Hq={Hq}, d_qk={d_qk}, d_v={xp.d_v}) + {args.decode} step ({decode})",
            "global_batch": 1 if sharded(args, world) else world, "seq_len": xp.T,
            "parallelism": (f"rows{world} (query rows and decode sequences split, no exchange)"
                            if sharded(args, world) else f"replicas{world}"),
            "l2": f"inputs larger than L2: {xp.T * Hq * d_qk * 2 / 1e9:.1f} GB of queries, "
                  f"{xp.S * d_qk * 2 / 1e6:.0f} MB latent cache (L2 126 MB)"}


class Batch:
    def __init__(self, x, dsa):
        self.x = x
        self.T, self.S = x.T, x.S
        self.H_I, self.d_I = x.q_idx.shape[1], x.q_idx.shape[2]
        self.Hq, self.d_qk = x.q.shape[1], x.q.shape[2]
        dev = x.q.device
        self.idx = torch.empty((self.T, x.k), dtype=torch.int32, device=dev)
        self.out = torch.empty((self.T, self.Hq, x.d_v), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((self.T, self.Hq), dtype=torch.float32, device=dev)
        self.ws = dsa.alloc_workspace(self.T, self.S, self.H_I, self.d_I, x.k, self.Hq,
                                      self.d_qk, x.d_v, dev)
        self.work = algorithmic_work(x)
        self.paged = None   # (k_pages, kv_pages, block_table, seq, page_size) for a paged cache


def run_indexer(dsa, b, stream):
    x = b.x
    if b.paged is not None:
        kp, vp, bt, seq, ps = b.paged
        dsa.indexer_topk_paged(x.q_idx, x.w, kp, ps, bt, seq, x.pos, x.k, idx=b.idx, workspace=b.ws,
                               stream=stream)
        return
    dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base, idx=b.idx,
                     workspace=b.ws, stream=stream)


def run_attn(dsa, b, stream):
    x = b.x
    if b.paged is not None:
        kp, vp, bt, seq, ps = b.paged
        dsa.sparse_mla_attn_paged(x.q, vp, ps, bt, seq, x.pos, b.idx, x.scale, x.d_v, out=b.out,
                                  lse=b.lse, stream=stream)
        return
    dsa.sparse_mla_attn(x.q, x.kv, b.idx, x.scale, x.d_v, pos=x.pos, k_base=x.k_base, out=b.out,
                        lse=b.lse, workspace=b.ws, stream=stream)


def profiled_traffic(profile: str, key: str, sources) -> float | None:
    """DRAM bytes per launch recorded in a committed ncu summary (`profiles/`),
    or None once any of the kernel's source files has changed since those
    counters were taken (the summary records a sha256 prefix of them)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", profile)
    csrc = os.path.join(ROOT, "sparse_attention_20_b200", "csrc")
    try:
        text = open(prof).read()
        want = re.search(key + r"_source_sha256_16:\s*([0-9a-f]+)", text).group(1)
        value = float(re.search(key + r"_traffic_bytes_per_launch:\s*([0-9.e+]+)", text).group(1))
        h = hashlib.sha256()
        for f in sources:
            h.update(open(os.path.join(csrc, f), "rb").read())
    except (OSError, AttributeError, ValueError):
        return None
    return value if h.hexdigest()[:16] == want else None


def attn_traffic():
    """DRAM bytes per prefill attention launch (128K workload)."""
    return profiled_traffic("sparse_mla_attn_tc_prefill128k.md", "attn",
                            ("attn_tc.cuh", "sm100.cuh", "common.cuh", "dsa.cu"))


MHA_SOURCES = ("mha_tc.cuh", "mha_attn.cuh", "attn_bwd.cuh", "sm100.cuh", "common.cuh", "dsa.cu")


def fp8_gemm_tflops(n=8192, reps=10):
    """Burst FP8 (e4m3) dense GEMM rate of this GPU, n^3 through cuBLAS
    (torch._scaled_mm), best of `reps`; None if unavailable."""
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except (RuntimeError, AttributeError, TypeError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# --------------------------------------------------------- CPU baseline

def time_oracle_sample(x, rows):
    import numpy as np
    import oracle
    r = torch.tensor(rows, device=x.q.device)
    q_idx = x.q_idx[r].cpu().numpy()
    w = x.w[r].cpu().numpy()
    k_idx = x.k_idx.cpu().numpy()
    q = x.q[r].cpu()
    kv = x.kv.cpu()
    pos = x.positions()[r].cpu().numpy()
    base = x.bases()[r].cpu().numpy()
    t0 = time.perf_counter()
    idx = oracle.indexer_topk(q_idx, w, k_idx, pos, base, x.k)
    oracle.sparse_attn(q, kv, None, pos, base, x.scale, x.d_v, idx_rows=idx)
    return time.perf_counter() - t0, oracle.num_threads()


def cpu_baseline(x, seed=0, target_s=15.0):
    """The oracle as it stands on a bounded sample of query rows of workload x."""
    import oracle
    threads = oracle.num_threads()
    g = torch.Generator().manual_seed(seed)
    n = max(4, threads)
    rows = sorted(torch.randperm(x.T, generator=g)[:n].tolist())
    dt, cores = time_oracle_sample(x, rows)
    # grow towards the target duration (at most twice) while the sample is short
    for _ in range(2):
        if dt >= target_s / 2 or len(rows) >= x.T:
            break
        n2 = min(x.T, int(len(rows) * min(64.0, target_s / max(dt, 1e-3))))
        rows = sorted(torch.randperm(x.T, generator=g)[:n2].tolist())
        dt, cores = time_oracle_sample(x, rows)
    return dict(value=len(rows) / dt, unit="tokens/s", cores=cores, kind="oracle",
                sample=f"{len(rows)} uniformly drawn query rows of the {x.config} workload "
                       f"(L={x.T}); indexer scores of all causal keys, full sort, fp64 "
                       f"attention over the selected rows; {dt:.1f} s")


# ----------------------------------------------------------- ours

def bench_ours(args, world, rank, local):
    import sparse_attention_20_b200 as dsa
    from sparse_attention_20_b200 import build as dsa_build
    if rank == 0:
        dsa_build.build()
    barrier(world)
    dsa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    split = sharded(args, world)
    # split: every rank draws the same workload and runs its part of it;
    # replicas: every rank runs a whole workload of its own
    seed = args.seed if split else args.seed + rank
    xp = synth.make_inputs(args.prefill, device=dev, seed=seed, **prefill_kw(args))
    xd = synth.make_inputs(args.decode, device=dev, seed=seed)
    xp_full, xd_full = xp, xd
    if split:
        xp, xd = shard_inputs(xp, world, rank), shard_inputs(xd, world, rank)
    bp, bd = Batch(xp, dsa), Batch(xd, dsa)
    if args.decode_page_size:
        ps = args.decode_page_size
        kp, vp, bt, seq = synth.page_caches(xd, ps, seed=args.seed)
        bd.paged = (kp, vp, bt, seq, ps)
        bd.ws = dsa.alloc_workspace(xd.T, bt.shape[1] * ps, bd.H_I, bd.d_I, xd.k, bd.Hq, bd.d_qk, xd.d_v,
                                    dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None: ev[0].record(stream)
        run_indexer(dsa, bp, stream)
        if ev is not None: ev[1].record(stream)
        run_attn(dsa, bp, stream)
        if ev is not None: ev[2].record(stream)
        run_indexer(dsa, bd, stream)
        if ev is not None: ev[3].record(stream)
        run_attn(dsa, bd, stream)
        if ev is not None: ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = dsa.launch_count() - n0
    clk = clocks.stop()
    total_ms = max_over_ranks(world, start.elapsed_time(end))
    parts = [[e[j].elapsed_time(e[j + 1]) for e in evs] for j in range(4)]
    p_idx, p_attn, d_idx, d_attn = (max_over_ranks(world, statistics.mean(p)) for p in parts)
    assert dsa.device_status() == 0, dsa.last_error()

    ms_step = total_ms / args.steps
    prefill_ms = p_idx + p_attn
    decode_ms = d_idx + d_attn
    # whole-job units: the full workload once (split) or once per rank (replicas)
    tokens = xp_full.T if split else world * xp.T
    seqs = xd_full.T if split else world * xd.T
    peaks = measured_peaks()
    wp, wd = bp.work, bd.work
    attn_tflops = wp["attn_flops"] / (p_attn * 1e-3) / 1e12
    # Denominators: each kernel is one launch of tens of milliseconds at most,
    # timed on its own, so its peak is the burst figure (bf16 from
    # MEASURED_PEAKS.json; FP8 measured here by a cuBLAS GEMM, else 2 x bf16
    # burst, the nominal ratio). The sustained figures are reported beside them.
    fp8_burst = fp8_gemm_tflops()
    if fp8_burst:
        fp8_peak = fp8_burst
        fp8_source = f"measured FP8 GEMM burst (cuBLAS e4m3 8192^3, this run)"
    else:
        fp8_peak = 2.0 * peaks["bf16"]
        fp8_source = f"2 x {peaks['source']} bf16 burst (nominal FP8 ratio)"
    fp8_sustained = fp8_peak * peaks["bf16_sustained"] / peaks["bf16"]
    result = {
        "metric": METRIC,
        "value": tokens / (ms_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the pages' 128K workloads)",
        "config": workload_config(args, xp_full, world),
        "prefill_tokens_per_s": tokens / (prefill_ms * 1e-3),
        "decode": {"value": seqs / (decode_ms * 1e-3), "unit": "seqs/s",
                   "ms_per_step": decode_ms,
                   "hbm_gbs": (wd["idx_bytes"] + wd["attn_bytes"]) / (decode_ms * 1e-3) / 1e9,
                   "hbm_frac": (wd["idx_bytes"] + wd["attn_bytes"]) / (decode_ms * 1e-3) / 1e9
                   / peaks["hbm"]},
        "kernels_ms": {"prefill_indexer_topk": p_idx, "prefill_sparse_attn": p_attn,
                       "decode_indexer_topk": d_idx, "decode_sparse_attn": d_attn},
        "roofline": {"bound": "tensor", "kernel": "prefill sparse MLA attention",
                     "achieved": attn_tflops, "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16"],
                     "traffic": attn_traffic() if xp.config == "prefill128k" and xp.T == 131072
                     else None,
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": attn_tflops / peaks["bf16_sustained"]},
        "rooflines": {
            "prefill_indexer_topk": {"bound": "tensor", "unit": "TFLOP/s",
                                     "achieved": wp["idx_flops"] / (p_idx * 1e-3) / 1e12,
                                     "peak": fp8_peak,
                                     "frac": wp["idx_flops"] / (p_idx * 1e-3) / 1e12 / fp8_peak,
                                     "peak_source": fp8_source,
                                     "frac_of_sustained": wp["idx_flops"] / (p_idx * 1e-3) / 1e12
                                     / fp8_sustained},
            "decode_step": {"bound": "hbm", "unit": "GB/s",
                            "achieved": (wd["idx_bytes"] + wd["attn_bytes"]) / (decode_ms * 1e-3)
                            / 1e9, "peak": peaks["hbm"],
                            "frac": (wd["idx_bytes"] + wd["attn_bytes"]) / (decode_ms * 1e-3) / 1e9
                            / peaks["hbm"], "peak_source": f"{peaks['source']} HBM copy"},
        },
        "gpu_launches": launches,
        "clocks": clk,
    }
    result["topk"] = topk_phases(dsa, bp, bd, stream)
    if split:
        result["shard"] = {"prefill_rows": list(xp.meta["rows"]), "decode_seqs": list(xd.meta["rows"]),
                           "rank": rank}
    if not args.no_e2e:
        result["e2e"] = bench_e2e(args, world, dsa, bp, bd, stream, tokens)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(xp, seed=args.seed)
    return result


def topk_phases(dsa, bp, bd, stream):
    """The indexer's phases timed on their own (one extra step after the timed
    region, CUDA events around each phase inside the library): the Top-k
    selection alone, reported as GB/s over the bytes it moves, per row that
    needs a selection (n > k).

    - Prefill (streaming indexer): the threshold keeps about 2k (score, s)
      pairs of 8 bytes (all n when n <= 2k), read once, plus the k int32
      indices written.
    - Decode (up to 2048 rows over long key ranges): the select reads the
      row's dense score row once (4 bytes per key), each of the row's four
      CTAs stages the row's group maxima (4 bytes each: one per 16 keys, or
      per 4 keys where there are fewer than k 16-key groups), and the k int32
      indices are written."""
    out = {}
    for name, b in (("prefill", bp), ("decode", bd)):
        dsa.phase_timing(True)
        run_indexer(dsa, b, stream)
        torch.cuda.synchronize()
        ph = dsa.phase_times()
        dsa.phase_timing(False)
        n = b.x.positions().cpu().long() + 1
        k = b.x.k
        sel = n > k
        if name == "prefill":
            nbytes = float((torch.clamp(n[sel], max=2 * k) * 8).sum().item() + int(sel.sum().item()) * k * 4)
        else:
            ns = n[sel]
            tiles = (ns + 127) // 128
            m = torch.where(tiles * 8 >= k, tiles * 8, torch.where(tiles * 32 >= k, tiles * 32, 0))
            nbytes = float((ns * 4 + 4 * m * 4 + k * 4).sum().item())
        out[name] = {"scores_ms": ph["scores"], "threshold_ms": ph["threshold"], "select_ms": ph["select"],
                     "select_bytes": nbytes,
                     "select_gbs": nbytes / (ph["select"] * 1e-3) / 1e9 if ph["select"] > 0 else None}
    return out


def bench_e2e(args, world, dsa, bp, bd, stream, tokens):
    """Same step through the C ABI with inputs in pinned host memory: every step
    copies its inputs host->device and reads idx/out/lse back (consecutive
    steps' copies overlap in the two directions)."""
    def host(t):
        try:
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        except RuntimeError:
            h = torch.empty(t.shape, dtype=t.dtype)
        h.copy_(t)
        return h

    pairs_in, pairs_out = [], []
    for b in (bp, bd):
        x = b.x
        for t in (x.q_idx, x.w, x.k_idx, x.q, x.kv, x.pos, x.k_base):
            if t is not None:
                pairs_in.append((host(t), t))
        for t in (b.idx, b.out, b.lse):
            pairs_out.append((host(t), t))
    h2d = sum(h.numel() * h.element_size() for h, _ in pairs_in)
    d2h = sum(h.numel() * h.element_size() for h, _ in pairs_out)

    # Three streams: uploads, compute (the library's launches) and downloads.
    # A step's compute waits for its own upload and for the previous step's
    # download (the output buffers); its upload waits for the previous step's
    # compute (the input buffers). So step i+1's inputs upload while step i's
    # results download (PCIe runs both directions at once), and every step
    # still moves all of its inputs in and all of its results out.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    state = {"computed": None, "downloaded": None}

    def step():
        with torch.cuda.stream(s_in):
            if state["computed"] is not None:
                s_in.wait_event(state["computed"])
            for h, d in pairs_in:
                d.copy_(h, non_blocking=True)
            uploaded = torch.cuda.Event()
            uploaded.record(s_in)
        stream.wait_event(uploaded)
        if state["downloaded"] is not None:
            stream.wait_event(state["downloaded"])
        for b in (bp, bd):
            run_indexer(dsa, b, stream)
            run_attn(dsa, b, stream)
        computed = torch.cuda.Event()
        computed.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed)
            for h, d in pairs_out:
                h.copy_(d, non_blocking=True)
            downloaded = torch.cuda.Event()
            downloaded.record(s_out)
        state["computed"], state["downloaded"] = computed, downloaded

    step()
    torch.cuda.synchronize()
    state["computed"] = state["downloaded"] = None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(s_in)
    for _ in range(args.e2e_steps):
        step()
    s_out.wait_event(state["computed"])
    end.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(world, start.elapsed_time(end)) / args.e2e_steps
    return {"value": tokens / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "copies": "step i+1's upload overlaps step i's download; compute waits for both",
            "pinned": all(h.is_pinned() for h, _ in pairs_in + pairs_out)}


# ------------------------------------------------------ reference arm

def bench_reference(args, world, rank):
    """The CPU oracle as the reference arm, on bounded samples of the same workload."""
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.make_inputs(args.prefill, device=dev, seed=args.seed, **prefill_kw(args))
    threads = oracle.num_threads()
    g = torch.Generator().manual_seed(args.seed)
    per_step = max(2, threads)
    samples = []
    for i in range(args.warmup + args.steps):
        rows = sorted(torch.randperm(x.T, generator=g)[:per_step].tolist())
        dt, cores = time_oracle_sample(x, rows)
        if i >= args.warmup:
            samples.append((len(rows), dt))
    rows_total = sum(n for n, _ in samples)
    secs = sum(d for _, d in samples)
    value = rows_total / secs
    sample = (f"{per_step} uniformly drawn query rows of the {x.config} workload per step "
              f"(L={x.T}); oracle indexer + full sort + fp64 attention")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(args, x, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def bench_varlen(args, world, rank, local):
    """Batched (variable-length) prefill: packed causal sequences of the
    prefill128k shapes, indexer per sequence + attention with pos / k_base."""
    import sparse_attention_20_b200 as dsa
    from sparse_attention_20_b200 import build as dsa_build
    if rank == 0:
        dsa_build.build()
    barrier(world)
    dsa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    lens = [int(v) for v in args.varlen.split(",")]
    x = synth.varlen_prefill_inputs(args.prefill, device=dev, seed=args.seed + rank, lens=lens)
    cu = x.meta["cu"]
    H_I, d_I = x.q_idx.shape[1], x.q_idx.shape[2]
    ws = dsa.alloc_workspace(max(lens), max(lens), H_I, d_I, x.k, x.q.shape[1], x.q.shape[2], x.d_v, dev)
    idx = torch.empty((x.T, x.k), dtype=torch.int32, device=dev)
    out = torch.empty((x.T, x.q.shape[1], x.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((x.T, x.q.shape[1]), dtype=torch.float32, device=dev)
    pos, base = dsa.varlen_rows(cu, cu, dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None: ev[0].record(stream)
        dsa.indexer_topk_varlen(x.q_idx, x.w, x.k_idx, cu, cu, x.k, idx=idx, workspace=ws, stream=stream)
        if ev is not None: ev[1].record(stream)
        dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v, pos=pos, k_base=base, out=out, lse=lse,
                            workspace=ws, stream=stream)
        if ev is not None: ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = dsa.launch_count() - n0
    clk = clocks.stop()
    ms_step = max_over_ranks(world, start.elapsed_time(end)) / args.steps
    t_idx = max_over_ranks(world, statistics.mean(e[0].elapsed_time(e[1]) for e in evs))
    t_attn = max_over_ranks(world, statistics.mean(e[1].elapsed_time(e[2]) for e in evs))
    assert dsa.device_status() == 0, dsa.last_error()
    work = algorithmic_work(x)
    peaks = measured_peaks()
    attn_tf = work["attn_flops"] / (t_attn * 1e-3) / 1e12
    return {
        "metric": "DSA batched prefill tokens/s (packed causal sequences)",
        "value": job_throughput(world, x.T, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.prefill} shapes, {len(lens)} packed sequences of {lens} tokens",
                   "global_batch": world * len(lens), "seq_len": max(lens),
                   "parallelism": f"replicas{world}"},
        "kernels_ms": {"indexer_topk_varlen": t_idx, "sparse_attn": t_attn},
        "roofline": {"bound": "tensor", "kernel": "sparse MLA attention", "achieved": attn_tf,
                     "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": attn_tf / peaks["bf16"], "traffic": None,
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": attn_tf / peaks["bf16_sustained"]},
        "indexer_tflops": work["idx_flops"] / (t_idx * 1e-3) / 1e12,
        "gpu_launches": launches, "clocks": clk,
    }


def bench_bwd(args, world, rank, local):
    """Sparse attention backward: dq and dkv of one causal prefill (all rows, k
    selected latent rows each) from the forward's out / lse and a seeded dout.
    The selection is the GPU indexer's Top-k (real overlap between rows, so
    the dkv scatter sees realistic contention); it and the forward run once,
    untimed. A step is zeroing dkv plus the backward call."""
    import sparse_attention_20_b200 as dsa
    from sparse_attention_20_b200 import build as dsa_build
    if rank == 0:
        dsa_build.build()
    barrier(world)
    dsa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    x = synth.prefill_inputs(args.bwd, device=dev, seed=args.seed + rank, L=args.seq_len, T=args.rows)
    Hq, d_qk, d_v = x.q.shape[1], x.q.shape[2], x.d_v
    idx, out, lse = dsa.forward(x.q_idx, x.w, x.k_idx, x.q, x.kv, x.k, x.scale, d_v)
    dout = synth.grad_out(x, args.seed + rank)
    dq = torch.empty((x.T, Hq, d_qk), dtype=torch.float32, device=dev)
    dkv = torch.empty((x.S, d_qk), dtype=torch.float32, device=dev)
    lib = dsa.load_library()
    ws = torch.empty(int(lib.dsa_sparse_mla_attn_bwd_workspace_size(x.T, Hq, x.k)), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def step():
        dkv.zero_()
        dsa.sparse_mla_attn_bwd(x.q, x.kv, idx, out, lse, dout, x.scale, dq=dq, dkv=dkv, workspace=ws,
                                stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = dsa.launch_count() - n0
    clk = clocks.stop()
    ms_step = max_over_ranks(world, start.elapsed_time(end)) / args.steps
    assert dsa.device_status() == 0, dsa.last_error()
    # bf16 MMA flops per (row, valid slot, head): z (d_qk), dp (d_v), dq (d_qk), dkv (d_qk + d_v)
    sel = torch.clamp(x.positions().cpu().long() + 1, max=x.k)
    flops = float(sel.sum().item()) * Hq * 2 * (3 * d_qk + 2 * d_v)
    peaks = measured_peaks()
    tf = flops / (ms_step * 1e-3) / 1e12
    res = {
        "metric": "sparse MLA attention backward tokens/s (dq + dkv)",
        "value": job_throughput(world, x.T, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.bwd} causal prefill backward, L={x.S}, rows={x.T}, k={x.k}, Hq={Hq}, "
                               f"d_qk={d_qk}, d_v={d_v}; inputs larger than L2, no flush",
                   "global_batch": world, "seq_len": x.T, "parallelism": f"replicas{world}"},
        "roofline": {"bound": "tensor", "kernel": "attention backward (dkv + dq kernels, one call)",
                     "achieved": tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16"], "traffic": None,
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": tf / peaks["bf16_sustained"]},
        "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        g = torch.Generator().manual_seed(args.seed)
        rows = sorted(torch.randperm(x.T, generator=g)[:8].tolist())
        r = torch.tensor(rows, device=dev)
        t0 = time.perf_counter()
        oracle.sparse_attn_bwd(x.q[r].cpu(), x.kv.cpu(), idx[r].cpu(), x.positions()[r].cpu(),
                               torch.zeros(len(rows), dtype=torch.int32), x.scale, d_v, dout[r].cpu())
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": len(rows) / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                               "sample": f"{len(rows)} uniformly drawn query rows of the {args.bwd} "
                                         f"backward (fp64, one thread); {dt:.1f} s"}
    return res


def bench_kl(args, world, rank, local):
    """Indexer KL loss over the selected sets (the sparse training stage's
    indexer objective) and its gradient to w, q^I, k^I, for every row of one
    causal prefill. The selected sets are the GPU indexer's Top-k and lse the
    attention forward's, both computed once, untimed. A step is zeroing dk_idx
    plus the loss call."""
    import sparse_attention_20_b200 as dsa
    from sparse_attention_20_b200 import build as dsa_build
    if rank == 0:
        dsa_build.build()
    barrier(world)
    dsa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    x = synth.prefill_inputs(args.kl, device=dev, seed=args.seed + rank, L=args.seq_len, T=args.rows)
    Hq, d_qk = x.q.shape[1], x.q.shape[2]
    H_I, d_I = x.q_idx.shape[1], x.q_idx.shape[2]
    idx, _, lse = dsa.forward(x.q_idx, x.w, x.k_idx, x.q, x.kv, x.k, x.scale, x.d_v)
    dk = torch.empty((x.S, d_I), dtype=torch.float32, device=dev)
    lib = dsa.load_library()
    ws = torch.empty(int(lib.dsa_indexer_kl_workspace_size(x.T, x.k)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        dk.zero_()
        return dsa.indexer_kl(x.q, x.kv, idx, lse, x.q_idx, x.w, x.k_idx, x.scale, dk_idx=dk, workspace=ws,
                              stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    start.record(stream)
    for _ in range(args.steps):
        res = step()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = dsa.launch_count() - n0
    clk = clocks.stop()
    ms_step = max_over_ranks(world, start.elapsed_time(end)) / args.steps
    assert dsa.device_status() == 0, dsa.last_error()
    assert torch.isfinite(res[0]).all()
    # bf16 MMA flops of the head-summed probabilities: 2 Hq d_qk per (row, selected slot)
    sel = torch.clamp(x.positions().cpu().long() + 1, max=x.k)
    flops = float(sel.sum().item()) * 2 * Hq * d_qk
    peaks = measured_peaks()
    tf = flops / (ms_step * 1e-3) / 1e12
    out = {
        "metric": "indexer KL loss + gradient tokens/s (selected sets)",
        "value": job_throughput(world, x.T, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.kl} causal prefill, L={x.S}, rows={x.T}, k={x.k}, Hq={Hq}, d_qk={d_qk}, "
                               f"H_I={H_I}, d_I={d_I}; inputs larger than L2, no flush",
                   "global_batch": world, "seq_len": x.T, "parallelism": f"replicas{world}"},
        "roofline": {"bound": "tensor", "kernel": "head-summed attention probabilities + per-row loss (one call)",
                     "achieved": tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16"], "traffic": None,
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": tf / peaks["bf16_sustained"]},
        "mean_loss": float(res[0].mean().item()),
        "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        g = torch.Generator().manual_seed(args.seed)
        rows = sorted(torch.randperm(x.T, generator=g)[:8].tolist())
        r = torch.tensor(rows, device=dev)
        t0 = time.perf_counter()
        oracle.indexer_kl(x.q[r].cpu(), x.kv.cpu(), idx[r].cpu(), x.positions()[r].cpu(),
                          torch.zeros(len(rows), dtype=torch.int32), x.scale, x.q_idx[r].cpu(), x.w[r].cpu(),
                          x.k_idx.cpu())
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": len(rows) / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                               "sample": f"{len(rows)} uniformly drawn query rows of the {args.kl} KL loss "
                                         f"(fp64, one thread); {dt:.1f} s"}
    return out


def bench_mha(args, world, rank, local):
    """MLA in MHA mode on a short prefill (every causal key kept): dense causal
    attention with per-head keys and values. A step is one call."""
    import sparse_attention_20_b200 as dsa
    from sparse_attention_20_b200 import build as dsa_build
    if rank == 0:
        dsa_build.build()
    barrier(world)
    dsa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v, scale = synth.mha_inputs(args.mha, device=dev, seed=args.seed + rank, L=args.seq_len)
    T, Hq, d_h = q.shape
    S, d_hv = k.shape[0], v.shape[2]
    out = torch.empty((T, Hq, d_hv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    step = lambda: dsa.mla_mha_attn(q, k, v, scale, out=out, lse=lse, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    n0 = dsa.launch_count()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = dsa.launch_count() - n0
    clk = clocks.stop()
    ms_step = max_over_ranks(world, start.elapsed_time(end)) / args.steps
    assert dsa.device_status() == 0, dsa.last_error()
    pairs = sum(min(S, t + S - T + 1) for t in range(T))
    flops = float(pairs) * Hq * 2 * (d_h + d_hv)
    peaks = measured_peaks()
    tf = flops / (ms_step * 1e-3) / 1e12
    res = {
        "metric": "MLA MHA-mode causal attention tokens/s (short prefill)",
        "value": job_throughput(world, T, ms_step), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.mha}: L={S}, rows={T}, Hq={Hq}, d_h={d_h}, d_hv={d_hv}, dense causal; "
                               f"inputs larger than L2, no flush",
                   "global_batch": world, "seq_len": S, "parallelism": f"replicas{world}"},
        "roofline": {"bound": "tensor", "kernel": "mha_tc_kernel" if (d_h, d_hv) == (192, 128) else "mha_causal_kernel",
                     "achieved": tf,
                     "peak": peaks["bf16"], "unit": "TFLOP/s", "frac": tf / peaks["bf16"],
                     "frac_of_sustained": tf / peaks["bf16_sustained"],
                     "traffic": (profiled_traffic("mha_tc_short_prefill2k.md", "mha", MHA_SOURCES)
                                 if args.mha == "mha_short" and args.seq_len is None else None),
                     "peak_source": f"{peaks['source']} bf16 burst"},
        "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        import numpy as np
        import oracle
        g = torch.Generator().manual_seed(args.seed)
        rows = sorted(torch.randperm(T, generator=g)[:8].tolist())
        r = torch.tensor(rows)
        t0 = time.perf_counter()
        oracle.mha_attn(q.cpu()[r], k.cpu(), v.cpu(), (r + S - T).int().numpy(), np.zeros(len(rows), np.int32),
                        scale)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": len(rows) / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                               "sample": f"{len(rows)} uniformly drawn query rows of {args.mha} (fp64, one "
                                         f"thread); {dt:.1f} s"}
    return res


def main():
    args = parse()
    if args.impl == "reference":
        # rank 0 alone times the oracle; other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(bench_reference(args, world, 0)), flush=True)
        return
    world, rank, local = dist_setup(args)
    mode = (bench_bwd if args.bwd else bench_kl if args.kl else bench_mha if args.mha
            else bench_varlen if args.varlen else bench_ours)
    res = mode(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
