"""Parity of the CUDA path (through the C ABI) with the CPU oracle on B200.

Sizes: small cases run the oracle on every row (several tiles, ragged tails);
the full-size workloads (32K, 128K prefill, 64-sequence decode) check sampled
rows in the exact launch configuration bench.py times.
"""
import os

import numpy as np
import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build
from parity import check_attention, check_indexer, host_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dsa_build.build()
    dsa.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()
    assert dsa.device_status() == 0


def _run(x, **kw):
    idx, out, lse = dsa.forward(x.q_idx, x.w, x.k_idx, x.q, x.kv, x.k, x.scale, x.d_v, pos=x.pos,
                                k_base=x.k_base, **kw)
    torch.cuda.synchronize()
    return idx, out, lse


def _take(t, rows):
    return t[torch.tensor(rows, device=t.device)].cpu()


# ----------------------------------------------------------- small, full check

def test_tiny_indexer_bit_exact_and_attention_all_rows():
    x = synth.prefill_inputs("tiny", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=True, h=h)
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)


def test_forward_equals_separate_calls():
    x = synth.prefill_inputs("tiny", device="cuda", seed=1)
    idx, out, lse = _run(x)
    idx2 = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    out2, lse2 = dsa.sparse_mla_attn(x.q, x.kv, idx2, x.scale, x.d_v, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    assert torch.equal(torch.sort(idx, 1)[0], torch.sort(idx2, 1)[0])
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("L,k", [(333, 64), (130, 200)])
def test_small_realistic_all_rows(L, k):
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=2, L=L, overrides=dict(k=k))
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=False, h=h)
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)


def test_integer_indexer_bit_exact_d128():
    x = synth.prefill_inputs("prefill32k_int", device="cuda", seed=3, L=1500,
                             overrides=dict(k=300))
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    torch.cuda.synchronize()
    rows = list(range(0, x.T, 3)) + [x.T - 1]
    check_indexer(x, _take(idx, rows), rows, exact=True)


def test_explicit_pos_and_k_base_packed_rows():
    """Queries of three sequences in one packed cache, with ragged lengths."""
    x = synth.decode_inputs("decode", device="cuda", seed=4, B=5, ctx=[1, 17, 300, 129, 2050],
                            overrides=dict(k=128))
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=False, h=h)
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)


def test_decode_integer_inputs_bit_exact():
    x = synth.decode_inputs("decode", device="cuda", seed=5, B=6, ctx=[40, 1000, 3000, 64, 65, 5000],
                            overrides=dict(indexer="int", k=256))
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    check_indexer(x, idx.cpu(), list(range(x.T)), exact=True)


# Up to 2048 query rows per call take the decode form (every key of a row
# scored into a dense score row, then a per-row select); more rows take the
# chunked form (chunk Top-k under a sampled threshold, then a merge). A test
# reaches the chunked form by repeating each query row `reps` times.
DECODE_FORM_ROWS = 2048


def _repeat_queries(x, reps):
    if reps == 1:
        return x
    r = lambda t: t.repeat_interleave(reps, dim=0)
    return synth.DSAInputs(x.config, r(x.q_idx), r(x.w), x.k_idx, r(x.q), x.kv, r(x.pos), r(x.k_base),
                           x.k, x.scale, x.d_v, meta=x.meta)


def _check_repeated(x, reps, idx):
    rows = list(range(0, x.T, reps))
    assert reps == 1 or x.T > DECODE_FORM_ROWS
    check_indexer(x, _take(idx, rows), rows, exact=True)
    if reps > 1:   # every copy of a query row selects the same set
        v = idx.view(-1, reps, x.k)
        assert torch.equal(v, v[:, :1].expand_as(v))


@pytest.mark.parametrize("reps", [1, 700])
def test_decode_multi_chunk_integer_bit_exact(reps):
    """Rows of one to five 8192-key chunks; integer FP8-exact inputs make many
    scores tie across chunks."""
    x = synth.decode_inputs("decode", device="cuda", seed=9, B=5, ctx=[8193, 16384, 20000, 40000, 9000],
                            overrides=dict(indexer="int", k=2048))
    x = _repeat_queries(x, reps)
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    _check_repeated(x, reps, idx)


@pytest.mark.parametrize("reps", [1, 700])
def test_decode_threshold_overshoot_still_exact(reps):
    """Only keys on a regular grid (s mod 4096 < 128) are non-zero: a threshold
    sampled on that grid keeps far fewer than k keys (chunked form), and most
    16-key groups tie at score 0, so the group-maximum filter keeps more pairs
    than fit in shared memory (decode form). The rows must still get their
    exact Top-k (ties at score 0 go to the lowest s)."""
    x = synth.decode_inputs("decode", device="cuda", seed=10, B=3, ctx=[30000, 50000, 12000],
                            overrides=dict(indexer="int", k=2048))
    base = x.bases().cpu().long()
    pos = x.positions().cpu().long()
    keep = torch.zeros(x.k_idx.shape[0], dtype=torch.bool)
    for b, p in zip(base.tolist(), pos.tolist()):
        s = torch.arange(p + 1)
        keep[b + s[(s % 4096) < 128]] = True
    x.k_idx[~keep.to(x.k_idx.device)] = 0
    x = _repeat_queries(x, reps)
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    _check_repeated(x, reps, idx)


def test_decode_all_scores_equal_takes_the_lowest_positions():
    """Every key row identical: all scores tie, so each row's Top-k is its k
    lowest positions (both the staged and the global-memory selections)."""
    x = synth.decode_inputs("decode", device="cuda", seed=17, B=4, ctx=[9000, 16000, 20000, 70000],
                            overrides=dict(indexer="int", k=2048))
    x.k_idx[:] = x.k_idx[0]
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    want = torch.arange(x.k, dtype=torch.int32, device="cuda").expand(x.T, x.k)
    assert torch.equal(idx, want)
    check_indexer(x, idx.cpu(), list(range(x.T)), exact=True)


def test_decode_row_longer_than_a_score_row_is_exact():
    """A row of more than 2^20 keys is not scored into the workspace; the
    select recomputes its scores and takes the exact Top-k (integer inputs)."""
    x = synth.decode_inputs("decode", device="cuda", seed=18, B=2, ctx=[1100000, 30000],
                            overrides=dict(indexer="int", k=2048))
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    check_indexer(x, idx.cpu(), list(range(x.T)), exact=True)


def test_k_at_least_L_selects_every_past_token():
    x = synth.prefill_inputs("tiny", device="cuda", seed=6, L=100, overrides=dict(k=128))
    idx, out, lse = _run(x)
    for t in range(x.T):
        row = idx[t].cpu().numpy()
        assert sorted(row[: t + 1].tolist()) == list(range(t + 1))
        assert (row[t + 1:] == -1).all()
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), list(range(x.T)))


def test_k_equals_one_and_single_row():
    x = synth.prefill_inputs("tiny", device="cuda", seed=7, overrides=dict(k=1))
    pos = torch.tensor([200], dtype=torch.int32, device="cuda")
    idx = dsa.indexer_topk(x.q_idx[200:201].contiguous(), x.w[200:201].contiguous(), x.k_idx, 1,
                           pos=pos)
    torch.cuda.synchronize()
    full = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, 1)
    torch.cuda.synchronize()
    assert idx[0, 0].item() == full[200, 0].item()
    check_indexer(x, full.cpu(), list(range(x.T)), exact=True)


@pytest.mark.parametrize("splits", [2, 5, 16])
def test_attention_splits_and_lse_merge_cuda_core(splits):
    """CUDA-core kernel (Hq = 4, d_qk = 80) with each row's set split into
    parts and merged by log-sum-exp; parts of short rows are empty."""
    x = synth.prefill_inputs("tiny", device="cuda", seed=8, L=200, overrides=dict(k=96))
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    out1, lse1 = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, 1)
    outs, lses = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, splits)
    torch.cuda.synchronize()
    rows = list(range(x.T))
    check_attention(x, idx.cpu(), outs.cpu(), lses.cpu(), rows)
    assert (out1.float() - outs.float()).abs().max().item() < 2e-2


@pytest.mark.parametrize("splits", [2, 3, 5, 16])
def test_decode_split_tensor_core_matches_oracle(splits):
    """The decode variant on the tensor-core kernel: each row's selected set
    split across clusters (ranges of whole 64-entry chunks; with short rows
    and 16 parts some parts are empty), parts merged by log-sum-exp. Every row
    against the oracle, and against the unsplit kernel."""
    x = synth.decode_inputs("decode", device="cuda", seed=13, B=9,
                            ctx=[9000, 1, 63, 64, 65, 700, 2047, 131072, 40000])
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    out1, lse1 = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, 1, pos=x.pos, k_base=x.k_base)
    outs, lses = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, splits, pos=x.pos,
                                           k_base=x.k_base)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_attention(x, idx.cpu(), outs.cpu(), lses.cpu(), rows, h=h)
    assert (out1.float() - outs.float()).abs().max().item() < 2e-2
    assert (lse1 - lses).abs().max().item() < 1e-3


def test_decode_64_sequences_split_launch():
    """The 64-sequence decode step with its rows split in two (every row
    against the oracle) and the library's own choice of parts."""
    x = synth.decode_inputs("decode", device="cuda", seed=0)
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    for splits in (0, 2):
        out, lse = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, splits, pos=x.pos,
                                             k_base=x.k_base)
        torch.cuda.synchronize()
        check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)


def test_invalid_entries_are_ignored():
    """-1 padding and s > pos inside the read range do not contribute."""
    x = synth.prefill_inputs("tiny", device="cuda", seed=9)
    t = 100
    idx = torch.full((x.T, x.k), -1, dtype=torch.int32, device="cuda")
    idx[t, :4] = torch.tensor([5, 250, 7, -1], dtype=torch.int32)
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v)
    torch.cuda.synchronize()
    ref_idx = torch.full_like(idx, -1)
    ref_idx[t, :2] = torch.tensor([5, 7], dtype=torch.int32)
    check_attention(x, ref_idx[[t]].cpu(), out[[t]].cpu(), lse[[t]].cpu(), [t])


# ----------------------------------------------------- full-size workloads

def _sampled(T, k, n):
    return synth.sample_rows(T, k, n, seed=0)


def test_prefill4k_all_rows_indexer_sampled_attention():
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    check_indexer(x, idx.cpu(), rows, exact=False)
    srows = _sampled(x.T, x.k, 48)
    check_attention(x, _take(idx, srows), _take(out, srows), _take(lse, srows), srows)


# Full-size configurations: 256 sampled query rows (rows 0, k-1, k, L-1 and a
# seeded random set), every one checked for both the indexer and attention.
N_SAMPLED = 256


def test_prefill32k_integer_indexer_bit_exact_sampled():
    x = synth.prefill_inputs("prefill32k_int", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = _sampled(x.T, x.k, N_SAMPLED)
    assert len(rows) == N_SAMPLED
    h = host_inputs(x, rows)
    check_indexer(x, _take(idx, rows), rows, exact=True, h=h)
    check_attention(x, _take(idx, rows), _take(out, rows), _take(lse, rows), rows, h=h)


def test_tail_prefill_last_rows_of_a_longer_sequence():
    """Chunked prefill: the last 700 query rows of a 6000-token sequence (pos
    implied as t + S - T, no explicit pos): streaming indexer and tensor-core
    attention with every row's range starting past its own index."""
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=12, L=6000, T=700)
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    check_indexer(x, idx.cpu(), rows, exact=False)
    srows = rows[::50] + [x.T - 1]
    check_attention(x, _take(idx, srows), _take(out, srows), _take(lse, srows), srows)


def test_prefill_threshold_overshoot_falls_back_exactly():
    """Causal prefill through the streaming tensor-core indexer with keys that
    are non-zero only on every 32nd 128-key tile (where the threshold is
    sampled): far fewer than k keys pass the sampled threshold, the select
    kernel's exact recompute must give the oracle's Top-k (ties at score 0 go
    to the lowest s)."""
    x = synth.prefill_inputs("prefill32k_int", device="cuda", seed=11, L=12288)
    s = torch.arange(x.S, device=x.k_idx.device)
    x.k_idx[(s // 128) % 32 != 0] = 0
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    torch.cuda.synchronize()
    rows = _sampled(x.T, x.k, 48) + [x.T - 2, 4096, 4097, 8191]
    check_indexer(x, _take(idx, rows), rows, exact=True)


def test_prefill_select_ties_take_the_radix_path_exactly():
    """The prefill Top-k select ranks a row's candidates through a histogram
    over their key range and falls back to the radix select when every
    candidate ties or the bin holding the k-th entry holds more than 128
    entries. Keys repeating four distinct rows give four distinct scores per
    query row (boundary bins of hundreds of ties); keys all equal give rows
    whose candidates all tie. Either way the result is the oracle's Top-k
    (ties to the lowest s)."""
    for distinct, seed in ((4, 13), (1, 14)):
        x = synth.prefill_inputs("prefill32k_int", device="cuda", seed=seed, L=6144)
        s = torch.arange(x.S, device=x.k_idx.device)
        x.k_idx[:] = x.k_idx[s % distinct]
        idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
        torch.cuda.synchronize()
        rows = _sampled(x.T, x.k, 24) + [x.k, x.k + 1, 4095, x.T - 1]
        check_indexer(x, _take(idx, rows), rows, exact=True)
        if distinct == 1:
            # every score equal: the lowest k positions, in ascending order
            want = torch.arange(x.k, dtype=torch.int32)
            for t in (x.k, 4095, x.T - 1):
                assert torch.equal(idx[t].cpu(), want)


def test_prefill32k_sampled():
    x = synth.prefill_inputs("prefill32k", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = _sampled(x.T, x.k, N_SAMPLED)
    assert len(rows) == N_SAMPLED
    h = host_inputs(x, rows)
    check_indexer(x, _take(idx, rows), rows, exact=False, h=h)
    check_attention(x, _take(idx, rows), _take(out, rows), _take(lse, rows), rows, h=h)


def test_prefill128k_sampled():
    """The 128K prefill in bench.py's launch configuration (one indexer call
    over all 131072 rows, one attention call)."""
    x = synth.prefill_inputs("prefill128k", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = _sampled(x.T, x.k, N_SAMPLED)
    assert len(rows) == N_SAMPLED
    h = host_inputs(x, rows)
    check_indexer(x, _take(idx, rows), rows, exact=False, h=h)
    check_attention(x, _take(idx, rows), _take(out, rows), _take(lse, rows), rows, h=h)
    del x, idx, out, lse
    torch.cuda.empty_cache()


def test_decode_64_sequences():
    x = synth.decode_inputs("decode", device="cuda", seed=0)
    idx, out, lse = _run(x)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=False, h=h)
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)


def test_streaming_indexer_rows_are_ascending_and_repeatable():
    """The streaming indexer writes each row in ascending s, the same on every
    call (so attention over it sums in a fixed order and repeats bit for bit)."""
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=14, L=3000)
    a = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    b = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    n = torch.clamp(x.positions().long() + 1, max=x.k)
    v = a.long()
    valid = torch.arange(x.k, device="cuda")[None, :] < n[:, None]
    assert ((v[:, 1:] > v[:, :-1]) | ~valid[:, 1:]).all()
    o1, l1 = dsa.sparse_mla_attn(x.q, x.kv, a, x.scale, x.d_v)
    o2, l2 = dsa.sparse_mla_attn(x.q, x.kv, b, x.scale, x.d_v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_phase_timing_reports_the_indexer_phases():
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=15)
    dsa.phase_timing(True)
    try:
        dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
        torch.cuda.synchronize()
        ph = dsa.phase_times()
    finally:
        dsa.phase_timing(False)
    assert ph["scores"] > 0 and ph["threshold"] > 0 and ph["select"] > 0
    dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    torch.cuda.synchronize()
    assert all(v == 0 for v in dsa.phase_times().values())   # off: nothing recorded


def test_decode_rows_beyond_the_fused_threshold_path():
    """Rows longer than 24 chunks of 8192 keys keep their sampled scores in
    global memory (shorter rows in shared memory); both kinds in one call,
    integer inputs, bit-exact."""
    x = synth.decode_inputs("decode", device="cuda", seed=16, B=3, ctx=[200000, 9000, 300001],
                            overrides=dict(indexer="int", k=2048))
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    check_indexer(x, idx.cpu(), list(range(x.T)), exact=True)
