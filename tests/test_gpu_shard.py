"""The multi-GPU split of the path, run rank by rank on one GPU: the query rows
of one causal prefill and the sequences of a decode batch are cut into the
library's contiguous ranges (dsa_partition_prefill_rows /
dsa_partition_decode_seqs), each range runs as its own forward call on the
slices bench.py hands a rank, and the concatenated results must equal one
call over everything, bit for bit (the ranks exchange nothing). The attention
is compared at one part per row: with few rows the library's own choice
splits rows into parts, and that count depends on how many rows a call has
(parts change the rounding, not the result beyond it)."""
import os
import sys

import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build
from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dsa_build.build()
    dsa.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()
    assert dsa.device_status() == 0


def _fwd(x):
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    out, lse = dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, 1, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    return idx, out, lse


@pytest.mark.parametrize("name,kw,world", [
    ("prefill4k", dict(L=6000), 3),                     # streaming tensor-core indexer per range
    ("prefill4k", dict(L=3000, T=2500), 4),             # a tail prefill split again
    ("tiny", dict(L=256), 5),                           # general indexer, CUDA-core attention
    ("decode", dict(B=7, ctx=[9000, 300, 20000, 4096, 70000, 2048, 12345]), 3),
])
def test_split_equals_one_call_bit_for_bit(name, kw, world):
    x = synth.make_inputs(name, device="cuda", seed=31, **kw)
    idx, out, lse = _fwd(x)
    parts = [bench.shard_inputs(x, world, r) for r in range(world)]
    covered = []
    for p in parts:
        a, b = p.meta["rows"]
        covered.append((a, b))
        if b == a:
            continue
        pi, po, pl = _fwd(p)
        assert torch.equal(pi, idx[a:b]), (name, a, b)
        assert torch.equal(po, out[a:b]) and torch.equal(pl, lse[a:b]), (name, a, b)
    assert covered[0][0] == 0 and covered[-1][1] == x.T
    assert all(covered[i][1] == covered[i + 1][0] for i in range(world - 1))
