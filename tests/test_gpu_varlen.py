"""Batched (variable-length) prefill: packed causal sequences through
dsa_indexer_topk_varlen (the streaming tensor-core indexer per sequence) and
the attention with per-row pos / k_base, against the oracle."""
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


def _varlen(x):
    cu = x.meta["cu"]
    idx = dsa.indexer_topk_varlen(x.q_idx, x.w, x.k_idx, cu, cu, x.k)
    pos, base = dsa.varlen_rows(cu, cu, x.q.device)
    assert torch.equal(pos, x.pos) and torch.equal(base, x.k_base)
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v, pos=pos, k_base=base)
    torch.cuda.synchronize()
    return idx, out, lse


def test_varlen_integer_indexer_bit_exact():
    x = synth.varlen_prefill_inputs("prefill32k_int", device="cuda", seed=3, lens=[700, 2600, 4500],
                                    overrides=dict(k=1024))
    idx, _, _ = _varlen(x)
    rows = list(range(0, x.T, 7)) + [699, 700, 3299, 3300, x.T - 1]
    check_indexer(x, idx[torch.tensor(rows, device=idx.device)].cpu(), rows, exact=True)


def test_varlen_realistic_indexer_and_attention():
    x = synth.varlen_prefill_inputs("prefill4k", device="cuda", seed=4, lens=[300, 3000, 2100])
    idx, out, lse = _varlen(x)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=False, h=h)
    srows = rows[::97] + [299, 300, 3299, x.T - 1]
    t = torch.tensor(srows, device=idx.device)
    check_attention(x, idx[t].cpu(), out[t].cpu(), lse[t].cpu(), srows)


def test_varlen_equals_one_call_per_sequence():
    x = synth.varlen_prefill_inputs("prefill4k", device="cuda", seed=5, lens=[2500, 4100])
    idx, _, _ = _varlen(x)
    cu = x.meta["cu"]
    for b in range(len(cu) - 1):
        a, e = cu[b], cu[b + 1]
        ref = dsa.indexer_topk(x.q_idx[a:e].contiguous(), x.w[a:e].contiguous(),
                               x.k_idx[a:e].contiguous(), x.k)
        torch.cuda.synchronize()
        assert torch.equal(torch.sort(idx[a:e], 1)[0], torch.sort(ref, 1)[0])
