"""The debug build (libdsa_debug.so, -DDSA_DEBUG) on B200: its device-side
checks of the index sets read clean on correct runs (the tiny and 4K
configurations, prefill and decode), and count exactly the entries a caller
plants that the attention ignores or never reads (entries past pos[t], -1
inside the read range, valid entries past it, repeats) without faulting.
The library under test is swapped in for the release one for the module."""
import numpy as np
import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build
from parity import check_attention, check_indexer, host_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _debug_lib():
    dsa_build.build()
    path = dsa_build.build(debug=True)
    saved = dsa._lib
    dsa._lib = None
    lib = dsa.load_library(path)
    assert lib.dsa_debug_build() == 1
    dsa.debug_counters(reset=True)
    assert dsa.device_status() == 0
    yield
    torch.cuda.synchronize()
    dsa._lib = saved


def _clean():
    torch.cuda.synchronize()
    assert dsa.device_status() == 0, dsa.last_error()
    assert all(v == 0 for v in dsa.debug_counters().values())


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("prefill4k", {}),
                                     ("decode", dict(B=5, ctx=[300, 9000, 2049, 64, 20000]))])
def test_debug_build_reads_clean_on_correct_runs(name, kw):
    x = synth.make_inputs(name, device="cuda", seed=41, **kw)
    idx, out, lse = dsa.forward(x.q_idx, x.w, x.k_idx, x.q, x.kv, x.k, x.scale, x.d_v, pos=x.pos,
                                k_base=x.k_base)
    _clean()
    rows = list(range(0, x.T, max(1, x.T // 64)))
    r = torch.tensor(rows, device="cuda")
    h = host_inputs(x, rows)
    check_indexer(x, idx[r].cpu(), rows, exact=(name == "tiny"), h=h)
    check_attention(x, idx[r].cpu(), out[r].cpu(), lse[r].cpu(), rows, h=h)
    # the split decode form and the no-workspace indexer are checked too
    dsa.sparse_mla_attn_split(x.q, x.kv, idx, x.scale, x.d_v, 3, pos=x.pos, k_base=x.k_base)
    dsa.indexer_topk_noalloc(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    _clean()


def test_debug_build_counts_planted_entries():
    x = synth.prefill_inputs("tiny", device="cuda", seed=42)
    k = x.k                      # 32
    idx = torch.full((x.T, k), -1, dtype=torch.int32)
    t = 100                      # n = 101 candidates, m = 32 entries read
    idx[t, :6] = torch.tensor([5, 250, 7, -1, 7, 9])   # 250 > pos, -1 inside, 7 repeated
    idx[t, 28] = 3               # a valid entry at slot 28 < m: fine
    u = 10                       # n = 11 candidates, m = 11 entries read
    idx[u, :11] = torch.arange(11)
    idx[u, 12] = 4               # valid entry past m: never read
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, idx.cuda(), x.scale, x.d_v)
    torch.cuda.synchronize()
    st = dsa.device_status()
    assert st == -6, st
    got = dsa.debug_counters()
    # row t: 250 beyond pos; one -1 inside; 7 repeated; the other rows are
    # all -1 inside their read range (m - 0 valid entries each)
    pad = sum(min(k, tt + 1) for tt in range(x.T) if tt not in (t, u)) + (32 - 6 - 1) + 1
    assert got["beyond_pos"] == 1
    assert got["duplicate"] == 1
    assert got["dropped"] == 1
    assert got["pad_inside"] == pad
    assert got["bad_page"] == 0 and got["selection"] == 0
    # the planted entries are ignored: row t attends {5, 7, 7, 9, 3}
    ref = torch.full_like(idx, -1)
    ref[t, :5] = torch.tensor([5, 7, 7, 9, 3])
    check_attention(x, ref[[t]], out[[t]].cpu(), lse[[t]].cpu(), [t])
    assert dsa.device_status() == 0        # the status word was cleared
