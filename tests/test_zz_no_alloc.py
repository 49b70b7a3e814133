"""dsa_indexer_topk_noalloc: the indexer entry point for callers that cannot
give the library device memory (no workspace argument; its scratch is an
array the library holds). Called through the C ABI and compared with
dsa_indexer_topk on the same inputs, twice in a row, because the shared
scratch keeps the previous call's contents, and with the CPU oracle.
Collected last on purpose."""
import ctypes

import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from parity import check_indexer
from sparse_attention_20_b200 import build as dsa_build

STATIC_MAX_S = 4 << 20


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_S_beyond_its_scratch():
    dsa_build.build()
    lib = dsa.load_library()
    fake = ctypes.c_void_p(0x10000)
    rc = lib.dsa_indexer_topk_noalloc(fake, fake, fake, None, None, 4, STATIC_MAX_S + 1, 8, 128,
                                      2048, fake, None)
    assert rc == -2 and b"scratch" in lib.dsa_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["decode", "prefill"])
def test_noalloc_matches_workspace_entry_point_twice(case):
    dsa_build.build()
    lib = dsa.load_library()
    if case == "decode":
        x = synth.decode_inputs("decode", device="cuda", seed=21, B=12,
                                ctx=[131072, 9000, 70000, 8192, 120001, 33333, 4096, 100000,
                                     65536, 12345, 98765, 131071])
    else:
        # integer-valued FP8 inputs: every score is exact, so any two correct
        # Top-k implementations select the same set
        x = synth.prefill_inputs("prefill32k_int", device="cuda", seed=22, L=4096)
    assert x.S <= STATIC_MAX_S
    T, H_I, d_I = x.q_idx.shape
    ref = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        got = torch.full_like(ref, -7)
        rc = lib.dsa_indexer_topk_noalloc(_p(x.q_idx), _p(x.w), _p(x.k_idx), _p(x.pos),
                                          _p(x.k_base), T, x.S, H_I, d_I, x.k, _p(got), stream)
        assert rc == 0, lib.dsa_last_error()
        torch.cuda.synchronize()
        # each row is a set: compare in sorted order
        assert torch.equal(torch.sort(got, dim=1)[0], torch.sort(ref, dim=1)[0])
    assert dsa.device_status() == 0
    # and against the oracle: exact sets on integer inputs, the tolerance rule
    # on realistic ones (every row of the decode case, sampled prefill rows)
    rows = list(range(T)) if case == "decode" else synth.sample_rows(T, x.k, 64, seed=3)
    r = torch.tensor(rows, device=got.device)
    check_indexer(x, got[r].cpu(), rows, exact=(case == "prefill"))


@pytest.mark.gpu
def test_noalloc_many_rows_over_few_keys():
    """T = 70000 query rows over S = 64 keys: the scratch holds 65536 score
    rows, so the call works through the rows in blocks of at most 65535 (the
    grid's y limit); every row must still get its exact Top-k."""
    dsa_build.build()
    dsa.load_library()
    x = synth.decode_inputs("decode", device="cuda", seed=23, B=1, ctx=[64],
                            overrides=dict(indexer="int", k=16))
    T = 70000
    q_idx = x.q_idx.expand(T, -1, -1).contiguous()
    w = synth.integers((T, x.w.shape[1]), -2, 2, 23, "noalloc_rows", "w", "cuda")
    pos = synth.integers((T,), 0, 63, 23, "noalloc_rows", "pos", "cuda").to(torch.int32)
    ref = dsa.indexer_topk(q_idx, w, x.k_idx, x.k, pos=pos)
    got = dsa.indexer_topk_noalloc(q_idx, w, x.k_idx, x.k, pos=pos)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    assert torch.equal(torch.sort(got, dim=1)[0], torch.sort(ref, dim=1)[0])
    rows = [0, 1, 65534, 65535, 65536, T - 1] + list(range(100, T, 7919))
    r = torch.tensor(rows, device="cuda")
    h = dict(q_idx=q_idx[r].cpu().numpy(), w=w[r].cpu().numpy(), k_idx=x.k_idx.cpu().numpy(),
             pos=pos[r].cpu().numpy(), base=torch.zeros(len(rows), dtype=torch.int32).numpy())
    check_indexer(x, got[r].cpu(), rows, exact=True, h=h)
