"""Parity of MLA MHA-mode causal attention (CUDA, through the C ABI) with the
fp64 CPU oracle on B200. The kernel rounds the probabilities to bf16 before
the P.V MMAs, like the sparse forward, so the attention parity rule applies:
rel-L2 <= 1e-2 and max-abs <= 3e-2 on out, |lse - oracle| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dsa_build.build()
    dsa.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()
    assert dsa.device_status() == 0


def _check(q, k, v, scale, rows=None):
    out, lse = dsa.mla_mha_attn(q, k, v, scale)
    torch.cuda.synchronize()
    T, S = q.shape[0], k.shape[0]
    rows = list(range(T)) if rows is None else rows
    r = torch.tensor(rows)
    pos = (r + S - T).int().numpy()
    ro, rl = oracle.mha_attn(q.cpu()[r], k.cpu(), v.cpu(), pos, np.zeros(len(rows), np.int32), scale)
    o = out.cpu()[r].double().numpy()
    l = lse.cpu()[r].double().numpy()
    rel = np.linalg.norm(o - ro) / np.linalg.norm(ro)
    assert rel <= 1e-2 and np.abs(o - ro).max() <= 3e-2, (rel, np.abs(o - ro).max())
    assert np.abs(l - rl).max() <= 1e-3


@pytest.mark.parametrize("L,T", [(300, None), (300, 100), (1, None), (129, 1)])
def test_mha_small_heads_all_rows(L, T):
    """d_h = d_hv = 64, 4 heads; ragged query tiles, a tail prefill, one token."""
    _check(*synth.mha_inputs("mha_small", device="cuda", seed=0, L=L, T=T))


@pytest.mark.parametrize("L,Hq", [(777, 8), (200, 3)])
def test_mha_192_128_all_rows(L, Hq):
    _check(*synth.mha_inputs("mha_short", device="cuda", seed=1, L=L, Hq=Hq))


@pytest.mark.parametrize("L,T,Hq", [(1000, 300, 4), (129, 1, 2), (256, 256, 1)])
def test_mha_192_128_tail_rows(L, T, Hq):
    """The last T query rows of L tokens (pos[t] = t + L - T): query tiles
    start past key tiles, the single-row case, and exact 128-row tiles."""
    _check(*synth.mha_inputs("mha_short", device="cuda", seed=3, L=L, T=T, Hq=Hq))


def test_mha_short_prefill_sampled_rows():
    """The 2048-token, 128-head short prefill bench.py --mha times."""
    q, k, v, scale = synth.mha_inputs("mha_short", device="cuda", seed=2)
    _check(q, k, v, scale, rows=synth.sample_rows(q.shape[0], 2048, 24, seed=2))
