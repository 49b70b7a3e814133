"""Parity of the indexer KL loss and its gradient (CUDA, through the C ABI)
with the fp64 CPU oracle on B200.

Inputs: synth tensors, a score-free seeded selection (synth.selection) or
every causal key (the dense warm-up form); the GPU takes the GPU attention
forward's lse for the same idx, the oracle computes its own. Tolerance: the
GPU forms the head-summed probabilities from bf16 MMAs with fp32
accumulation and the forward's fp32 lse (off by up to ~1e-3 on the
tensor-core path), the index scores exactly in fp32 products with fp32 sums,
and the log-sum-exp in fp32; per row |loss - oracle| <= 5e-3 max(1, |loss|),
and rel-L2 <= 1e-2 on dw, dq_idx and dk_idx. Element by element, every entry
of dw, dq_idx and dk_idx is within 1e-2 of its tensor's largest magnitude
(the per-element error is the same relative error on the larger terms of its
sum).
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


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _gpu(x, idx, **kw):
    _, lse = dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v, pos=x.pos, k_base=x.k_base)
    res = dsa.indexer_kl(x.q, x.kv, idx, lse, x.q_idx, x.w, x.k_idx, x.scale, pos=x.pos, k_base=x.k_base, **kw)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    return [r.cpu().numpy() for r in res]


def _oracle(x, idx, rows=None):
    r = slice(None) if rows is None else rows
    return oracle.indexer_kl(x.q[r].cpu(), x.kv.cpu(), idx[r], x.positions().cpu()[r], x.bases().cpu()[r],
                             x.scale, x.q_idx[r].cpu(), x.w[r].cpu(), x.k_idx.cpu())


def _elementwise(a, b):
    """max |a - b| over the tensor, as a fraction of max |b|."""
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _check(g, o, with_dk=True):
    loss, dw, dq, dk = g
    rl, rdw, rdq, rdk = o
    assert np.all(np.abs(loss - rl) <= 5e-3 * np.maximum(1.0, np.abs(rl))), np.abs(loss - rl).max()
    assert _rel(dw, rdw) < 1e-2 and _rel(dq, rdq) < 1e-2, (_rel(dw, rdw), _rel(dq, rdq))
    assert _elementwise(dw, rdw) <= 1e-2 and _elementwise(dq, rdq) <= 1e-2, (_elementwise(dw, rdw),
                                                                          _elementwise(dq, rdq))
    if with_dk:
        assert _rel(dk, rdk) < 1e-2, _rel(dk, rdk)
        assert _elementwise(dk, rdk) <= 1e-2, _elementwise(dk, rdk)


@pytest.mark.parametrize("L,k", [(256, 32), (200, 96), (160, 256)])
def test_kl_tiny_shapes_all_rows(L, k):
    """H_I = 4, d_I = 32, Hq = 4, d_qk = 80; k = 256 >= L is the dense warm-up form."""
    x = synth.prefill_inputs("tiny", device="cuda", seed=0, L=L, overrides=dict(k=k))
    idx = synth.selection(x.positions().cpu(), x.k, 0)
    _check(_gpu(x, idx.cuda()), _oracle(x, idx))


@pytest.mark.parametrize("L,k,T", [(300, 64, None), (2500, 2048, 6)])
def test_kl_mla_shapes(L, k, T):
    x = synth.prefill_inputs("prefill4k", device="cuda", seed=1, L=L, T=T, overrides=dict(k=k))
    idx = synth.selection(x.positions().cpu(), x.k, 1)
    _check(_gpu(x, idx.cuda()), _oracle(x, idx))


def test_kl_multi_pass_and_empty_rows():
    x = synth.prefill_inputs("tiny", device="cuda", seed=2, L=150)
    idx = synth.selection(x.positions().cpu(), x.k, 2)
    idx[[0, 9, 149]] = -1
    ws = torch.empty(3 * 64 * 4, dtype=torch.uint8, device="cuda")   # three rows per pass
    g = _gpu(x, idx.cuda(), workspace=ws)
    g1 = _gpu(x, idx.cuda())
    for a, b in zip(g[:3], g1[:3]):
        assert np.array_equal(a, b)
    assert not g[0][[0, 9, 149]].any() and not g[1][[0, 9, 149]].any() and not g[2][[0, 9, 149]].any()
    _check(g, _oracle(x, idx))


def test_kl_prefill32k_sampled_rows():
    """The 32K prefill as bench.py --kl runs it (the GPU Top-k as the selected
    sets is replaced here by a seeded selection the oracle can take): loss, dw
    and dq_idx of sampled rows against the oracle row by row."""
    x = synth.prefill_inputs("prefill32k", device="cuda", seed=3)
    idx = synth.selection(x.positions().cpu(), x.k, 3)
    loss, dw, dq, dk = _gpu(x, idx.cuda())
    rows = synth.sample_rows(x.T, x.k, 6, seed=3)
    rl, rdw, rdq, _ = _oracle(x, idx, rows)
    _check((loss[rows], dw[rows], dq[rows], None), (rl, rdw, rdq, None), with_dk=False)
    assert np.isfinite(dk).all() and np.abs(dk).max() > 0
