"""Parity of the sparse MQA attention backward (CUDA, through the C ABI) with
the fp64 CPU oracle on B200.

Inputs: synth tensors, a score-free seeded selection (synth.selection) and a
seeded dout; the GPU backward takes the GPU forward's out / lse, the oracle
computes its own. Tolerance: the kernels round p and scale*dz to bf16 before
their MMAs (relative error 2^-9 per element, averaging out over the k
selected rows) and accumulate in fp32, so the relative L2 error of dq and
dkv sits near 3e-3; the bound is 1e-2 on the whole tensor and 2e-2 per
query row of dq. Element by element: the same rounding bounds the error of
one element by a few 2^-9 of the larger terms of its sum, so every element
of dq and dkv must be within 1e-2 of the largest magnitude of its tensor
(dq: of its query row's, 2e-2).
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


def _gpu(x, idx, dout, **kw):
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v, pos=x.pos, k_base=x.k_base)
    dq, dkv = dsa.sparse_mla_attn_bwd(x.q, x.kv, idx, out, lse, dout, x.scale, pos=x.pos,
                                      k_base=x.k_base, **kw)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    return dq.cpu().numpy(), dkv.cpu().numpy()


def _case(name, seed, **kw):
    x = synth.prefill_inputs(name, device="cuda", seed=seed, **kw)
    idx = synth.selection(x.positions().cpu(), x.k, seed)
    return x, idx, synth.grad_out(x, seed)


def _oracle(x, idx, dout):
    return oracle.sparse_attn_bwd(x.q.cpu(), x.kv.cpu(), idx, x.positions().cpu(), x.bases().cpu(),
                                  x.scale, x.d_v, dout.cpu())


def _elementwise(a, b, frac):
    """max |a - b| over the tensor, as a fraction of max |b|."""
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _check(dq, dkv, rdq, rdkv):
    assert _rel(dq, rdq) < 1e-2 and _rel(dkv, rdkv) < 1e-2, (_rel(dq, rdq), _rel(dkv, rdkv))
    per_row = [_rel(dq[t], rdq[t]) for t in range(dq.shape[0]) if np.abs(rdq[t]).max() > 0]
    assert max(per_row) < 2e-2, max(per_row)
    assert _elementwise(dq, rdq, 1e-2) <= 1e-2, _elementwise(dq, rdq, 1e-2)
    assert _elementwise(dkv, rdkv, 1e-2) <= 1e-2, _elementwise(dkv, rdkv, 1e-2)
    per_row_max = [_elementwise(dq[t], rdq[t], 2e-2) for t in range(dq.shape[0]) if np.abs(rdq[t]).max() > 0]
    assert max(per_row_max) <= 2e-2, max(per_row_max)
    assert not dkv[np.abs(rdkv).max(axis=1) == 0].any()   # rows nobody selected stay zero


@pytest.mark.parametrize("name,L,k", [("tiny", 256, 32), ("tiny", 200, 96)])
def test_bwd_small_shapes_all_rows(name, L, k):
    """Hq=4 (padded head tile), d_qk=80 (a 16-column tail), k below and above 64."""
    x, idx, dout = _case(name, 0, L=L, overrides=dict(k=k))
    dq, dkv = _gpu(x, idx.cuda(), dout)
    _check(dq, dkv, *_oracle(x, idx, dout))


@pytest.mark.parametrize("L,k,T", [(300, 64, None), (2500, 2048, 6)])
def test_bwd_mla_shapes(L, k, T):
    """Hq=128, d_qk=576, d_v=512; short rows (fewer candidates than k) and full 2048 rows."""
    x, idx, dout = _case("prefill4k", 1, L=L, T=T, overrides=dict(k=k))
    dq, dkv = _gpu(x, idx.cuda(), dout)
    _check(dq, dkv, *_oracle(x, idx, dout))


def test_bwd_multi_pass_and_empty_rows():
    """A workspace of 3 rows forces several passes; rows without entries give dq = 0."""
    x, idx, dout = _case("tiny", 2, L=150)
    idx[[0, 7, 149]] = -1
    ws = torch.empty(3 * 16 * (64 * 2 + 4), dtype=torch.uint8, device="cuda")
    dq, dkv = _gpu(x, idx.cuda(), dout, workspace=ws)
    dq1, dkv1 = _gpu(x, idx.cuda(), dout)
    assert np.array_equal(dq, dq1)
    assert np.allclose(dkv, dkv1, rtol=1e-5, atol=1e-6)
    assert not dq[[0, 7, 149]].any()
    _check(dq, dkv, *_oracle(x, idx, dout))


def test_bwd_dkv_accumulates():
    x, idx, dout = _case("tiny", 3, L=128)
    d = idx.cuda()
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, d, x.scale, x.d_v)
    _, dkv = dsa.sparse_mla_attn_bwd(x.q, x.kv, d, out, lse, dout, x.scale)
    _, dkv2 = dsa.sparse_mla_attn_bwd(x.q, x.kv, d, out, lse, dout, x.scale, dkv=dkv.clone())
    torch.cuda.synchronize()
    assert torch.allclose(dkv2, 2 * dkv, rtol=1e-5, atol=1e-6)


def test_bwd_prefill32k_sampled_rows_and_column_sums():
    """The 32K-token prefill backward as bench.py --bwd runs it (k = 2048 per row):
    dq of sampled rows against the oracle row by row, and dkv against the column
    sums every backward obeys (sum_s p_s = 1, sum_s dz_s = 0): the columns < d_v
    of dkv sum to the sum of dout over rows and heads, the rest to 0."""
    x, idx, dout = _case("prefill32k", 4)
    dq, dkv = _gpu(x, idx.cuda(), dout)
    rows = synth.sample_rows(x.T, x.k, 6, seed=4)
    pos = x.positions().cpu()[rows]
    rdq, _ = oracle.sparse_attn_bwd(x.q[rows].cpu(), x.kv.cpu(), idx[rows], pos,
                                    torch.zeros(len(rows), dtype=torch.int32), x.scale, x.d_v,
                                    dout[rows].cpu())
    assert _rel(dq[rows], rdq) < 1e-2
    assert _elementwise(dq[rows], rdq, 1e-2) <= 1e-2
    col = dkv.astype(np.float64).sum(axis=0)
    want = dout.double().sum(dim=(0, 1)).cpu().numpy()
    mag = np.abs(dkv).astype(np.float64).sum(axis=0)
    assert np.all(np.abs(col[: x.d_v] - want) <= 1e-3 * mag[: x.d_v] + 1e-2)
    assert np.all(np.abs(col[x.d_v:]) <= 1e-3 * mag[x.d_v:] + 1e-2)


def test_bwd_prefill32k_dkv_of_sampled_rows_element_by_element():
    """dkv at the 32K shapes checked in full: the backward of 64 sampled query
    rows alone (each with its 2048 selected latent rows of the 32K cache), so
    dkv holds exactly those rows' scatter-adds and the oracle can form the
    same sum; compared element by element and by rel-L2, with dq."""
    x, idx, dout = _case("prefill32k", 5)
    rows = synth.sample_rows(x.T, x.k, 64, seed=5)
    r = torch.tensor(rows, device="cuda")
    q, o_idx, g = x.q[r].contiguous(), idx[rows], dout[r].contiguous()
    pos = x.positions()[r].contiguous()
    d_idx = o_idx.cuda()
    out, lse = dsa.sparse_mla_attn(q, x.kv, d_idx, x.scale, x.d_v, pos=pos)
    dq, dkv = dsa.sparse_mla_attn_bwd(q, x.kv, d_idx, out, lse, g, x.scale, pos=pos)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    rdq, rdkv = oracle.sparse_attn_bwd(q.cpu(), x.kv.cpu(), o_idx, pos.cpu(),
                                       torch.zeros(len(rows), dtype=torch.int32), x.scale, x.d_v, g.cpu())
    _check(dq.cpu().numpy(), dkv.cpu().numpy(), rdq, rdkv)
