"""Pins of the oracle's sparse attention backward (CPU only).

The backward is the gradient of sum(dout * out) of u_t = Attn(h_t, {c_s}) over
the selected latent rows ("Paper Breakdown: DeepSeek-V3.2", section 2, and
the "Sparse Training" row of its continued pre-training table, which trains
the main model through the selected entries). It is pinned by things other
than its own formula: central finite differences of a separately written
fp64 forward, torch autograd on dense causal MQA (k >= L), a closed form for
identical keys, and invariants (order of idx, linearity in dout, zero dout).
"""
import numpy as np
import pytest
import torch

import oracle


def _case(seed, R=3, Hq=2, d_qk=12, d_v=8, S=20, k=8):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(R, Hq, d_qk, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, d_qk, generator=g).to(torch.bfloat16)
    dout = torch.randn(R, Hq, d_v, generator=g).to(torch.bfloat16)
    pos = np.array([S - 1 - 3 * r for r in range(R)], np.int32)
    idx = np.full((R, k), -1, np.int32)
    rng = np.random.default_rng(seed)
    for r in range(R):
        sel = rng.permutation(pos[r] + 1)[: k - 2]
        idx[r, : len(sel)] = sel
        idx[r, k - 1] = pos[r] + 1 if pos[r] + 1 < S else -1   # beyond pos: not a candidate
    return q, kv, dout, idx, pos, np.zeros(R, np.int32), 0.3, d_v


def _f64(t):
    return t.to(torch.float64).numpy()


def _loss(q, kv, dout, idx, pos, base, scale, d_v):
    """sum(dout * out) with out the sparse MQA attention, in plain numpy fp64."""
    total = 0.0
    for r in range(q.shape[0]):
        sel = [int(i) for i in idx[r] if 0 <= i <= pos[r]]
        if not sel:
            continue
        C = kv[base[r] + np.array(sel)]
        z = scale * (q[r] @ C.T)
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        total += float((dout[r] * (p @ C[:, :d_v])).sum())
    return total


def test_numpy_forward_matches_oracle_forward():
    q, kv, dout, idx, pos, base, scale, d_v = _case(1)
    out, _ = oracle.sparse_attn(q, kv, idx, pos, base, scale, d_v)
    assert np.isclose(_loss(_f64(q), _f64(kv), _f64(dout), idx, pos, base, scale, d_v),
                      float((out * _f64(dout)).sum()), rtol=1e-13)


def _central_diff(x, f, eps=1e-5):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        hi = f()
        x[i] = old - eps
        lo = f()
        x[i] = old
        g[i] = (hi - lo) / (2 * eps)
    return g


@pytest.mark.parametrize("seed", [2, 3])
def test_backward_matches_finite_differences(seed):
    q, kv, dout, idx, pos, base, scale, d_v = _case(seed)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, dout)
    qf, kvf, gf = _f64(q), _f64(kv), _f64(dout)
    f = lambda: _loss(qf, kvf, gf, idx, pos, base, scale, d_v)
    assert np.allclose(dq, _central_diff(qf, f), rtol=1e-7, atol=1e-8)
    assert np.allclose(dkv, _central_diff(kvf, f), rtol=1e-7, atol=1e-8)
    assert np.abs(dkv).max() > 0.1   # the case has gradient to check


def test_backward_dense_equals_torch_autograd_of_causal_mqa():
    """k >= L selects every s <= t: the gradients of dense causal MQA."""
    T, Hq, d_qk, d_v, scale = 10, 3, 16, 8, 0.25
    g = torch.Generator().manual_seed(4)
    q = torch.randn(T, Hq, d_qk, generator=g).to(torch.bfloat16)
    kv = torch.randn(T, d_qk, generator=g).to(torch.bfloat16)
    dout = torch.randn(T, Hq, d_v, generator=g).to(torch.bfloat16)
    idx = np.tile(np.arange(16, dtype=np.int32)[::-1], (T, 1))   # every key, reversed, 6 past T
    pos = np.arange(T, dtype=np.int32)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, np.zeros(T, np.int32), scale, d_v, dout)
    qa = q.to(torch.float64).requires_grad_()
    kva = kv.to(torch.float64).requires_grad_()
    z = scale * torch.einsum("thd,sd->ths", qa, kva)
    mask = torch.arange(T)[None, :] > torch.arange(T)[:, None]
    p = torch.softmax(z.masked_fill(mask[:, None, :], float("-inf")), dim=-1)
    out = torch.einsum("ths,sc->thc", p, kva[:, :d_v])
    (out * dout.to(torch.float64)).sum().backward()
    assert np.allclose(dq, qa.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dkv, kva.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_backward_identical_keys_closed_form():
    """All selected rows equal: p is uniform, dz = 0, so dq = 0 and each row gets dout/n."""
    R, Hq, d_qk, d_v, S = 2, 2, 8, 4, 12
    g = torch.Generator().manual_seed(5)
    q = torch.randn(R, Hq, d_qk, generator=g).to(torch.bfloat16)
    kv = torch.randn(1, d_qk, generator=g).to(torch.bfloat16).expand(S, d_qk).contiguous()
    dout = torch.randn(R, Hq, d_v, generator=g).to(torch.bfloat16)
    idx = np.array([[1, 4, 7, 9, -1], [0, 2, 3, 5, 11]], np.int32)
    pos = np.array([9, 11], np.int32)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, np.zeros(R, np.int32), 0.5, d_v, dout)
    assert np.abs(dq).max() < 1e-14
    want = np.zeros((S, d_qk))
    gd = _f64(dout)
    for r, n in ((0, 4), (1, 5)):
        for s in idx[r][idx[r] >= 0]:
            want[s, :d_v] += gd[r].sum(axis=0) / n
    assert np.allclose(dkv, want, rtol=1e-13, atol=1e-14)


def test_backward_order_invariance_linearity_zero_and_empty_rows():
    q, kv, dout, idx, pos, base, scale, d_v = _case(6)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, dout)
    rng = np.random.default_rng(0)
    shuffled = np.stack([rng.permutation(r) for r in idx])
    dq2, dkv2 = oracle.sparse_attn_bwd(q, kv, shuffled, pos, base, scale, d_v, dout)
    assert np.allclose(dq, dq2, rtol=1e-12, atol=1e-14)
    assert np.allclose(dkv, dkv2, rtol=1e-12, atol=1e-14)
    dq3, dkv3 = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, dout * 2)   # exact in bf16
    assert np.allclose(dq3, 2 * dq, rtol=1e-13, atol=1e-15)
    assert np.allclose(dkv3, 2 * dkv, rtol=1e-13, atol=1e-15)
    dq0, dkv0 = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, torch.zeros_like(dout))
    assert not dq0.any() and not dkv0.any()
    none = np.full_like(idx, -1)
    none[0, 0] = pos[0] + 5   # beyond pos only
    dqn, dkvn = oracle.sparse_attn_bwd(q, kv, none, pos, base, scale, d_v, dout)
    assert not dqn.any() and not dkvn.any()


def test_backward_k_base_offsets_the_scatter():
    """Row t of a packed sequence scatters into rows k_base + s of the shared cache."""
    q, kv, dout, idx, pos, base, scale, d_v = _case(7)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, dout)
    pad = torch.randn(5, kv.shape[1]).to(torch.bfloat16)
    dq2, dkv2 = oracle.sparse_attn_bwd(q, torch.cat([pad, kv]), idx, pos, base + 5, scale, d_v, dout)
    assert (dq == dq2).all()
    assert not dkv2[:5].any() and (dkv2[5:] == dkv).all()


def test_finite_difference_pin_catches_a_dropped_term():
    """A backward without the -D term (written here, on the CPU) fails the same pin."""
    q, kv, dout, idx, pos, base, scale, d_v = _case(8)
    qf, kvf, gf = _f64(q), _f64(kv), _f64(dout)
    bad = np.zeros_like(qf)
    for r in range(qf.shape[0]):
        sel = [int(i) for i in idx[r] if 0 <= i <= pos[r]]
        C = kvf[np.array(sel)]
        z = scale * (qf[r] @ C.T)
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        bad[r] = scale * (p * (gf[r] @ C[:, :d_v].T)) @ C
    fd = _central_diff(qf, lambda: _loss(qf, kvf, gf, idx, pos, base, scale, d_v))
    assert not np.allclose(bad, fd, rtol=1e-7, atol=1e-8)


def test_backward_column_sums_of_dkv():
    """sum_s p_s = 1 and sum_s dz_s = 0 per row and head, so summed over the cache
    rows dkv[:, :d_v] = sum over rows and heads of dout, and dkv[:, d_v:] sums to 0."""
    q, kv, dout, idx, pos, base, scale, d_v = _case(9, R=4, Hq=3, d_qk=16, d_v=8, S=30, k=12)
    dq, dkv = oracle.sparse_attn_bwd(q, kv, idx, pos, base, scale, d_v, dout)
    col = dkv.sum(axis=0)
    assert np.allclose(col[:d_v], _f64(dout).sum(axis=(0, 1)), rtol=1e-12, atol=1e-12)
    assert np.allclose(col[d_v:], 0.0, atol=1e-12)
