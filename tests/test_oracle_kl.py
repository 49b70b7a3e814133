"""Pins of the oracle's indexer KL loss (CPU only).

L_t = KL(p_t || softmax(I_t)) over row t's selected set S_t, p_t the main
attention summed over heads and L1-normalised ("Paper Breakdown:
DeepSeek-V3.2", "Continued Pre-Training (2.1.1)" table; the pages leave p
undefined, so that reading is pinned here by its consequences), with the
gradient with respect to the indexer's w, q^I and k^I (p held constant).
Pinned by: finite differences and torch autograd of a separately written
numpy/torch loss, the closed forms for w = 0 (L = log n - H(p)) and q = w = 0
(L = 0, no gradient), order invariance, non-negativity, and a planted sign
error that the finite-difference pin rejects.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _e4m3(x):
    return x.clamp(-448, 448).to(torch.float8_e4m3fn)


def _case(seed, R=3, Hq=3, d_qk=16, S=24, k=10, H_I=2, d_I=8):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(R, Hq, d_qk, generator=g).to(torch.bfloat16)
    kv = torch.randn(S, d_qk, generator=g).to(torch.bfloat16)
    qi = _e4m3(torch.randn(R, H_I, d_I, generator=g))
    ki = _e4m3(torch.randn(S, d_I, generator=g))
    w = torch.randn(R, H_I, generator=g) / math.sqrt(H_I)
    pos = np.array([S - 1 - 4 * r for r in range(R)], np.int32)
    idx = np.full((R, k), -1, np.int32)
    rng = np.random.default_rng(seed)
    for r in range(R):
        sel = rng.permutation(pos[r] + 1)[: k - 1]
        idx[r, : len(sel)] = sel
    return dict(q=q, kv=kv, idx=idx, pos=pos, base=np.zeros(R, np.int32), scale=0.25, qi=qi, w=w, ki=ki)


def _run(c):
    return oracle.indexer_kl(c["q"], c["kv"], c["idx"], c["pos"], c["base"], c["scale"],
                             c["qi"].view(torch.uint8), c["w"], c["ki"].view(torch.uint8))


def _loss(c, w, qi, ki):
    """sum_t KL(p_t || softmax(I_t)) in plain numpy fp64 (w, qi, ki real-valued)."""
    q, kv = c["q"].double().numpy(), c["kv"].double().numpy()
    total = 0.0
    for r in range(q.shape[0]):
        sel = np.array([int(i) for i in c["idx"][r] if 0 <= i <= c["pos"][r]])
        C = kv[c["base"][r] + sel]
        z = c["scale"] * (q[r] @ C.T)
        P = np.exp(z - z.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        p = P.sum(axis=0)
        p /= p.sum()
        u = qi[r] @ ki[c["base"][r] + sel].T
        I = w[r] @ np.maximum(u, 0.0)
        logsig = I - (I.max() + np.log(np.exp(I - I.max()).sum()))
        total += float((p * (np.log(p) - logsig)).sum())
    return total


def _central_diff(x, f, eps=1e-6):
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


def _reals(c):
    return c["w"].double().numpy().copy(), c["qi"].double().numpy().copy(), c["ki"].double().numpy().copy()


@pytest.mark.parametrize("seed", [1, 2])
def test_kl_matches_finite_differences(seed):
    c = _case(seed)
    loss, dw, dq, dk = _run(c)
    w, qi, ki = _reals(c)
    u = np.einsum("rjd,sd->rjs", qi, ki)
    assert np.abs(u).min() > 1e-3   # no ReLU kink within reach of the differences
    f = lambda: _loss(c, w, qi, ki)
    assert np.isclose(loss.sum(), f(), rtol=1e-12)
    assert np.allclose(dw, _central_diff(w, f), rtol=1e-6, atol=1e-8)
    assert np.allclose(dq, _central_diff(qi, f), rtol=1e-6, atol=1e-8)
    assert np.allclose(dk, _central_diff(ki, f), rtol=1e-6, atol=1e-8)
    assert np.abs(dk).max() > 1e-2


def test_kl_matches_torch_autograd():
    c = _case(3, R=4, Hq=5, d_qk=32, S=40, k=16, H_I=4, d_I=16)
    loss, dw, dq, dk = _run(c)
    w = c["w"].double().requires_grad_()
    qi = c["qi"].double().requires_grad_()
    ki = c["ki"].double().requires_grad_()
    q, kv = c["q"].double(), c["kv"].double()
    total = 0.0
    for r in range(q.shape[0]):
        sel = torch.tensor([int(i) for i in c["idx"][r] if 0 <= i <= c["pos"][r]])
        p = torch.softmax(c["scale"] * q[r] @ kv[sel].T, dim=1).sum(0)
        p = p / p.sum()
        I = w[r] @ torch.relu(qi[r] @ ki[sel].T)
        total = total + torch.nn.functional.kl_div(torch.log_softmax(I, 0), p, reduction="sum")
    total.backward()
    assert np.isclose(loss.sum(), total.item(), rtol=1e-12)
    assert np.allclose(dw, w.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dq, qi.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dk, ki.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_kl_closed_forms():
    c = _case(4)
    c["w"] = torch.zeros_like(c["w"])   # I = 0: softmax(I) uniform over the n entries
    loss, dw, dq, dk = _run(c)
    q, kv = c["q"].double().numpy(), c["kv"].double().numpy()
    for r in range(q.shape[0]):
        sel = c["idx"][r][c["idx"][r] >= 0]
        z = c["scale"] * q[r] @ kv[sel].T
        P = np.exp(z - z.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        p = P.mean(0)
        assert np.isclose(loss[r], math.log(len(sel)) + float((p * np.log(p)).sum()), rtol=1e-12)
    assert not dq.any() and not dk.any()   # w = 0 blocks the q^I, k^I paths
    c["q"] = torch.zeros_like(c["q"])   # p uniform too: no loss, no gradient
    loss, dw, dq, dk = _run(c)
    assert np.abs(loss).max() < 1e-15 and np.abs(dw).max() < 1e-15


def test_kl_order_invariance_non_negative_and_empty_rows():
    c = _case(5, R=5)
    loss, dw, dq, dk = _run(c)
    assert (loss > 0).all()
    rng = np.random.default_rng(0)
    c2 = dict(c, idx=np.stack([rng.permutation(r) for r in c["idx"]]))
    l2, dw2, dq2, dk2 = _run(c2)
    assert np.allclose(loss, l2, rtol=1e-12) and np.allclose(dk, dk2, rtol=1e-12, atol=1e-15)
    c3 = dict(c, idx=np.full_like(c["idx"], -1))
    l3, dw3, dq3, dk3 = _run(c3)
    assert not l3.any() and not dw3.any() and not dq3.any() and not dk3.any()


def test_finite_difference_pin_catches_a_sign_error():
    """dI = p - softmax(I) (the sign flipped, written here on the CPU) fails the pin."""
    c = _case(6)
    w, qi, ki = _reals(c)
    q, kv = c["q"].double().numpy(), c["kv"].double().numpy()
    bad = np.zeros_like(w)
    for r in range(q.shape[0]):
        sel = np.array([int(i) for i in c["idx"][r] if 0 <= i <= c["pos"][r]])
        z = c["scale"] * q[r] @ kv[sel].T
        P = np.exp(z - z.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        p = P.mean(0)
        u = np.maximum(qi[r] @ ki[sel].T, 0)
        I = w[r] @ u
        sig = np.exp(I - I.max())
        sig /= sig.sum()
        bad[r] = u @ (p - sig)
    fd = _central_diff(w, lambda: _loss(c, w, qi, ki))
    assert not np.allclose(bad, fd, rtol=1e-6, atol=1e-8)
