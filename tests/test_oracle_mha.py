"""Pins of the oracle's MLA MHA-mode attention (CPU only).

MHA mode gives every head its own key and value rows; MQA mode shares one
latent row c_s across heads (the bilingual paper summary's section list,
"Appendix A MHA and MQA Modes of MLA"; "Paper Breakdown: DeepSeek-V3.2",
"DSA under MLA (MQA Mode)"). Pinned by: equality with the MQA-mode oracle when
the per-head keys and values are the latent row expanded by per-head
up-projections and those are absorbed into the query and the output (integer
data, so every value is exact in bf16 and the two modes see identical logits);
torch's causal scaled_dot_product_attention; the closed form of row 0.
"""
import numpy as np
import torch

import oracle


def _bf(a):
    return torch.tensor(np.asarray(a, np.float64), dtype=torch.float32).to(torch.bfloat16)


def test_mha_mode_equals_mqa_mode_with_absorbed_projections():
    rng = np.random.default_rng(0)
    L, Hq, r_kv, r_pe, d_nope, d_v = 12, 3, 8, 4, 6, 5
    c_kv = rng.integers(-1, 2, (L, r_kv)).astype(np.float64)     # latent part of c_s
    k_pe = rng.integers(-1, 2, (L, r_pe)).astype(np.float64)     # rope part, shared by heads
    W_uk = rng.integers(-1, 2, (Hq, r_kv, d_nope)).astype(np.float64)
    W_uv = rng.integers(-1, 2, (Hq, r_kv, d_v)).astype(np.float64)
    q_nope = rng.integers(-1, 2, (L, Hq, d_nope)).astype(np.float64)
    q_pe = rng.integers(-1, 2, (L, Hq, r_pe)).astype(np.float64)
    # MHA mode: per-head keys [c_kv W_uk^h ; k_pe], values c_kv W_uv^h
    k = np.concatenate([np.einsum("sr,hrd->shd", c_kv, W_uk), np.broadcast_to(k_pe[:, None], (L, Hq, r_pe))], 2)
    v = np.einsum("sr,hrd->shd", c_kv, W_uv)
    q = np.concatenate([q_nope, q_pe], 2)
    # MQA mode: query absorbed into the latent space, one latent row per key
    q_abs = np.concatenate([np.einsum("hrd,thd->thr", W_uk, q_nope), q_pe], 2)
    c = np.concatenate([c_kv, k_pe], 1)
    pos = np.arange(L, dtype=np.int32)
    base = np.zeros(L, np.int32)
    scale = 0.3
    o_mha, l_mha = oracle.mha_attn(_bf(q), _bf(k), _bf(v), pos, base, scale)
    idx = np.tile(np.arange(L, dtype=np.int32), (L, 1))
    o_mqa, l_mqa = oracle.sparse_attn(_bf(q_abs), _bf(c), idx, pos, base, scale, r_kv)
    assert np.allclose(l_mha, l_mqa, rtol=1e-13, atol=1e-13)
    # MHA output = the MQA latent output expanded by W_uv of each head
    assert np.allclose(o_mha, np.einsum("thr,hrd->thd", o_mqa, W_uv), rtol=1e-12, atol=1e-12)


def test_mha_matches_torch_causal_sdpa():
    g = torch.Generator().manual_seed(1)
    L, Hq, d_h, d_hv = 40, 4, 24, 16
    q = torch.randn(L, Hq, d_h, generator=g).to(torch.bfloat16)
    k = torch.randn(L, Hq, d_h, generator=g).to(torch.bfloat16)
    v = torch.randn(L, Hq, d_hv, generator=g).to(torch.bfloat16)
    out, lse = oracle.mha_attn(q, k, v, np.arange(L, dtype=np.int32), np.zeros(L, np.int32), 0.2)
    qd, kd, vd = (x.double().transpose(0, 1) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=0.2)
    z = 0.2 * qd @ kd.transpose(1, 2)
    z = z.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    assert np.allclose(out, ref.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(lse, torch.logsumexp(z, -1).transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_mha_row0_closed_form_and_offsets():
    g = torch.Generator().manual_seed(2)
    q = torch.randn(3, 2, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(10, 2, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(10, 2, 4, generator=g).to(torch.bfloat16)
    out, lse = oracle.mha_attn(q, k, v, np.array([0, 0, 3], np.int32), np.array([0, 5, 5], np.int32), 0.5)
    for r, b in ((0, 0), (1, 5)):
        assert np.array_equal(out[r], v[b].double().numpy())
        assert np.allclose(lse[r], 0.5 * (q[r].double() * k[b].double()).sum(-1).numpy(), rtol=1e-14)
    o2, l2 = oracle.mha_attn(q[2:], k[5:], v[5:], np.array([3], np.int32), np.array([0], np.int32), 0.5)
    assert np.array_equal(o2[0], out[2]) and np.array_equal(l2[0], lse[2])
