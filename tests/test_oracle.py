"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: the FP8/BF16 format
definitions and torch's casts, hand-derived worked examples (tests/golden/),
integer brute force, algebraic identities of the index score, a full
lexicographic sort and the rank definition of Top-k, attention closed forms,
torch's SDPA on gathered rows, order invariance, the dense-attention special
case k >= L, and the log-sum-exp merge of split sets.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth


def _e4m3(vals):
    return synth.to_e4m3_bytes(torch.tensor(vals, dtype=torch.float32)).numpy()


# ------------------------------------------------------------------ decoding

def test_e4m3_table_matches_format_definition():
    t = oracle.e4m3_table()
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0          # largest finite
    assert t[0x01] == 2.0 ** -9                              # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9                          # largest subnormal
    assert t[0x08] == 2.0 ** -6                              # smallest normal
    assert t[0x3C] == 1.5 and t[0x40] == 2.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])       # S.1111.111
    assert t[0x00] == 0.0 and t[0x80] == 0.0
    assert np.isfinite(t[[c for c in range(256) if c & 0x7F != 0x7F]]).all()


def test_e4m3_table_matches_torch_cast():
    t = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(t) == nan).all()
    assert (t[~nan] == ref[~nan]).all()


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 100).to(torch.bfloat16)
    x[:4] = torch.tensor([0.0, -0.0, 1.0, -3.5]).to(torch.bfloat16)
    got = oracle.bf16_to_f64(x)
    assert (got == x.to(torch.float64).numpy()).all()


# ------------------------------------------------------------- index score

def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_indexer_worked_examples(golden_dir):
    g = _golden(golden_dir, "indexer_worked_example.json")
    for case in g["cases"]:
        q = _e4m3(case["q"])
        keys = _e4m3(case["keys"])
        n = len(case["keys"])
        sc = oracle.indexer_scores(q, np.array(case["w"], np.float32), keys, n)
        assert sc.tolist() == case["scores"], case["name"]
        for k, want in case["topk"].items():
            assert oracle.topk(sc, int(k)).tolist() == want, (case["name"], k)


def _brute_int64(q_idx, w, k_idx, t, n, base=0):
    """Integer brute force: e4m3 integers -> int64 dots, ReLU, integer weights."""
    tab = oracle.e4m3_table()
    qi = tab[q_idx[t]].astype(np.int64)                 # [H_I, d_I]
    ki = tab[k_idx[base:base + n]].astype(np.int64)     # [n, d_I]
    wi = w[t].astype(np.int64)
    dots = ki @ qi.T                                     # [n, H_I]
    return (np.maximum(dots, 0) * wi[None, :]).sum(axis=1)


def test_indexer_int64_brute_force_tiny():
    x = synth.prefill_inputs("tiny", seed=3)
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    assert (w == np.round(w)).all()
    for t in range(0, x.T, 7):
        got = oracle.indexer_scores(q_idx[t], w[t], k_idx, t + 1)
        want = _brute_int64(q_idx, w, k_idx, t, t + 1)
        assert (got.astype(np.int64) == want).all() and (got == want).all()


def test_indexer_scores_rows_int64_brute_force_packed():
    """The many-rows form (rows in parallel, ragged pos, packed k_base) equals
    integer brute force row by row and leaves NaN past each row's pos."""
    x = synth.decode_inputs("decode", seed=4, B=4, ctx=[1, 60, 300, 129],
                            overrides=dict(H_I=4, d_I=32, indexer="int", k=16))
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    pos, base = x.pos.numpy(), x.k_base.numpy()
    got = oracle.indexer_scores_rows(q_idx, w, k_idx, pos, base)
    assert got.shape == (4, int(pos.max()) + 1)
    for b in range(4):
        n = int(pos[b]) + 1
        want = _brute_int64(q_idx, w, k_idx[base[b]:], b, n)
        assert (got[b, :n] == want).all()
        assert np.isnan(got[b, n:]).all()


def test_indexer_relu_identity():
    """ReLU(x) - ReLU(-x) = x: negating head j changes I by exactly w_j (q_j . k)."""
    x = synth.prefill_inputs("tiny", seed=5)
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    tab = oracle.e4m3_table()
    t, n = 200, 201
    base = oracle.indexer_scores(q_idx[t], w[t], k_idx, n).astype(np.float64)
    for j in range(q_idx.shape[1]):
        qn = q_idx[t].copy()
        qn[j] ^= 0x80                                    # e4m3 sign flip
        flipped = oracle.indexer_scores(qn, w[t], k_idx, n).astype(np.float64)
        dot = tab[k_idx[:n]] @ tab[q_idx[t, j]]
        assert (base - flipped == w[t, j] * dot).all()


def test_indexer_weight_scaling_and_head_permutation():
    x = synth.prefill_inputs("tiny", seed=6)
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    t, n = 150, 151
    base = oracle.indexer_scores(q_idx[t], w[t], k_idx, n)
    assert (oracle.indexer_scores(q_idx[t], 2 * w[t], k_idx, n) == 2 * base).all()
    assert (oracle.indexer_scores(q_idx[t], -w[t], k_idx, n) == -base).all()
    perm = np.array([2, 0, 3, 1])
    assert (oracle.indexer_scores(q_idx[t][perm], w[t][perm], k_idx, n) == base).all()


def test_indexer_unit_vector_keys_closed_form():
    """k_s = c e_{d(s)}: I_s = sum_j w_j ReLU(c q_j[d(s)])."""
    H_I, d_I, n = 3, 16, 40
    rng = np.random.default_rng(0)
    qv = rng.integers(-4, 5, size=(H_I, d_I)).astype(np.float32)
    wv = rng.integers(-2, 3, size=H_I).astype(np.float32)
    keys = np.zeros((n, d_I), np.float32)
    c = np.where(np.arange(n) % 2 == 0, 2.0, -0.5)
    dsel = (np.arange(n) * 5) % d_I
    keys[np.arange(n), dsel] = c
    sc = oracle.indexer_scores(_e4m3(qv), wv, _e4m3(keys), n)
    want = (wv[None, :] * np.maximum(c[:, None] * qv[:, dsel].T, 0)).sum(axis=1)
    assert (sc == want.astype(np.float32)).all()


def test_indexer_k_base_offsets_packed_sequences():
    """A row of a packed cache scores the same as the sequence alone."""
    x = synth.decode_inputs("decode", seed=1, B=3, ctx=[50, 70, 33],
                            overrides=dict(H_I=4, d_I=32, indexer="int", Hq=4, d_qk=80, d_v=64))
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    base = x.k_base.numpy()
    for b, n in enumerate(x.meta["ctx"]):
        packed = oracle.indexer_scores(q_idx[b], w[b], k_idx, n, k_base=int(base[b]))
        alone = oracle.indexer_scores(q_idx[b], w[b], k_idx[base[b]:base[b] + n], n)
        assert (packed == alone).all()
        assert (packed == _brute_int64(q_idx, w, k_idx, b, n, base=int(base[b]))).all()


# ----------------------------------------------------------------- Top-k

def _topk_by_rank_definition(sc, k):
    """s is selected iff fewer than k entries rank strictly before it."""
    n = sc.size
    sel = []
    for s in range(n):
        before = np.sum(sc > sc[s]) + np.sum((sc == sc[s]) & (np.arange(n) < s))
        if before < k:
            sel.append(s)
    return sorted(sel)


@pytest.mark.parametrize("n,k", [(1, 4), (5, 5), (37, 8), (200, 32), (513, 100)])
def test_topk_matches_full_sort_and_rank_definition(n, k):
    rng = np.random.default_rng(n * 31 + k)
    for values in (rng.standard_normal(n), rng.integers(-3, 4, size=n)):   # distinct / many ties
        sc = values.astype(np.float32)
        got = oracle.topk(sc, k)
        order = np.lexsort((np.arange(n), -sc.astype(np.float64)))
        want = np.full(k, -1, np.int32)
        want[: min(k, n)] = order[:k]
        assert (got == want).all()
        assert sorted(got[got >= 0].tolist()) == _topk_by_rank_definition(sc, k)


def test_topk_all_equal_takes_lowest_indices():
    assert oracle.topk(np.zeros(10, np.float32), 4).tolist() == [0, 1, 2, 3]


def test_indexer_topk_rows_causal_and_padding():
    x = synth.prefill_inputs("tiny", seed=7)
    idx = oracle.indexer_topk(x.q_idx, x.w, x.k_idx, x.positions(), x.bases(), x.k)
    for t in range(x.T):
        row = idx[t]
        valid = row[row >= 0]
        assert len(valid) == min(x.k, t + 1)
        assert (row[len(valid):] == -1).all()
        assert valid.max() <= t and len(set(valid.tolist())) == len(valid)
        if t + 1 <= x.k:
            assert sorted(valid.tolist()) == list(range(t + 1))


def test_indexer_topk_rows_match_brute_force():
    x = synth.prefill_inputs("tiny", seed=8)
    q_idx, k_idx, w = x.q_idx.numpy(), x.k_idx.numpy(), x.w.numpy()
    rows = [40, 100, 255]
    idx = oracle.indexer_topk(q_idx, w, k_idx, x.positions(), x.bases(), x.k, rows=rows)
    for r, t in enumerate(rows):
        sc = _brute_int64(q_idx, w, k_idx, t, t + 1).astype(np.float32)
        assert sorted(idx[r].tolist()) == _topk_by_rank_definition(sc, x.k)


# ------------------------------------------------------------- attention

def _bf16(a):
    return torch.tensor(np.asarray(a, np.float64), dtype=torch.float32).to(torch.bfloat16)


def test_attention_two_keys_closed_form(golden_dir):
    g = _golden(golden_dir, "attention_two_keys.json")
    q = _bf16(g["q"])[None]
    kv = _bf16(g["kv"])
    idx = np.array([[0, 1]], np.int32)
    out, lse = oracle.sparse_attn(q, kv, idx, [1], [0], g["scale"], g["d_v"])
    assert np.allclose(out[0], g["out"], rtol=1e-15, atol=1e-18)
    assert np.allclose(lse[0], g["lse"], rtol=1e-15, atol=0)


def test_attention_single_key_and_t0():
    x = synth.prefill_inputs("tiny", seed=9)
    q = oracle.bf16_to_f64(x.q)
    kv = oracle.bf16_to_f64(x.kv)
    idx = np.full((1, x.k), -1, np.int32)
    for s in (0, 17):
        idx[0, 0] = s
        out, lse = oracle.sparse_attn(x.q[[30]], x.kv, idx, [30], [0], x.scale, x.d_v)
        assert (out[0] == np.broadcast_to(kv[s, : x.d_v], out[0].shape)).all()
        z = x.scale * (q[30] @ kv[s])
        assert np.allclose(lse[0], z, rtol=1e-14, atol=1e-14)


def test_attention_zero_query_is_uniform_mean():
    x = synth.prefill_inputs("tiny", seed=10)
    q0 = torch.zeros_like(x.q[:1])
    sel = np.array([[3, 9, 27, 81, 100, -1, -1, 250]], np.int32)  # 250 > pos: ignored
    out, lse = oracle.sparse_attn(q0, x.kv, sel, [200], [0], x.scale, x.d_v)
    kv = oracle.bf16_to_f64(x.kv)
    mean = kv[[3, 9, 27, 81, 100], : x.d_v].mean(axis=0)
    assert np.allclose(out[0], mean[None, :], rtol=1e-13, atol=1e-15)
    assert np.allclose(lse[0], math.log(5), rtol=1e-14)


def test_attention_matches_torch_sdpa_on_gathered_rows():
    x = synth.prefill_inputs("prefill4k", seed=11, L=96, overrides=dict(k=48))
    rng = np.random.default_rng(0)
    t = 90
    sel = rng.permutation(t + 1)[: x.k].astype(np.int32)
    out, lse = oracle.sparse_attn(x.q[[t]], x.kv, sel[None], [t], [0], x.scale, x.d_v)
    q = x.q[t].to(torch.float64)                        # [Hq, d_qk]
    K = x.kv[torch.from_numpy(sel).long()].to(torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], K[None].expand(q.shape[0], -1, -1),
        K[None, :, : x.d_v].expand(q.shape[0], -1, -1), scale=x.scale)[:, 0]
    ref_lse = torch.logsumexp(x.scale * (q @ K.T), dim=1)
    assert np.allclose(out[0], ref.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(lse[0], ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_order_invariance():
    x = synth.prefill_inputs("tiny", seed=12)
    idx = oracle.indexer_topk(x.q_idx, x.w, x.k_idx, x.positions(), x.bases(), x.k)
    rows = [5, 64, 255]
    o1, l1 = oracle.sparse_attn(x.q, x.kv, idx, x.positions(), x.bases(), x.scale, x.d_v, rows)
    rng = np.random.default_rng(1)
    shuffled = np.stack([rng.permutation(r) for r in idx])
    o2, l2 = oracle.sparse_attn(x.q, x.kv, shuffled, x.positions(), x.bases(), x.scale, x.d_v,
                                rows)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)
    assert np.allclose(l1, l2, rtol=1e-13, atol=1e-14)


def test_dsa_with_k_at_least_L_equals_dense_causal_mqa():
    x = synth.prefill_inputs("tiny", seed=13, L=48, overrides=dict(k=64))
    idx = oracle.indexer_topk(x.q_idx, x.w, x.k_idx, x.positions(), x.bases(), x.k)
    out, lse = oracle.sparse_attn(x.q, x.kv, idx, x.positions(), x.bases(), x.scale, x.d_v)
    for t in range(x.T):
        d_out, d_lse = oracle.dense_attn_row(x.q[t], x.kv, t, 0, x.scale, x.d_v)
        assert np.allclose(out[t], d_out, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse[t], d_lse, rtol=1e-12, atol=1e-12)


def test_lse_merge_of_split_set_equals_whole():
    x = synth.prefill_inputs("tiny", seed=14)
    idx = oracle.indexer_topk(x.q_idx, x.w, x.k_idx, x.positions(), x.bases(), x.k)
    t = 250
    whole_o, whole_l = oracle.sparse_attn(x.q, x.kv, idx, x.positions(), x.bases(), x.scale,
                                          x.d_v, [t])
    parts = [idx[t, :5], idx[t, 5:19], idx[t, 19:]]
    po, pl = [], []
    for p in parts:
        row = np.full((1, x.k), -1, np.int32)
        row[0, : len(p)] = p
        o, l = oracle.sparse_attn(x.q[[t]], x.kv, row, [t], [0], x.scale, x.d_v)
        po.append(o[0])
        pl.append(l[0])
    empty = np.full((1, x.k), -1, np.int32)
    o, l = oracle.sparse_attn(x.q[[t]], x.kv, empty, [t], [0], x.scale, x.d_v)
    assert np.isneginf(l).all() and (o == 0).all()
    po.append(o[0])
    pl.append(l[0])
    mo, ml = oracle.lse_merge(np.stack(po), np.stack(pl))
    assert np.allclose(mo, whole_o[0], rtol=1e-12, atol=1e-14)
    assert np.allclose(ml, whole_l[0], rtol=1e-13, atol=1e-14)


def test_decode_row_equals_prefill_row_on_same_data():
    """Query n-1 of a length-n prefill and a decode query over the same n cached rows."""
    pre = synth.prefill_inputs("tiny", seed=15, L=120)
    n = 100
    # pack [60 unrelated rows | first n rows of the prefill sequence]
    junk = synth.prefill_inputs("tiny", seed=99, L=60)
    k_cache = torch.cat([junk.k_idx, pre.k_idx[:n]])
    kv_cache = torch.cat([junk.kv, pre.kv[:n]])
    idx_pre = oracle.indexer_topk(pre.q_idx, pre.w, pre.k_idx, pre.positions(), pre.bases(),
                                  pre.k, rows=[n - 1])
    idx_dec = oracle.indexer_topk(pre.q_idx[[n - 1]], pre.w[[n - 1]], k_cache, [n - 1], [60],
                                  pre.k)
    assert (idx_pre == idx_dec).all()
    o1, l1 = oracle.sparse_attn(pre.q[[n - 1]], pre.kv, idx_pre, [n - 1], [0], pre.scale, pre.d_v)
    o2, l2 = oracle.sparse_attn(pre.q[[n - 1]], kv_cache, idx_dec, [n - 1], [60], pre.scale,
                                pre.d_v)
    assert (o1 == o2).all() and (l1 == l2).all()


# ------------------------------------------- planted mistakes fail the pins

def test_pins_catch_a_dropped_relu_and_a_sign_error(golden_dir):
    """Mutants of the score formula (written here, on the CPU) fail the worked example."""
    g = _golden(golden_dir, "indexer_worked_example.json")["cases"][0]
    q = np.array(g["q"], np.float64)
    k = np.array(g["keys"], np.float64)
    w = np.array(g["w"], np.float64)
    no_relu = (k @ q.T * w).sum(axis=1)
    flipped = (np.maximum(k @ q.T, 0) * -w).sum(axis=1)
    transposed = (np.maximum(k @ q.T[::-1], 0) * w).sum(axis=1)
    for mutant in (no_relu, flipped, transposed):
        assert mutant.tolist() != g["scores"]
