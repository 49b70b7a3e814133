"""Host-side helpers (no GPU): the page-pool builder places every key of every
sequence where the block table says, the varlen row maps give each packed row
its sequence's range, the score-free selection is a valid set per row, and the
MHA-mode inputs have their shapes."""
import torch

import synth
import sparse_attention_20_b200 as dsa


def test_page_caches_put_every_key_where_the_table_says():
    x = synth.decode_inputs("decode", B=4, ctx=[100, 300, 64, 129], overrides=dict(k=32))
    for ps in (64, 128):
        kp, vp, bt, seq = synth.page_caches(x, ps, seed=1)
        assert kp.shape[0] % ps == 0 and vp.shape[0] == kp.shape[0]
        used = []
        for b in range(x.T):
            n = int(x.positions()[b]) + 1
            b0 = int(x.bases()[b])
            rows = [int(bt[b, s // ps]) * ps + s % ps for s in range(n)]
            assert torch.equal(kp[rows], x.k_idx[b0:b0 + n])
            assert torch.equal(vp[rows], x.kv[b0:b0 + n])
            npg = (n + ps - 1) // ps
            used += bt[b, :npg].tolist()
            assert (bt[b, npg:] == -1).all()       # unused entries
        assert len(set(used)) == len(used)          # no page shared by two sequences
        assert torch.equal(seq, torch.arange(x.T, dtype=torch.int32))


def test_varlen_rows_and_inputs_agree():
    lens = [5, 1, 7]
    x = synth.varlen_prefill_inputs("tiny", lens=lens)
    assert x.meta["cu"] == [0, 5, 6, 13]
    pos, base = dsa.varlen_rows(x.meta["cu"], x.meta["cu"], "cpu")
    assert torch.equal(pos, x.pos) and torch.equal(base, x.k_base)
    assert pos.tolist() == [0, 1, 2, 3, 4, 0, 0, 1, 2, 3, 4, 5, 6]
    # suffix-aligned tails: 2 of 5 keys in the first sequence, 3 of 7 in the second
    pos2, base2 = dsa.varlen_rows([0, 2, 5], [0, 5, 12], "cpu")
    assert pos2.tolist() == [3, 4, 4, 5, 6] and base2.tolist() == [0, 0, 5, 5, 5]


def test_selection_rows_are_valid_sets():
    """synth.selection: min(k, pos+1) distinct in-range entries first, -1 after,
    for rows shorter and longer than k, an empty row and a one-key row."""
    import numpy as np
    pos = np.array([-1, 0, 5, 63, 64, 1000, 4095])
    for k in (1, 64, 100):
        sel = synth.selection(pos, k, seed=3).numpy()
        assert sel.shape == (len(pos), k) and sel.dtype == np.int32
        for row, p in zip(sel, pos):
            n = min(k, int(p) + 1) if p >= 0 else 0
            assert (row[n:] == -1).all()
            v = row[:n]
            assert len(set(v.tolist())) == n and ((v >= 0) & (v <= p)).all()
    a = synth.selection(pos, 64, seed=3)
    assert torch.equal(a, synth.selection(pos, 64, seed=3))          # seeded
    assert not torch.equal(a, synth.selection(pos, 64, seed=4))


def test_mha_inputs_shapes_and_tail():
    q, k, v, scale = synth.mha_inputs("mha_small", L=50, T=20)
    assert q.shape == (20, 4, 64) and k.shape == (50, 4, 64) and v.shape == (50, 4, 64)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16 and abs(scale - 0.125) < 1e-12
