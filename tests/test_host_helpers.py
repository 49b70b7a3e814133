"""Host-side helpers of the serving forms (no GPU): the page-pool builder
places every key of every sequence where the block table says, and the
varlen row maps give each packed row its sequence's range."""
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
