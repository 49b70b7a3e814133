"""Paged key / latent caches (block tables over a shuffled page pool): the
paged decode path gives the same indices and bit-identical attention as the
contiguous path on the same data (the contiguous call with one part per row,
as the paged kernel runs; the library's own choice splits few rows into
parts, which changes the rounding), and matches the oracle."""
import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build
from parity import check_attention, check_indexer, host_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dsa_build.build()
    dsa.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    torch.cuda.synchronize()
    assert dsa.device_status() == 0


def _both(x, page_size):
    kp, vp, bt, seq = synth.page_caches(x, page_size, seed=page_size)
    idx_c = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k, pos=x.pos, k_base=x.k_base)
    idx_p = dsa.indexer_topk_paged(x.q_idx, x.w, kp, page_size, bt, seq, x.pos, x.k)
    torch.cuda.synchronize()
    assert torch.equal(torch.sort(idx_c, 1)[0], torch.sort(idx_p, 1)[0])
    out_c, lse_c = dsa.sparse_mla_attn_split(x.q, x.kv, idx_c, x.scale, x.d_v, 1, pos=x.pos, k_base=x.k_base)
    out_p, lse_p = dsa.sparse_mla_attn_paged(x.q, vp, page_size, bt, seq, x.pos, idx_c, x.scale, x.d_v)
    torch.cuda.synchronize()
    assert torch.equal(out_c, out_p) and torch.equal(lse_c, lse_p)
    return idx_p, out_p, lse_p


@pytest.mark.parametrize("page_size", [64, 128, 256])
def test_paged_decode_matches_contiguous_bit_for_bit(page_size):
    x = synth.decode_inputs("decode", device="cuda", seed=6, B=7,
                            ctx=[9000, 20000, 64, 130, 16385, 40000, 8191])
    _both(x, page_size)


def test_paged_decode_integer_inputs_match_oracle():
    x = synth.decode_inputs("decode", device="cuda", seed=7, B=5, ctx=[12000, 300, 30000, 8193, 5000],
                            overrides=dict(indexer="int", k=1024))
    idx, out, lse = _both(x, 64)
    rows = list(range(x.T))
    h = host_inputs(x, rows)
    check_indexer(x, idx.cpu(), rows, exact=True, h=h)
    check_attention(x, idx.cpu(), out.cpu(), lse.cpu(), rows, h=h)
