"""Parity rules between the CUDA path and the CPU oracle (shared by the GPU
tests, smoke() and bench.py).

Indexer / selector:
  * integer-valued FP8 inputs: every score is an integer below 2^24, exact in
    any summation order, so the selected sets must be identical;
  * realistic inputs: each row holds min(k, pos+1) distinct in-range indices,
    and every selected s has I_orc[s] >= kth_orc - 1e-3 * max(|kth_orc|, eps)
    with eps = 1e-3 * max_s |I_orc[s]| (an absolute floor for k-th scores near
    zero, which signed head weights make possible).
Attention (fed the GPU's own idx, so near-tie swaps do not count against it):
  rel-L2 <= 1e-2 and max-abs <= 3e-2 on out (bf16), |lse - lse_orc| <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

IDX_REL = 1e-3
OUT_REL_L2 = 1e-2
OUT_MAX_ABS = 3e-2
LSE_ABS = 1e-3


def _cpu(t):
    return t.detach().cpu() if isinstance(t, torch.Tensor) else t


def host_inputs(x, rows):
    """The oracle's view of an input batch: full caches, the given query rows."""
    rows = np.asarray(rows, dtype=np.int64)
    r = torch.from_numpy(rows).to(x.q_idx.device)
    return dict(
        q_idx=_cpu(x.q_idx[r]).numpy(), w=_cpu(x.w[r]).numpy(), k_idx=_cpu(x.k_idx).numpy(),
        q=_cpu(x.q[r]), kv=_cpu(x.kv), pos=_cpu(x.positions()[r]).numpy(),
        base=_cpu(x.bases()[r]).numpy())


def check_indexer(x, idx_gpu, rows, exact: bool, h=None):
    """idx_gpu: [len(rows), k] selected by the CUDA path for these rows."""
    h = h or host_inputs(x, rows)
    idx_gpu = np.asarray(_cpu(idx_gpu))
    k = x.k
    if exact:
        ref = oracle.indexer_topk(h["q_idx"], h["w"], h["k_idx"], h["pos"], h["base"], k)
    else:
        scores = oracle.indexer_scores_rows(h["q_idx"], h["w"], h["k_idx"], h["pos"], h["base"])
    for r, t in enumerate(rows):
        row = idx_gpu[r]
        n = int(h["pos"][r]) + 1
        m = min(k, n)
        valid = row[:m]
        assert (row[m:] == -1).all(), f"row {t}: padding"
        assert (valid >= 0).all() and (valid < n).all(), f"row {t}: out of range"
        assert len(np.unique(valid)) == m, f"row {t}: duplicates"
        if exact:
            assert np.array_equal(np.sort(valid), np.sort(ref[r][:m])), f"row {t}: set differs"
        else:
            sc = scores[r, :n].astype(np.float64)
            if m == n:
                continue
            kth = np.sort(sc)[::-1][m - 1]
            eps = 1e-3 * np.abs(sc).max()
            tol = IDX_REL * max(abs(kth), eps)
            worst = sc[valid].min()
            assert worst >= kth - tol, f"row {t}: selected score {worst} < kth {kth} - {tol}"


def check_attention(x, idx_gpu, out_gpu, lse_gpu, rows, h=None):
    """out_gpu [R, Hq, d_v] bf16, lse_gpu [R, Hq] for query rows `rows`."""
    h = h or host_inputs(x, rows)
    idx_gpu = np.asarray(_cpu(idx_gpu))
    ref_o, ref_l = oracle.sparse_attn(h["q"], h["kv"], None, h["pos"], h["base"], x.scale, x.d_v,
                                      idx_rows=idx_gpu)
    o = _cpu(out_gpu).to(torch.float64).numpy()
    l = _cpu(lse_gpu).to(torch.float64).numpy()
    for r, t in enumerate(rows):
        d = o[r] - ref_o[r]
        rel = np.linalg.norm(d) / max(np.linalg.norm(ref_o[r]), 1e-30)
        assert rel <= OUT_REL_L2, f"row {t}: rel-L2 {rel}"
        assert np.abs(d).max() <= OUT_MAX_ABS, f"row {t}: max-abs {np.abs(d).max()}"
        fin = np.isfinite(ref_l[r])
        assert (np.isfinite(l[r]) == fin).all(), f"row {t}: lse finiteness"
        assert np.abs(l[r][fin] - ref_l[r][fin]).max(initial=0) <= LSE_ABS, f"row {t}: lse"
    return ref_o, ref_l
