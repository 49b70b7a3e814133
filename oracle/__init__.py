"""CPU oracle for the DeepSeek Sparse Attention (DSA) hot path (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers. The CUDA path never imports this package and shares no code with it.

The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64), which cites the
passages it follows. This module only marshals numpy arrays and builds the
shared library with gcc when it is missing or older than its source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_e4m3_table.argtypes = [P]
            lib.oracle_bf16_decode.argtypes = [P, i64, P]
            lib.oracle_num_threads.restype = i32
            lib.oracle_set_threads.argtypes = [i32]
            lib.oracle_indexer_row.argtypes = [P, P, P, i64, i64, i32, i32, P]
            lib.oracle_topk_row.argtypes = [P, i64, i32, P]
            lib.oracle_indexer_scores_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i64, P]
            lib.oracle_indexer_topk_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i32, P]
            lib.oracle_sparse_attn_row.argtypes = [P, P, i64, i64, P, i32, i32, i32, i32, dbl, P, P]
            lib.oracle_sparse_attn_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, dbl,
                                                    P, P]
            lib.oracle_dense_attn_row.argtypes = [P, P, i64, i64, i32, i32, i32, dbl, P, P]
            lib.oracle_lse_merge.argtypes = [P, P, i32, i32, i32, P, P]
            lib.oracle_sparse_attn_bwd_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, dbl,
                                                        P, P, P]
            lib.oracle_mha_attn_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i32, dbl, P, P]
            lib.oracle_indexer_kl_rows.argtypes = [P, P, P, P, P, i32, i32, i32, i32, dbl, P, P, P, i32,
                                                   i32, P, P, P, P]
            _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    """bf16 data as raw uint16 (accepts torch bf16 tensors or uint16 arrays)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and "bfloat16" in str(a.dtype):
        a = a.detach().cpu().contiguous().view(__import__("torch").int16).numpy()
    return np.ascontiguousarray(a).view(np.uint16)


def _u8(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(a).view(np.uint8)


def _np(a, dtype):
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def e4m3_table() -> np.ndarray:
    out = np.empty(256, np.float64)
    _load().oracle_e4m3_table(out.ctypes.data_as(ctypes.c_void_p))
    return out


def bf16_to_f64(a) -> np.ndarray:
    u = _u16(a)
    out = np.empty(u.shape, np.float64)
    _load().oracle_bf16_decode(u.ctypes.data_as(ctypes.c_void_p), u.size,
                               out.ctypes.data_as(ctypes.c_void_p))
    return out


def indexer_scores(q_row, w_row, keys, n: int, k_base: int = 0) -> np.ndarray:
    """I_{t,s} for s < n of one row: q_row e4m3 [H_I, d_I], w_row [H_I], keys e4m3 [*, d_I]."""
    q, qp = _c(_u8(q_row), np.uint8)
    w, wp = _c(_np(w_row, np.float32), np.float32)
    kk, kp = _c(_u8(keys), np.uint8)
    H_I, d_I = q.shape
    out = np.empty(int(n), np.float32)
    _load().oracle_indexer_row(qp, wp, kp, int(k_base), int(n), H_I, d_I,
                               out.ctypes.data_as(ctypes.c_void_p))
    return out


def indexer_scores_rows(q_rows, w_rows, keys, pos, k_base) -> np.ndarray:
    """I_{t,s} of R query rows at once (rows in parallel): float32 [R, max(pos)+1],
    row r valid for s <= pos[r] and NaN past it. q_rows e4m3 [R, H_I, d_I],
    w_rows [R, H_I], keys e4m3 [*, d_I], pos / k_base int [R]."""
    q, qp = _c(_u8(q_rows), np.uint8)
    w, wp = _c(_np(w_rows, np.float32), np.float32)
    kk, kp = _c(_u8(keys), np.uint8)
    p, pp = _c(_np(pos, np.int32), np.int32)
    b, bp = _c(_np(k_base, np.int32), np.int32)
    R, H_I, d_I = q.shape
    ld = int(p.max()) + 1 if R else 1
    out = np.full((R, ld), np.nan, np.float32)
    _load().oracle_indexer_scores_rows(qp, wp, kp, pp, bp, R, H_I, d_I, ld,
                                       out.ctypes.data_as(ctypes.c_void_p))
    return out


def topk(scores, k: int) -> np.ndarray:
    """Top-k of one score row in rank order (score desc, index asc), -1 padded."""
    s, sp = _c(_np(scores, np.float32), np.float32)
    out = np.empty(int(k), np.int32)
    _load().oracle_topk_row(sp, s.size, int(k), out.ctypes.data_as(ctypes.c_void_p))
    return out


def indexer_topk(q_idx, w, keys, pos, k_base, k: int, rows=None) -> np.ndarray:
    """Selected indices for query rows ``rows`` (default: all): int32 [R, k], rank order.

    q_idx e4m3 [T, H_I, d_I]; w [T, H_I]; keys e4m3 [S, d_I]; pos, k_base int [T].
    """
    q_idx = _u8(q_idx)
    T = q_idx.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    q, qp = _c(q_idx[rows], np.uint8)
    ww, wp = _c(_np(w, np.float32)[rows], np.float32)
    kk, kp = _c(_u8(keys), np.uint8)
    pp, ppp = _c(_np(pos, np.int32)[rows], np.int32)
    bb, bbp = _c(_np(k_base, np.int32)[rows], np.int32)
    R, H_I, d_I = q.shape
    out = np.empty((R, int(k)), np.int32)
    _load().oracle_indexer_topk_rows(qp, wp, kp, ppp, bbp, R, H_I, d_I, int(k),
                                     out.ctypes.data_as(ctypes.c_void_p))
    return out


def sparse_attn(q, kv, idx, pos, k_base, scale: float, d_v: int, rows=None, idx_rows=None):
    """Attention of rows ``rows`` over their selected entries.

    q bf16 [T, Hq, d_qk] (or the rows already gathered, when ``idx_rows`` is
    given together with per-row pos/k_base), kv bf16 [S, d_qk], idx int32 [T, k].
    Returns (out fp64 [R, Hq, d_v], lse fp64 [R, Hq]).
    """
    qu = _u16(q)
    T = qu.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    if idx_rows is None:
        q_r, qp = _c(qu[rows], np.uint16)
        i_r, ip = _c(_np(idx, np.int32)[rows], np.int32)
        p_r, pp = _c(_np(pos, np.int32)[rows], np.int32)
        b_r, bp = _c(_np(k_base, np.int32)[rows], np.int32)
    else:
        q_r, qp = _c(qu, np.uint16)
        i_r, ip = _c(_np(idx_rows, np.int32), np.int32)
        p_r, pp = _c(_np(pos, np.int32), np.int32)
        b_r, bp = _c(_np(k_base, np.int32), np.int32)
    kvu, kvp = _c(_u16(kv), np.uint16)
    R, Hq, d_qk = q_r.shape
    k = i_r.shape[1]
    out = np.empty((R, Hq, int(d_v)), np.float64)
    lse = np.empty((R, Hq), np.float64)
    _load().oracle_sparse_attn_rows(qp, kvp, ip, pp, bp, R, k, Hq, d_qk, int(d_v), float(scale),
                                    out.ctypes.data_as(ctypes.c_void_p),
                                    lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def sparse_attn_bwd(q, kv, idx, pos, k_base, scale: float, d_v: int, dout):
    """Gradients of sum(dout * out) of the sparse attention of every row of q
    (bf16 [T, Hq, d_qk]) over its idx entries: (dq fp64 [T, Hq, d_qk],
    dkv fp64 [S, d_qk]); dout bf16 [T, Hq, d_v]. pos / k_base int32 [T]."""
    q_r, qp = _c(_u16(q), np.uint16)
    kvu, kvp = _c(_u16(kv), np.uint16)
    i_r, ip = _c(_np(idx, np.int32), np.int32)
    p_r, pp = _c(_np(pos, np.int32), np.int32)
    b_r, bp = _c(_np(k_base, np.int32), np.int32)
    g_r, gp = _c(_u16(dout), np.uint16)
    R, Hq, d_qk = q_r.shape
    k = i_r.shape[1]
    dq = np.zeros((R, Hq, d_qk), np.float64)
    dkv = np.zeros((kvu.shape[0], d_qk), np.float64)
    _load().oracle_sparse_attn_bwd_rows(qp, kvp, ip, pp, bp, R, k, Hq, d_qk, int(d_v), float(scale), gp,
                                        dq.ctypes.data_as(ctypes.c_void_p),
                                        dkv.ctypes.data_as(ctypes.c_void_p))
    return dq, dkv


def indexer_kl(q, kv, idx, pos, k_base, scale: float, q_idx, w, k_idx):
    """Indexer KL loss over each row's selected set and its gradient:
    (loss fp64 [T], dw fp64 [T, H_I], dq_idx fp64 [T, H_I, d_I], dk_idx fp64 [S, d_I]).
    q bf16 [T, Hq, d_qk], kv bf16 [S, d_qk], q_idx e4m3 [T, H_I, d_I], w fp32 [T, H_I],
    k_idx e4m3 [S, d_I], idx/pos/k_base int32."""
    q_r, qp = _c(_u16(q), np.uint16)
    kvu, kvp = _c(_u16(kv), np.uint16)
    i_r, ip = _c(_np(idx, np.int32), np.int32)
    p_r, pp = _c(_np(pos, np.int32), np.int32)
    b_r, bp = _c(_np(k_base, np.int32), np.int32)
    qi, qip = _c(_u8(q_idx), np.uint8)
    w_r, wp = _c(_np(w, np.float32), np.float32)
    ki, kip = _c(_u8(k_idx), np.uint8)
    R, Hq, d_qk = q_r.shape
    _, H_I, d_I = qi.shape
    k = i_r.shape[1]
    loss = np.zeros(R, np.float64)
    dw = np.zeros((R, H_I), np.float64)
    dq = np.zeros((R, H_I, d_I), np.float64)
    dk = np.zeros((ki.shape[0], d_I), np.float64)
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _load().oracle_indexer_kl_rows(qp, kvp, ip, pp, bp, R, k, Hq, d_qk, float(scale), qip, wp, kip, H_I,
                                   d_I, vp(loss), vp(dw), vp(dq), vp(dk))
    return loss, dw, dq, dk


def mha_attn(q, k, v, pos, k_base, scale: float):
    """Dense causal attention with per-head keys and values (MLA in MHA mode):
    (out fp64 [R, Hq, d_hv], lse fp64 [R, Hq]). q bf16 [R, Hq, d_h], k bf16
    [S, Hq, d_h], v bf16 [S, Hq, d_hv]; row r sees keys k_base[r] + 0..pos[r]."""
    q_r, qp = _c(_u16(q), np.uint16)
    k_r, kp = _c(_u16(k), np.uint16)
    v_r, vp = _c(_u16(v), np.uint16)
    p_r, pp = _c(_np(pos, np.int32), np.int32)
    b_r, bp = _c(_np(k_base, np.int32), np.int32)
    R, Hq, d_h = q_r.shape
    d_hv = v_r.shape[2]
    out = np.zeros((R, Hq, d_hv), np.float64)
    lse = np.zeros((R, Hq), np.float64)
    _load().oracle_mha_attn_rows(qp, kp, vp, pp, bp, R, Hq, d_h, d_hv, float(scale),
                                 out.ctypes.data_as(ctypes.c_void_p), lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def dense_attn_row(q_row, kv, pos: int, k_base: int, scale: float, d_v: int):
    """Dense causal MQA of one row over s = 0..pos: (out [Hq, d_v], lse [Hq])."""
    q, qp = _c(_u16(q_row), np.uint16)
    kvu, kvp = _c(_u16(kv), np.uint16)
    Hq, d_qk = q.shape
    out = np.empty((Hq, int(d_v)), np.float64)
    lse = np.empty(Hq, np.float64)
    _load().oracle_dense_attn_row(qp, kvp, int(k_base), int(pos), Hq, d_qk, int(d_v),
                                  float(scale), out.ctypes.data_as(ctypes.c_void_p),
                                  lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def lse_merge(o_parts, lse_parts):
    """Merge P partial (o [P, Hq, d_v], lse [P, Hq]) into (o [Hq, d_v], lse [Hq])."""
    o, op = _c(o_parts, np.float64)
    l, lp = _c(lse_parts, np.float64)
    P, Hq, d_v = o.shape
    out = np.empty((Hq, d_v), np.float64)
    lse = np.empty(Hq, np.float64)
    _load().oracle_lse_merge(op, lp, P, Hq, d_v, out.ctypes.data_as(ctypes.c_void_p),
                             lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse
