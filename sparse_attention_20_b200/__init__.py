"""DeepSeek Sparse Attention (DSA) hot path on B200 (sm_100a): Python binding.

A thin ctypes layer over ``libdsa.so`` (C ABI in ``include/dsa.h``): it checks
tensor dtypes/devices, passes raw device pointers and the current CUDA stream,
and raises on a non-zero status. Every step of the computation runs in the
library's CUDA kernels; PyTorch only provides device memory and streams. There
is no CPU fallback: without the built library (or without a GPU) every call
raises.

Entry points mirror the C ABI:
  * ``indexer_topk``     lightning indexer + Top-k selector -> idx [T, k]
  * ``sparse_mla_attn``  sparse MQA attention over idx -> out [T, Hq, d_v], lse [T, Hq]
  * ``forward``          both, on one stream
  * ``workspace_size``, ``device_status``, ``last_error``
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DEBUG_LIB_PATH = os.path.join(_PKG, "libdsa_debug.so")

DSA_OK = 0
STATUS_NAMES = {0: "DSA_OK", -1: "DSA_ERR_ARG", -2: "DSA_ERR_UNSUPPORTED", -3: "DSA_ERR_CUDA",
                -4: "DSA_ERR_TIMEOUT", -5: "DSA_ERR_WORKSPACE", -6: "DSA_ERR_CHECK"}

# Every symbol include/dsa.h declares.
EXPORTS = ("dsa_workspace_size", "dsa_indexer_topk", "dsa_sparse_mla_attn", "dsa_forward",
           "dsa_device_status", "dsa_last_error", "dsa_abi_version", "dsa_launch_count",
           "dsa_indexer_topk_noalloc", "dsa_selftest_bounded_wait", "dsa_indexer_topk_varlen",
           "dsa_indexer_topk_paged", "dsa_sparse_mla_attn_paged", "dsa_sparse_mla_attn_bwd",
           "dsa_sparse_mla_attn_bwd_workspace_size", "dsa_indexer_kl", "dsa_indexer_kl_workspace_size",
           "dsa_mla_mha_attn", "dsa_partition_prefill_rows", "dsa_partition_decode_seqs",
           "dsa_sparse_mla_attn_split", "dsa_sparse_mla_attn_split_workspace_size", "dsa_debug_build",
           "dsa_debug_counters", "dsa_phase_timing", "dsa_phase_times")


class DSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdsa.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} is missing: build it with "
                          "`python -m sparse_attention_20_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        lib.dsa_workspace_size.argtypes = [I] * 8
        lib.dsa_workspace_size.restype = Z
        lib.dsa_indexer_topk.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, Z, P]
        lib.dsa_indexer_topk.restype = I
        lib.dsa_sparse_mla_attn.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, Z, P]
        lib.dsa_sparse_mla_attn.restype = I
        lib.dsa_sparse_mla_attn_split.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P, Z, P]
        lib.dsa_sparse_mla_attn_split.restype = I
        lib.dsa_sparse_mla_attn_split_workspace_size.argtypes = [I, I, I, I]
        lib.dsa_sparse_mla_attn_split_workspace_size.restype = Z
        lib.dsa_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, Z,
                                    P]
        lib.dsa_forward.restype = I
        lib.dsa_device_status.argtypes = [P]
        lib.dsa_device_status.restype = I
        lib.dsa_last_error.restype = ctypes.c_char_p
        lib.dsa_abi_version.restype = I
        lib.dsa_launch_count.restype = ctypes.c_uint64
        lib.dsa_indexer_topk_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P]
        lib.dsa_indexer_topk_noalloc.restype = I
        lib.dsa_indexer_topk_varlen.argtypes = [P, P, P, P, P, I, I, I, I, P, P, Z, P]
        lib.dsa_indexer_topk_varlen.restype = I
        lib.dsa_indexer_topk_paged.argtypes = [P, P, P, I, I, P, I, I, P, P, I, I, I, I, P, P, Z, P]
        lib.dsa_indexer_topk_paged.restype = I
        lib.dsa_sparse_mla_attn_paged.argtypes = [P, P, I, I, P, I, I, P, P, P, I, I, I, I, I, F, P, P, P]
        lib.dsa_sparse_mla_attn_paged.restype = I
        lib.dsa_sparse_mla_attn_bwd_workspace_size.argtypes = [I, I, I]
        lib.dsa_sparse_mla_attn_bwd_workspace_size.restype = Z
        lib.dsa_sparse_mla_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P, P, Z,
                                                P]
        lib.dsa_sparse_mla_attn_bwd.restype = I
        lib.dsa_indexer_kl_workspace_size.argtypes = [I, I]
        lib.dsa_indexer_kl_workspace_size.restype = Z
        lib.dsa_indexer_kl.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, P, P, P, P, Z, P]
        lib.dsa_indexer_kl.restype = I
        lib.dsa_mla_mha_attn.argtypes = [P, P, P, I, I, I, I, I, F, P, P, P]
        lib.dsa_mla_mha_attn.restype = I
        lib.dsa_partition_prefill_rows.argtypes = [I] * 9 + [P]
        lib.dsa_partition_prefill_rows.restype = I
        lib.dsa_partition_decode_seqs.argtypes = [P, I, I, I, I, I, P]
        lib.dsa_partition_decode_seqs.restype = I
        lib.dsa_phase_timing.argtypes = [I]
        lib.dsa_phase_timing.restype = I
        lib.dsa_phase_times.argtypes = [P, I]
        lib.dsa_phase_times.restype = I
        lib.dsa_debug_build.restype = I
        lib.dsa_debug_counters.argtypes = [P, I, I]
        lib.dsa_debug_counters.restype = I
        lib.dsa_selftest_bounded_wait.argtypes = [I, P]
        lib.dsa_selftest_bounded_wait.restype = I
        _lib = lib
    return _lib


def last_error() -> str:
    return load_library().dsa_last_error().decode()


def _check(rc: int):
    if rc != DSA_OK:
        raise DSAError(rc, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, device=None) -> torch.Tensor:
    """A dense CUDA tensor (on `device` when given)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {device}")
    return t


def _arg(t: torch.Tensor, name: str, dtype, shape=None, device=None) -> torch.Tensor:
    """A dense CUDA tensor of this dtype and (when given) exactly this shape."""
    _dev(t, name, device)
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(int(v) for v in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(int(v) for v in shape)}")
    return t


def _fp8(t: torch.Tensor, name: str, device=None) -> torch.Tensor:
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    if not isinstance(t, torch.Tensor) or t.dtype != torch.uint8:
        raise TypeError(f"{name} must hold e4m3 bytes (uint8 or float8_e4m3fn)")
    return _dev(t, name, device)


def _i32(t: Optional[torch.Tensor], name: str, shape=None, device=None):
    if t is None:
        return None
    return _arg(t, name, torch.int32, shape, device)


def _out(t, name, dtype, shape, device, fill=None):
    """A caller-supplied output buffer, checked; a new one when None."""
    if t is None:
        if fill is None:
            return torch.empty(tuple(int(v) for v in shape), dtype=dtype, device=device)
        return torch.full(tuple(int(v) for v in shape), fill, dtype=dtype, device=device)
    return _arg(t, name, dtype, shape, device)


def _ws(t: torch.Tensor, device) -> int:
    """Workspace buffer on the operands' device; returns its size in bytes."""
    _dev(t, "workspace", device)
    return t.numel() * t.element_size()


def workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v) -> int:
    return int(load_library().dsa_workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v))


def alloc_workspace(T, S, H_I, d_I, k, Hq, d_qk, d_v, device=None) -> torch.Tensor:
    n = workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def _indexer_inputs(q_idx, w, k_idx, pos, k_base):
    """Checked indexer inputs: (q_idx, w, k_idx, pos, k_base, T, H_I, d_I, S, device)."""
    q_idx = _fp8(q_idx, "q_idx")
    dev = q_idx.device
    if q_idx.dim() != 3:
        raise ValueError(f"q_idx must be [T, H_I, d_I], got shape {tuple(q_idx.shape)}")
    T, H_I, d_I = q_idx.shape
    k_idx = _fp8(k_idx, "k_idx", dev)
    if k_idx.dim() != 2 or k_idx.shape[1] != d_I:
        raise ValueError(f"k_idx must be [S, {d_I}], got shape {tuple(k_idx.shape)}")
    w = _arg(w, "w", torch.float32, (T, H_I), dev)
    pos = _i32(pos, "pos", (T,), dev)
    k_base = _i32(k_base, "k_base", (T,), dev)
    return q_idx, w, k_idx, pos, k_base, T, H_I, d_I, k_idx.shape[0], dev


def _attn_inputs(q, kv, idx, pos, k_base, T=None):
    """Checked attention inputs: (q, kv, idx, pos, k_base, T, Hq, d_qk, S, k, device)."""
    q = _dev(q, "q")
    dev = q.device
    if q.dtype != torch.bfloat16 or q.dim() != 3:
        raise TypeError(f"q must be bfloat16 [T, Hq, d_qk], got {q.dtype} {tuple(q.shape)}")
    Tq, Hq, d_qk = q.shape
    if T is not None and Tq != T:
        raise ValueError(f"q has {Tq} rows, expected {T}")
    kv = _dev(kv, "kv", dev)
    if kv.dtype != torch.bfloat16 or kv.dim() != 2 or kv.shape[1] != d_qk:
        raise TypeError(f"kv must be bfloat16 [S, {d_qk}], got {kv.dtype} {tuple(kv.shape)}")
    idx = _dev(idx, "idx", dev)
    if idx.dtype != torch.int32 or idx.dim() != 2 or idx.shape[0] != Tq:
        raise TypeError(f"idx must be int32 [{Tq}, k], got {idx.dtype} {tuple(idx.shape)}")
    pos = _i32(pos, "pos", (Tq,), dev)
    k_base = _i32(k_base, "k_base", (Tq,), dev)
    return q, kv, idx, pos, k_base, Tq, Hq, d_qk, kv.shape[0], idx.shape[1], dev


def indexer_topk(q_idx, w, k_idx, k: int, pos=None, k_base=None, idx=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """idx [T, k] int32: the Top-k s per query row (a set, -1 padded)."""
    q_idx, w, k_idx, pos, k_base, T, H_I, d_I, S, dev = _indexer_inputs(q_idx, w, k_idx, pos, k_base)
    idx = _out(idx, "idx", torch.int32, (T, k), dev)
    if workspace is None:
        workspace = alloc_workspace(T, S, H_I, d_I, k, 1, 8, 2, dev)
    nbytes = _ws(workspace, dev)
    lib = load_library()
    _check(lib.dsa_indexer_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(pos), _ptr(k_base), T, S,
                                H_I, d_I, k, _ptr(idx), _ptr(workspace), nbytes, _stream(stream)))
    return idx


def indexer_topk_noalloc(q_idx, w, k_idx, k: int, pos=None, k_base=None, idx=None,
                         stream=None) -> torch.Tensor:
    """dsa_indexer_topk_noalloc: idx [T, k] with the library's own scratch
    (no workspace; calls on one device must not overlap)."""
    q_idx, w, k_idx, pos, k_base, T, H_I, d_I, S, dev = _indexer_inputs(q_idx, w, k_idx, pos, k_base)
    idx = _out(idx, "idx", torch.int32, (T, k), dev)
    _check(load_library().dsa_indexer_topk_noalloc(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(pos),
                                                   _ptr(k_base), T, S, H_I, d_I, k, _ptr(idx),
                                                   _stream(stream)))
    return idx


def varlen_rows(cu_q, cu_k, device):
    """(pos, k_base) int32 [T] of a packed batch of suffix-aligned causal
    sequences (cu_q / cu_k: host offsets): what dsa_sparse_mla_attn needs for
    the same rows."""
    cu_q = [int(v) for v in cu_q]
    cu_k = [int(v) for v in cu_k]
    pos, base = [], []
    for b in range(len(cu_q) - 1):
        Tb, Sb = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        pos.extend(range(Sb - Tb, Sb))
        base.extend([cu_k[b]] * Tb)
    return (torch.tensor(pos, dtype=torch.int32, device=device),
            torch.tensor(base, dtype=torch.int32, device=device))


def indexer_topk_varlen(q_idx, w, k_idx, cu_q, cu_k, k: int, idx=None, workspace=None,
                        stream=None) -> torch.Tensor:
    """idx [T, k] int32 for a packed batch of causal sequences; cu_q / cu_k are
    host offsets (lists or CPU tensors) of each sequence's query and key rows."""
    q_idx, w, k_idx, _, _, T, H_I, d_I, S, dev = _indexer_inputs(q_idx, w, k_idx, None, None)
    if len(cu_q) != len(cu_k) or len(cu_q) < 2:
        raise ValueError("cu_q and cu_k need n_seqs + 1 >= 2 entries each")
    cq = (ctypes.c_int32 * len(cu_q))(*[int(v) for v in cu_q])
    ck = (ctypes.c_int32 * len(cu_k))(*[int(v) for v in cu_k])
    n = len(cu_q) - 1
    if cq[n] != T or ck[n] != S:
        raise ValueError(f"cu_q[-1] = {cq[n]} and cu_k[-1] = {ck[n]} must equal T = {T} and S = {S}")
    idx = _out(idx, "idx", torch.int32, (T, k), dev)
    if workspace is None:
        t_max = max(cq[b + 1] - cq[b] for b in range(n))
        s_max = max(ck[b + 1] - ck[b] for b in range(n))
        workspace = alloc_workspace(max(t_max, 1), max(s_max, 1), H_I, d_I, k, 1, 8, 2, dev)
    nbytes = _ws(workspace, dev)
    _check(load_library().dsa_indexer_topk_varlen(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), ctypes.cast(cq, ctypes.c_void_p), ctypes.cast(ck, ctypes.c_void_p),
        n, H_I, d_I, k, _ptr(idx), _ptr(workspace), nbytes, _stream(stream)))
    return idx


def _paged_tables(block_table, seq, pos, T, dev):
    block_table = _dev(block_table, "block_table", dev)
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise TypeError("block_table must be int32 [n_seqs, max_pages]")
    return block_table, _i32(seq, "seq", (T,), dev), _i32(pos, "pos", (T,), dev)


def indexer_topk_paged(q_idx, w, k_pages, page_size: int, block_table, seq, pos, k: int, idx=None,
                       workspace=None, stream=None) -> torch.Tensor:
    """idx [T, k] over a paged FP8 key cache (k_pages [num_pages*page_size, d_I],
    block_table [n_seqs, max_pages], seq / pos [T]; see include/dsa.h)."""
    q_idx, w, k_pages, _, _, T, H_I, d_I, rows, dev = _indexer_inputs(q_idx, w, k_pages, None, None)
    if page_size <= 0 or rows % page_size:
        raise ValueError(f"k_pages has {rows} rows, not a whole number of {page_size}-row pages")
    block_table, seq, pos = _paged_tables(block_table, seq, pos, T, dev)
    num_pages = rows // page_size
    n_seqs, max_pages = block_table.shape
    idx = _out(idx, "idx", torch.int32, (T, k), dev)
    if workspace is None:
        workspace = alloc_workspace(T, max_pages * page_size, H_I, d_I, k, 1, 8, 2, dev)
    nbytes = _ws(workspace, dev)
    _check(load_library().dsa_indexer_topk_paged(
        _ptr(q_idx), _ptr(w), _ptr(k_pages), num_pages, page_size, _ptr(block_table), n_seqs, max_pages,
        _ptr(seq), _ptr(pos), T, H_I, d_I, k, _ptr(idx), _ptr(workspace), nbytes, _stream(stream)))
    return idx


def sparse_mla_attn_paged(q, kv_pages, page_size: int, block_table, seq, pos, idx, scale: float,
                          d_v: int, out=None, lse=None, stream=None):
    """(out, lse) of sparse MQA attention over a paged latent cache."""
    q, kv_pages, idx, _, _, T, Hq, d_qk, rows, k, dev = _attn_inputs(q, kv_pages, idx, None, None)
    if page_size <= 0 or rows % page_size:
        raise ValueError(f"kv_pages has {rows} rows, not a whole number of {page_size}-row pages")
    block_table, seq, pos = _paged_tables(block_table, seq, pos, T, dev)
    num_pages = rows // page_size
    n_seqs, max_pages = block_table.shape
    out = _out(out, "out", torch.bfloat16, (T, Hq, d_v), dev)
    lse = _out(lse, "lse", torch.float32, (T, Hq), dev)
    _check(load_library().dsa_sparse_mla_attn_paged(
        _ptr(q), _ptr(kv_pages), num_pages, page_size, _ptr(block_table), n_seqs, max_pages, _ptr(seq),
        _ptr(pos), _ptr(idx), T, Hq, d_qk, d_v, k, float(scale), _ptr(out), _ptr(lse),
        _stream(stream)))
    return out, lse


def sparse_mla_attn(q, kv, idx, scale: float, d_v: int, pos=None, k_base=None, out=None,
                    lse=None, workspace=None, stream=None):
    """(out bf16 [T, Hq, d_v], lse fp32 [T, Hq]) of sparse MQA attention over idx."""
    q, kv, idx, pos, k_base, T, Hq, d_qk, S, k, dev = _attn_inputs(q, kv, idx, pos, k_base)
    out = _out(out, "out", torch.bfloat16, (T, Hq, d_v), dev)
    lse = _out(lse, "lse", torch.float32, (T, Hq), dev)
    if workspace is None:
        workspace = alloc_workspace(T, S, 1, 32, k, Hq, d_qk, d_v, dev)
    nbytes = _ws(workspace, dev)
    lib = load_library()
    _check(lib.dsa_sparse_mla_attn(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), T, S, Hq,
                                   d_qk, d_v, k, float(scale), _ptr(out), _ptr(lse),
                                   _ptr(workspace), nbytes, _stream(stream)))
    return out, lse


def sparse_mla_attn_split(q, kv, idx, scale: float, d_v: int, splits: int, pos=None, k_base=None, out=None,
                          lse=None, workspace=None, stream=None):
    """sparse_mla_attn with each row's selected set split into `splits` parts
    (0 = the library's choice) merged by log-sum-exp: (out, lse)."""
    q, kv, idx, pos, k_base, T, Hq, d_qk, S, k, dev = _attn_inputs(q, kv, idx, pos, k_base)
    out = _out(out, "out", torch.bfloat16, (T, Hq, d_v), dev)
    lse = _out(lse, "lse", torch.float32, (T, Hq), dev)
    lib = load_library()
    if workspace is None:
        need = (workspace_size(T, S, 1, 32, k, Hq, d_qk, d_v) if splits == 0
                else int(lib.dsa_sparse_mla_attn_split_workspace_size(T, Hq, d_v, splits)))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    nbytes = _ws(workspace, dev)
    _check(lib.dsa_sparse_mla_attn_split(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), T, S, Hq, d_qk,
                                         d_v, k, float(scale), int(splits), _ptr(out), _ptr(lse), _ptr(workspace),
                                         nbytes, _stream(stream)))
    return out, lse


def sparse_mla_attn_bwd(q, kv, idx, out, lse, dout, scale: float, pos=None, k_base=None, dq=None,
                        dkv=None, workspace=None, stream=None):
    """(dq fp32 [T, Hq, d_qk], dkv fp32 [S, d_qk]) of sparse MQA attention over idx.

    out / lse are the forward's results for the same idx; dout is bf16
    [T, Hq, d_v]. dkv is accumulated into (a new zeroed tensor when None)."""
    q, kv, idx, pos, k_base, T, Hq, d_qk, S, k, dev = _attn_inputs(q, kv, idx, pos, k_base)
    out = _dev(out, "out", dev)
    if out.dtype != torch.bfloat16 or out.dim() != 3 or tuple(out.shape[:2]) != (T, Hq):
        raise TypeError(f"out must be bfloat16 [{T}, {Hq}, d_v], got {out.dtype} {tuple(out.shape)}")
    d_v = out.shape[2]
    dout = _arg(dout, "dout", torch.bfloat16, (T, Hq, d_v), dev)
    lse = _arg(lse, "lse", torch.float32, (T, Hq), dev)
    dq = _out(dq, "dq", torch.float32, (T, Hq, d_qk), dev)
    dkv = _out(dkv, "dkv", torch.float32, (S, d_qk), dev, fill=0.0)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_sparse_mla_attn_bwd_workspace_size(T, Hq, k)),
                                dtype=torch.uint8, device=dev)
    nbytes = _ws(workspace, dev)
    _check(lib.dsa_sparse_mla_attn_bwd(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), _ptr(out),
                                       _ptr(lse), _ptr(dout), T, S, Hq, d_qk, d_v, k, float(scale),
                                       _ptr(dq), _ptr(dkv), _ptr(workspace), nbytes, _stream(stream)))
    return dq, dkv


def indexer_kl(q, kv, idx, lse, q_idx, w, k_idx, scale: float, pos=None, k_base=None, dk_idx=None,
               workspace=None, stream=None):
    """Indexer KL loss over each row's selected set and its gradient:
    (loss fp32 [T], dw fp32 [T, H_I], dq_idx fp32 [T, H_I, d_I], dk_idx fp32 [S, d_I]).

    lse is the attention forward's log-sum-exp for the same idx. dk_idx is
    accumulated into (a new zeroed tensor when None)."""
    q, kv, idx, pos, k_base, T, Hq, d_qk, S, k, dev = _attn_inputs(q, kv, idx, pos, k_base)
    lse = _arg(lse, "lse", torch.float32, (T, Hq), dev)
    q_idx = _fp8(q_idx, "q_idx", dev)
    if q_idx.dim() != 3 or q_idx.shape[0] != T:
        raise ValueError(f"q_idx must be [{T}, H_I, d_I], got shape {tuple(q_idx.shape)}")
    _, H_I, d_I = q_idx.shape
    w = _arg(w, "w", torch.float32, (T, H_I), dev)
    k_idx = _fp8(k_idx, "k_idx", dev)
    if tuple(k_idx.shape) != (S, d_I):
        raise ValueError(f"k_idx must be [{S}, {d_I}] (one indexer key per latent row), got "
                         f"{tuple(k_idx.shape)}")
    loss = torch.empty(T, dtype=torch.float32, device=dev)
    dw = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    dq_idx = torch.empty((T, H_I, d_I), dtype=torch.float32, device=dev)
    dk_idx = _out(dk_idx, "dk_idx", torch.float32, (S, d_I), dev, fill=0.0)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_indexer_kl_workspace_size(T, k)), dtype=torch.uint8, device=dev)
    nbytes = _ws(workspace, dev)
    _check(lib.dsa_indexer_kl(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), _ptr(lse), _ptr(q_idx),
                              _ptr(w), _ptr(k_idx), T, S, Hq, d_qk, H_I, d_I, k, float(scale), _ptr(loss),
                              _ptr(dw), _ptr(dq_idx), _ptr(dk_idx), _ptr(workspace), nbytes,
                              _stream(stream)))
    return loss, dw, dq_idx, dk_idx


def mla_mha_attn(q, k, v, scale: float, out=None, lse=None, stream=None):
    """MLA in MHA mode, dense causal over one sequence: (out bf16 [T, Hq, d_hv],
    lse fp32 [T, Hq]); q [T, Hq, d_h], k [S, Hq, d_h], v [S, Hq, d_hv] bf16, the
    queries being the last T of the S tokens."""
    q = _dev(q, "q")
    dev = q.device
    if q.dtype != torch.bfloat16 or q.dim() != 3:
        raise TypeError(f"q must be bfloat16 [T, Hq, d_h], got {q.dtype} {tuple(q.shape)}")
    T, Hq, d_h = q.shape
    k = _dev(k, "k", dev)
    if k.dtype != torch.bfloat16 or k.dim() != 3 or tuple(k.shape[1:]) != (Hq, d_h):
        raise TypeError(f"k must be bfloat16 [S, {Hq}, {d_h}], got {k.dtype} {tuple(k.shape)}")
    S = k.shape[0]
    v = _dev(v, "v", dev)
    if v.dtype != torch.bfloat16 or v.dim() != 3 or tuple(v.shape[:2]) != (S, Hq):
        raise TypeError(f"v must be bfloat16 [{S}, {Hq}, d_hv], got {v.dtype} {tuple(v.shape)}")
    d_hv = v.shape[2]
    out = _out(out, "out", torch.bfloat16, (T, Hq, d_hv), dev)
    lse = _out(lse, "lse", torch.float32, (T, Hq), dev)
    _check(load_library().dsa_mla_mha_attn(_ptr(q), _ptr(k), _ptr(v), T, S, Hq, d_h, d_hv, float(scale),
                                           _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def forward(q_idx, w, k_idx, q, kv, k: int, scale: float, d_v: int, pos=None, k_base=None,
            idx=None, out=None, lse=None, workspace=None, stream=None):
    """The whole hot path: (idx, out, lse)."""
    q_idx, w, k_idx, pos, k_base, T, H_I, d_I, S, dev = _indexer_inputs(q_idx, w, k_idx, pos, k_base)
    q = _dev(q, "q", dev)
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[0] != T:
        raise TypeError(f"q must be bfloat16 [{T}, Hq, d_qk], got {q.dtype} {tuple(q.shape)}")
    _, Hq, d_qk = q.shape
    kv = _dev(kv, "kv", dev)
    if kv.dtype != torch.bfloat16 or tuple(kv.shape) != (S, d_qk):
        raise TypeError(f"kv must be bfloat16 [{S}, {d_qk}] (one latent row per indexer key), got "
                        f"{kv.dtype} {tuple(kv.shape)}")
    idx = _out(idx, "idx", torch.int32, (T, k), dev)
    out = _out(out, "out", torch.bfloat16, (T, Hq, d_v), dev)
    lse = _out(lse, "lse", torch.float32, (T, Hq), dev)
    if workspace is None:
        workspace = alloc_workspace(T, S, H_I, d_I, k, Hq, d_qk, d_v, dev)
    nbytes = _ws(workspace, dev)
    lib = load_library()
    _check(lib.dsa_forward(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q), _ptr(kv), _ptr(pos),
                           _ptr(k_base), T, S, H_I, d_I, Hq, d_qk, d_v, k, float(scale), _ptr(idx),
                           _ptr(out), _ptr(lse), _ptr(workspace), nbytes, _stream(stream)))
    return idx, out, lse


def partition_prefill_rows(T: int, S: int, k: int, H_I: int, d_I: int, Hq: int, d_qk: int, d_v: int,
                           parts: int) -> list:
    """Contiguous query-row ranges of one causal prefill for `parts` ranks:
    bounds (list of parts + 1 ints); rank r takes rows [bounds[r], bounds[r+1])."""
    b = (ctypes.c_int32 * (parts + 1))()
    _check(load_library().dsa_partition_prefill_rows(T, S, k, H_I, d_I, Hq, d_qk, d_v, parts,
                                                     ctypes.cast(b, ctypes.c_void_p)))
    return list(b)


def partition_decode_seqs(ctx, k: int, d_I: int, d_qk: int, parts: int) -> list:
    """Contiguous ranges of decode sequences (context lengths ctx, host ints)
    for `parts` ranks: bounds (list of parts + 1 ints)."""
    c = (ctypes.c_int32 * len(ctx))(*[int(v) for v in ctx])
    b = (ctypes.c_int32 * (parts + 1))()
    _check(load_library().dsa_partition_decode_seqs(ctypes.cast(c, ctypes.c_void_p), len(ctx), k, d_I, d_qk,
                                                    parts, ctypes.cast(b, ctypes.c_void_p)))
    return list(b)


def device_status(stream=None) -> int:
    """Wait for the stream and return (and clear) the device status word."""
    return int(load_library().dsa_device_status(_stream(stream)))


def selftest_bounded_wait(limit_ms: int = 100, stream=None) -> int:
    """Run the failure-detection self-test and return the device status it left
    (DSA_ERR_TIMEOUT = -4 when the bounded wait gave up as it should)."""
    _check(load_library().dsa_selftest_bounded_wait(int(limit_ms), _stream(stream)))
    return device_status(stream)


PHASES = ("scores", "threshold", "select")


def phase_timing(enable: bool) -> None:
    """Turn the indexer's per-phase event timing on or off (diagnostic)."""
    _check(load_library().dsa_phase_timing(int(bool(enable))))


def phase_times() -> dict:
    """Milliseconds per indexer phase since the last read (waits for the events)."""
    buf = (ctypes.c_double * len(PHASES))()
    _check(load_library().dsa_phase_times(ctypes.cast(buf, ctypes.c_void_p), len(PHASES)))
    return dict(zip(PHASES, list(buf)))


DEBUG_COUNTS = ("beyond_pos", "pad_inside", "dropped", "duplicate", "bad_page", "selection")


def debug_counters(reset: bool = True) -> dict:
    """Totals of the debug build's device checks (all 0 in the release build)."""
    buf = (ctypes.c_uint64 * len(DEBUG_COUNTS))()
    _check(load_library().dsa_debug_counters(ctypes.cast(buf, ctypes.c_void_p), len(DEBUG_COUNTS), int(reset)))
    return dict(zip(DEBUG_COUNTS, [int(v) for v in buf]))


def abi_version() -> int:
    return int(load_library().dsa_abi_version())


def launch_count() -> int:
    """Kernels launched through the library by this process so far."""
    return int(load_library().dsa_launch_count())
