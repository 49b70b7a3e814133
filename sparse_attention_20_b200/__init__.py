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

DSA_OK = 0
STATUS_NAMES = {0: "DSA_OK", -1: "DSA_ERR_ARG", -2: "DSA_ERR_UNSUPPORTED", -3: "DSA_ERR_CUDA",
                -4: "DSA_ERR_TIMEOUT", -5: "DSA_ERR_WORKSPACE"}

# Every symbol include/dsa.h declares.
EXPORTS = ("dsa_workspace_size", "dsa_indexer_topk", "dsa_sparse_mla_attn", "dsa_forward",
           "dsa_device_status", "dsa_last_error", "dsa_abi_version", "dsa_launch_count",
           "dsa_indexer_topk_noalloc", "dsa_selftest_bounded_wait", "dsa_indexer_topk_varlen",
           "dsa_indexer_topk_paged", "dsa_sparse_mla_attn_paged", "dsa_sparse_mla_attn_bwd",
           "dsa_sparse_mla_attn_bwd_workspace_size", "dsa_indexer_kl", "dsa_indexer_kl_workspace_size",
           "dsa_mla_mha_attn")


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


def _fp8(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError(f"{name} must hold e4m3 bytes (uint8 or float8_e4m3fn), got {t.dtype}")
    return _dev(t, name)


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _i32(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if t.dtype != torch.int32:
        raise TypeError(f"{name} must be int32")
    return _dev(t, name)


def workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v) -> int:
    return int(load_library().dsa_workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v))


def alloc_workspace(T, S, H_I, d_I, k, Hq, d_qk, d_v, device=None) -> torch.Tensor:
    n = workspace_size(T, S, H_I, d_I, k, Hq, d_qk, d_v)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def indexer_topk(q_idx, w, k_idx, k: int, pos=None, k_base=None, idx=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """idx [T, k] int32: the Top-k s per query row (a set, -1 padded)."""
    q_idx = _fp8(q_idx, "q_idx")
    k_idx = _fp8(k_idx, "k_idx")
    w = _dev(w, "w")
    if w.dtype != torch.float32:
        raise TypeError("w must be float32")
    T, H_I, d_I = q_idx.shape
    S = k_idx.shape[0]
    pos, k_base = _i32(pos, "pos"), _i32(k_base, "k_base")
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=q_idx.device)
    if workspace is None:
        workspace = alloc_workspace(T, S, H_I, d_I, k, 1, 8, 2, q_idx.device)
    lib = load_library()
    _check(lib.dsa_indexer_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(pos), _ptr(k_base), T, S,
                                H_I, d_I, k, _ptr(idx), _ptr(workspace), workspace.numel(),
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
    q_idx = _fp8(q_idx, "q_idx")
    k_idx = _fp8(k_idx, "k_idx")
    w = _dev(w, "w")
    if w.dtype != torch.float32:
        raise TypeError("w must be float32")
    T, H_I, d_I = q_idx.shape
    cq = (ctypes.c_int32 * len(cu_q))(*[int(v) for v in cu_q])
    ck = (ctypes.c_int32 * len(cu_k))(*[int(v) for v in cu_k])
    if len(cu_q) != len(cu_k) or len(cu_q) < 2:
        raise ValueError("cu_q and cu_k need n_seqs + 1 >= 2 entries each")
    n = len(cu_q) - 1
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=q_idx.device)
    if workspace is None:
        t_max = max(cq[b + 1] - cq[b] for b in range(n))
        s_max = max(ck[b + 1] - ck[b] for b in range(n))
        workspace = alloc_workspace(max(t_max, 1), max(s_max, 1), H_I, d_I, k, 1, 8, 2, q_idx.device)
    _check(load_library().dsa_indexer_topk_varlen(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), ctypes.cast(cq, ctypes.c_void_p), ctypes.cast(ck, ctypes.c_void_p),
        n, H_I, d_I, k, _ptr(idx), _ptr(workspace), workspace.numel(), _stream(stream)))
    return idx


def indexer_topk_paged(q_idx, w, k_pages, page_size: int, block_table, seq, pos, k: int, idx=None,
                       workspace=None, stream=None) -> torch.Tensor:
    """idx [T, k] over a paged FP8 key cache (k_pages [num_pages*page_size, d_I],
    block_table [n_seqs, max_pages], seq / pos [T]; see include/dsa.h)."""
    q_idx, k_pages = _fp8(q_idx, "q_idx"), _fp8(k_pages, "k_pages")
    w = _dev(w, "w")
    block_table, seq, pos = _i32(block_table, "block_table"), _i32(seq, "seq"), _i32(pos, "pos")
    T, H_I, d_I = q_idx.shape
    num_pages = k_pages.shape[0] // page_size
    n_seqs, max_pages = block_table.shape
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=q_idx.device)
    if workspace is None:
        workspace = alloc_workspace(T, max_pages * page_size, H_I, d_I, k, 1, 8, 2, q_idx.device)
    _check(load_library().dsa_indexer_topk_paged(
        _ptr(q_idx), _ptr(w), _ptr(k_pages), num_pages, page_size, _ptr(block_table), n_seqs, max_pages,
        _ptr(seq), _ptr(pos), T, H_I, d_I, k, _ptr(idx), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return idx


def sparse_mla_attn_paged(q, kv_pages, page_size: int, block_table, seq, pos, idx, scale: float,
                          d_v: int, out=None, lse=None, stream=None):
    """(out, lse) of sparse MQA attention over a paged latent cache."""
    q, kv_pages = _dev(q, "q"), _dev(kv_pages, "kv_pages")
    if q.dtype != torch.bfloat16 or kv_pages.dtype != torch.bfloat16:
        raise TypeError("q and kv_pages must be bfloat16")
    block_table, seq, pos = _i32(block_table, "block_table"), _i32(seq, "seq"), _i32(pos, "pos")
    idx = _i32(idx, "idx")
    T, Hq, d_qk = q.shape
    num_pages = kv_pages.shape[0] // page_size
    n_seqs, max_pages = block_table.shape
    if out is None:
        out = torch.empty((T, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    _check(load_library().dsa_sparse_mla_attn_paged(
        _ptr(q), _ptr(kv_pages), num_pages, page_size, _ptr(block_table), n_seqs, max_pages, _ptr(seq),
        _ptr(pos), _ptr(idx), T, Hq, d_qk, d_v, idx.shape[1], float(scale), _ptr(out), _ptr(lse),
        _stream(stream)))
    return out, lse


def sparse_mla_attn(q, kv, idx, scale: float, d_v: int, pos=None, k_base=None, out=None,
                    lse=None, workspace=None, stream=None):
    """(out bf16 [T, Hq, d_v], lse fp32 [T, Hq]) of sparse MQA attention over idx."""
    q, kv = _dev(q, "q"), _dev(kv, "kv")
    if q.dtype != torch.bfloat16 or kv.dtype != torch.bfloat16:
        raise TypeError("q and kv must be bfloat16")
    idx = _i32(idx, "idx")
    T, Hq, d_qk = q.shape
    S = kv.shape[0]
    k = idx.shape[1]
    pos, k_base = _i32(pos, "pos"), _i32(k_base, "k_base")
    if out is None:
        out = torch.empty((T, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(T, S, 1, 32, k, Hq, d_qk, d_v, q.device)
    lib = load_library()
    _check(lib.dsa_sparse_mla_attn(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), T, S, Hq,
                                   d_qk, d_v, k, float(scale), _ptr(out), _ptr(lse),
                                   _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def sparse_mla_attn_bwd(q, kv, idx, out, lse, dout, scale: float, pos=None, k_base=None, dq=None,
                        dkv=None, workspace=None, stream=None):
    """(dq fp32 [T, Hq, d_qk], dkv fp32 [S, d_qk]) of sparse MQA attention over idx.

    out / lse are the forward's results for the same idx; dout is bf16
    [T, Hq, d_v]. dkv is accumulated into (a new zeroed tensor when None)."""
    q, kv = _dev(q, "q"), _dev(kv, "kv")
    out, dout, lse = _dev(out, "out"), _dev(dout, "dout"), _dev(lse, "lse")
    if any(t.dtype != torch.bfloat16 for t in (q, kv, out, dout)):
        raise TypeError("q, kv, out and dout must be bfloat16")
    idx = _i32(idx, "idx")
    T, Hq, d_qk = q.shape
    S, d_v, k = kv.shape[0], out.shape[2], idx.shape[1]
    pos, k_base = _i32(pos, "pos"), _i32(k_base, "k_base")
    if dq is None:
        dq = torch.empty((T, Hq, d_qk), dtype=torch.float32, device=q.device)
    if dkv is None:
        dkv = torch.zeros((S, d_qk), dtype=torch.float32, device=q.device)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_sparse_mla_attn_bwd_workspace_size(T, Hq, k)),
                                dtype=torch.uint8, device=q.device)
    _check(lib.dsa_sparse_mla_attn_bwd(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), _ptr(out),
                                       _ptr(lse), _ptr(dout), T, S, Hq, d_qk, d_v, k, float(scale),
                                       _ptr(dq), _ptr(dkv), _ptr(workspace), workspace.numel(),
                                       _stream(stream)))
    return dq, dkv


def indexer_kl(q, kv, idx, lse, q_idx, w, k_idx, scale: float, pos=None, k_base=None, dk_idx=None,
               workspace=None, stream=None):
    """Indexer KL loss over each row's selected set and its gradient:
    (loss fp32 [T], dw fp32 [T, H_I], dq_idx fp32 [T, H_I, d_I], dk_idx fp32 [S, d_I]).

    lse is the attention forward's log-sum-exp for the same idx. dk_idx is
    accumulated into (a new zeroed tensor when None)."""
    q, kv, lse, w = _dev(q, "q"), _dev(kv, "kv"), _dev(lse, "lse"), _dev(w, "w")
    q_idx, k_idx = _fp8(q_idx, "q_idx"), _fp8(k_idx, "k_idx")
    if q.dtype != torch.bfloat16 or kv.dtype != torch.bfloat16:
        raise TypeError("q and kv must be bfloat16")
    idx = _i32(idx, "idx")
    T, Hq, d_qk = q.shape
    _, H_I, d_I = q_idx.shape
    S, k = kv.shape[0], idx.shape[1]
    pos, k_base = _i32(pos, "pos"), _i32(k_base, "k_base")
    dev = q.device
    loss = torch.empty(T, dtype=torch.float32, device=dev)
    dw = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    dq_idx = torch.empty((T, H_I, d_I), dtype=torch.float32, device=dev)
    if dk_idx is None:
        dk_idx = torch.zeros((S, d_I), dtype=torch.float32, device=dev)
    lib = load_library()
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_indexer_kl_workspace_size(T, k)), dtype=torch.uint8, device=dev)
    _check(lib.dsa_indexer_kl(_ptr(q), _ptr(kv), _ptr(idx), _ptr(pos), _ptr(k_base), _ptr(lse), _ptr(q_idx),
                              _ptr(w), _ptr(k_idx), T, S, Hq, d_qk, H_I, d_I, k, float(scale), _ptr(loss),
                              _ptr(dw), _ptr(dq_idx), _ptr(dk_idx), _ptr(workspace), workspace.numel(),
                              _stream(stream)))
    return loss, dw, dq_idx, dk_idx


def mla_mha_attn(q, k, v, scale: float, out=None, lse=None, stream=None):
    """MLA in MHA mode, dense causal over one sequence: (out bf16 [T, Hq, d_hv],
    lse fp32 [T, Hq]); q [T, Hq, d_h], k [S, Hq, d_h], v [S, Hq, d_hv] bf16, the
    queries being the last T of the S tokens."""
    q, k, v = _dev(q, "q"), _dev(k, "k"), _dev(v, "v")
    if any(t.dtype != torch.bfloat16 for t in (q, k, v)):
        raise TypeError("q, k and v must be bfloat16")
    T, Hq, d_h = q.shape
    S, d_hv = k.shape[0], v.shape[2]
    if out is None:
        out = torch.empty((T, Hq, d_hv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    _check(load_library().dsa_mla_mha_attn(_ptr(q), _ptr(k), _ptr(v), T, S, Hq, d_h, d_hv, float(scale),
                                           _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def forward(q_idx, w, k_idx, q, kv, k: int, scale: float, d_v: int, pos=None, k_base=None,
            idx=None, out=None, lse=None, workspace=None, stream=None):
    """The whole hot path: (idx, out, lse)."""
    q_idx, k_idx = _fp8(q_idx, "q_idx"), _fp8(k_idx, "k_idx")
    q, kv, w = _dev(q, "q"), _dev(kv, "kv"), _dev(w, "w")
    T, H_I, d_I = q_idx.shape
    _, Hq, d_qk = q.shape
    S = k_idx.shape[0]
    pos, k_base = _i32(pos, "pos"), _i32(k_base, "k_base")
    dev = q.device
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((T, Hq, d_v), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(T, S, H_I, d_I, k, Hq, d_qk, d_v, dev)
    lib = load_library()
    _check(lib.dsa_forward(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(q), _ptr(kv), _ptr(pos),
                           _ptr(k_base), T, S, H_I, d_I, Hq, d_qk, d_v, k, float(scale), _ptr(idx),
                           _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                           _stream(stream)))
    return idx, out, lse


def device_status(stream=None) -> int:
    """Wait for the stream and return (and clear) the device status word."""
    return int(load_library().dsa_device_status(_stream(stream)))


def selftest_bounded_wait(limit_ms: int = 100, stream=None) -> int:
    """Run the failure-detection self-test and return the device status it left
    (DSA_ERR_TIMEOUT = -4 when the bounded wait gave up as it should)."""
    _check(load_library().dsa_selftest_bounded_wait(int(limit_ms), _stream(stream)))
    return device_status(stream)


def abi_version() -> int:
    return int(load_library().dsa_abi_version())


def launch_count() -> int:
    """Kernels launched through the library by this process so far."""
    return int(load_library().dsa_launch_count())
