"""Host-side checks of the C-ABI library (no GPU): it builds for sm_100a, loads,
exports every symbol include/dsa.h declares, sizes workspaces, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build

HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa.load_library()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(dsa.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_build_targets_sm100a():
    flags = " ".join(dsa_build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags


def test_abi_version_and_empty_error(lib):
    assert lib.dsa_abi_version() == 1
    assert isinstance(lib.dsa_last_error(), bytes)


def test_workspace_sizes(lib):
    # 128K prefill: bounded per block of query rows (sampled scores + candidate
    # buffers of 32768 rows: 32768 * (4096 * 4 + 8192 * 8) bytes)
    ws = dsa.workspace_size(131072, 131072, 8, 128, 2048, 128, 576, 512)
    assert 0 < ws <= 32768 * (4096 * 4 + 8192 * 8) + (1 << 20)
    assert dsa.workspace_size(0, 10, 8, 128, 2048, 128, 576, 512) == 0
    small = dsa.workspace_size(256, 256, 4, 32, 32, 4, 80, 64)
    assert 0 < small < 1 << 20
    # decode-like: 64 rows over a 4.5M-key packed cache stay within one block
    dec = dsa.workspace_size(64, 4_500_000, 8, 128, 2048, 128, 576, 512)
    assert 0 < dec <= 1 << 30
    # the decode form of 64 rows over 128K keys: each row's dense score row
    # (131072 x 4 B) and its 16-key and 4-key group maxima ((8192 + 32768) x 4 B)
    assert dsa.workspace_size(64, 131072, 8, 128, 2048, 128, 576, 512) == 64 * (131072 + 8192 + 32768) * 4


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: checks fail first
ODD = ctypes.c_void_p(0x10004)


def test_indexer_rejects_bad_arguments(lib):
    f = lib.dsa_indexer_topk
    ws = ctypes.c_size_t(1 << 20)
    # NULL pointer
    assert f(None, FAKE, FAKE, None, None, 4, 4, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    assert b"NULL" in lib.dsa_last_error()
    # misaligned
    assert f(ODD, FAKE, FAKE, None, None, 4, 4, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    # sizes
    assert f(FAKE, FAKE, FAKE, None, None, 0, 4, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    assert f(FAKE, FAKE, FAKE, None, None, 8, 4, 8, 128, 2, FAKE, FAKE, ws, None) == -1  # T > S
    # unsupported dims
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 17, 128, 2, FAKE, FAKE, ws, None) == -2
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 8, 96, 2, FAKE, FAKE, ws, None) == -2
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 8, 128, 4097, FAKE, FAKE, ws, None) == -2
    # workspace too small
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 8, 128, 2, FAKE, FAKE, ctypes.c_size_t(8),
             None) == -5


def test_attention_rejects_bad_arguments(lib):
    f = lib.dsa_sparse_mla_attn
    ws = ctypes.c_size_t(1 << 20)
    sc = ctypes.c_float(0.1)
    assert f(FAKE, None, FAKE, None, None, 4, 4, 128, 576, 512, 64, sc, FAKE, FAKE, FAKE, ws,
             None) == -1
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 128, 570, 512, 64, sc, FAKE, FAKE, FAKE, ws,
             None) == -2
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 128, 576, 577, 64, sc, FAKE, FAKE, FAKE, ws,
             None) == -2
    assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 2000, 576, 512, 64, sc, FAKE, FAKE, FAKE, ws,
             None) == -2


def test_split_attention_arguments_and_workspace(lib):
    f = lib.dsa_sparse_mla_attn_split
    ws = ctypes.c_size_t(1 << 30)
    sc = ctypes.c_float(0.1)
    for bad in (-1, 17):
        assert f(FAKE, FAKE, FAKE, None, None, 4, 4, 128, 576, 512, 64, sc, bad, FAKE, FAKE, FAKE, ws,
                 None) == -1
        assert b"splits" in lib.dsa_last_error()
    # 4 parts of 64 rows need room for every part's fp32 output and log-sum-exp
    need = lib.dsa_sparse_mla_attn_split_workspace_size(64, 128, 512, 4)
    assert need >= 64 * 4 * 128 * (512 + 1) * 4
    assert lib.dsa_sparse_mla_attn_split_workspace_size(64, 128, 512, 1) == 0
    assert f(FAKE, FAKE, FAKE, None, None, 64, 64, 128, 576, 512, 64, sc, 4, FAKE, FAKE, FAKE,
             ctypes.c_size_t(need - 1), None) == -5


def test_attention_backward_rejects_bad_arguments(lib):
    f = lib.dsa_sparse_mla_attn_bwd
    sc = ctypes.c_float(0.1)
    ws = ctypes.c_size_t(1 << 20)

    def call(Hq=128, d_qk=576, d_v=512, k=64, dout=FAKE, wsb=ws, wsp=FAKE):
        return f(FAKE, FAKE, FAKE, None, None, FAKE, FAKE, dout, 4, 4, Hq, d_qk, d_v, k, sc, FAKE, FAKE,
                 wsp, wsb, None)

    assert call(dout=None) == -1
    assert call(Hq=129) == -2            # more heads than the backward takes
    assert call(d_qk=584, d_v=512) == -2  # d_qk above 576
    assert call(d_qk=576, d_v=504) == -2  # d_v not a multiple of 16
    assert call(wsb=ctypes.c_size_t(100)) == -5
    assert call(wsp=None) == -5
    # one row of scratch: g (bf16, heads padded to 16, slots to 64) and D (fp32 per head)
    assert lib.dsa_sparse_mla_attn_bwd_workspace_size(1, 4, 32) == 16 * 64 * 2 + 16 * 4
    assert lib.dsa_sparse_mla_attn_bwd_workspace_size(100000, 128, 2048) == 8192 * 128 * (2048 * 2 + 4)
    assert lib.dsa_sparse_mla_attn_bwd_workspace_size(0, 128, 2048) == 0


def test_indexer_kl_rejects_bad_arguments(lib):
    f = lib.dsa_indexer_kl
    sc = ctypes.c_float(0.1)

    def call(Hq=128, d_qk=576, H_I=8, d_I=128, k=64, lse=FAKE, wsb=ctypes.c_size_t(1 << 20), wsp=FAKE):
        return f(FAKE, FAKE, FAKE, None, None, lse, FAKE, FAKE, FAKE, 4, 4, Hq, d_qk, H_I, d_I, k, sc, FAKE,
                 FAKE, FAKE, FAKE, wsp, wsb, None)

    assert call(lse=None) == -1
    assert call(Hq=256) == -2
    assert call(H_I=17) == -2
    assert call(d_I=136) == -2          # not a multiple of 16
    assert call(H_I=16, d_I=512) == -2  # above 256
    assert call(k=5000) == -2
    assert call(wsb=ctypes.c_size_t(16)) == -5
    assert lib.dsa_indexer_kl_workspace_size(1, 2048) == 2048 * 4
    assert lib.dsa_indexer_kl_workspace_size(50000, 100) == 8192 * 128 * 4
    assert lib.dsa_indexer_kl_workspace_size(0, 100) == 0


def test_mha_rejects_bad_arguments(lib):
    f = lib.dsa_mla_mha_attn
    sc = ctypes.c_float(0.1)
    assert f(FAKE, None, FAKE, 4, 4, 8, 192, 128, sc, FAKE, FAKE, None) == -1
    assert f(FAKE, FAKE, FAKE, 5, 4, 8, 192, 128, sc, FAKE, FAKE, None) == -1   # T > S
    assert f(FAKE, FAKE, FAKE, 4, 4, 8, 128, 128, sc, FAKE, FAKE, None) == -2   # head dims


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((4, 8, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        dsa.indexer_topk(x, torch.zeros(4, 8), torch.zeros((4, 128), dtype=torch.uint8), 2)
    q = torch.zeros((4, 2, 64), dtype=torch.bfloat16)
    kv = torch.zeros((4, 64), dtype=torch.bfloat16)
    idx = torch.zeros((4, 2), dtype=torch.int32)
    out = torch.zeros((4, 2, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dsa.sparse_mla_attn_bwd(q, kv, idx, out, torch.zeros(4, 2), out, 0.1)
    with pytest.raises(ValueError):
        dsa.indexer_kl(q, kv, idx, torch.zeros(4, 2), x, torch.zeros(4, 8), torch.zeros((4, 128), dtype=torch.uint8),
                       0.1)
    with pytest.raises(ValueError):
        dsa.mla_mha_attn(q, q, q, 0.1)


def test_product_and_oracle_share_no_code():
    pkg = os.path.join(ROOT, "sparse_attention_20_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in text.lower(), fn
    for fn in os.listdir(os.path.join(ROOT, "oracle")):
        if fn.endswith((".py", ".c", ".h")):
            text = open(os.path.join(ROOT, "oracle", fn)).read()
            assert "import sparse_attention_20_b200" not in text
            assert "dsa.h" not in text


def test_selftest_rejects_bad_limit(lib):
    # the argument check comes before any launch
    assert lib.dsa_selftest_bounded_wait(0, None) == -1
    assert lib.dsa_selftest_bounded_wait(2001, None) == -1
    assert b"limit_ms" in lib.dsa_last_error()


def test_varlen_rejects_bad_offsets(lib):
    f = lib.dsa_indexer_topk_varlen
    ws = ctypes.c_size_t(1 << 20)
    good = (ctypes.c_int32 * 3)(0, 4, 8)
    bad0 = (ctypes.c_int32 * 3)(1, 4, 8)
    fewer_keys = (ctypes.c_int32 * 3)(0, 4, 6)     # second sequence: 4 rows over 2 keys
    cq = (ctypes.c_int32 * 3)(0, 4, 8)
    P = lambda a: ctypes.cast(a, ctypes.c_void_p)
    assert f(FAKE, FAKE, FAKE, None, P(good), 2, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    assert f(FAKE, FAKE, FAKE, P(bad0), P(good), 2, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    assert f(FAKE, FAKE, FAKE, P(cq), P(fewer_keys), 2, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    assert b"sequence 1" in lib.dsa_last_error()
    assert f(FAKE, FAKE, FAKE, P(cq), P(good), 0, 8, 128, 2, FAKE, FAKE, ws, None) == -1


def test_paged_rejects_bad_arguments(lib):
    f = lib.dsa_indexer_topk_paged
    ws = ctypes.c_size_t(1 << 20)
    # page size not a multiple of 64
    assert f(FAKE, FAKE, FAKE, 4, 48, FAKE, 1, 2, FAKE, FAKE, 1, 8, 128, 2, FAKE, FAKE, ws, None) == -2
    # NULL block table
    assert f(FAKE, FAKE, FAKE, 4, 64, None, 1, 2, FAKE, FAKE, 1, 8, 128, 2, FAKE, FAKE, ws, None) == -1
    # d_I other than 128
    assert f(FAKE, FAKE, FAKE, 4, 64, FAKE, 1, 2, FAKE, FAKE, 1, 8, 64, 2, FAKE, FAKE, ws, None) == -2
    g = lib.dsa_sparse_mla_attn_paged
    sc = ctypes.c_float(0.1)
    assert g(FAKE, FAKE, 4, 64, FAKE, 1, 2, FAKE, FAKE, FAKE, 1, 4, 80, 64, 32, sc, FAKE, FAKE,
             None) == -2   # tensor-core shapes only
    assert g(FAKE, FAKE, 0, 64, FAKE, 1, 2, FAKE, FAKE, FAKE, 1, 128, 576, 512, 32, sc, FAKE, FAKE,
             None) == -1
