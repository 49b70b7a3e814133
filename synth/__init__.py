"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) hot path.

This module only draws and encodes inputs (random numbers, FP8/BF16 encoding,
packing of decode caches). It holds none of the method's arithmetic, and it is
the only code shared by the CUDA path's tests/bench and the CPU oracle.

Workload recipes (DeepSeek-V3.2 breakdown page, section 2 "Architecture: DSA";
the research summary page, "Key points": 2048 selected tokens, few FP8 indexer
heads, MLA in MQA mode, 128K context):

* ``tiny``        L=256, H_I=4, d_I=32, k=32, Hq=4, d_qk=80 (64 latent + 16
                  rope), d_v=64. Indexer q/k integers uniform in [-4, 4] (exact
                  in e4m3), w integers in [-2, 2]; main q/kv ~ N(0,1) -> bf16;
                  scale 1/sqrt(80).
* ``prefill4k``   L=4096, H_I=8, d_I=128, k=2048, Hq=128, d_qk=576 (512 + 64),
                  d_v=512. Indexer q/k = e4m3(clip(N(0,1), +-448)),
                  w ~ N(0,1)/sqrt(8); q/kv ~ N(0,1) -> bf16; scale 1/sqrt(576).
* ``prefill32k``  as prefill4k with L=32768.
* ``prefill32k_int`` as prefill32k with integer indexer inputs (as ``tiny``).
* ``prefill128k`` as prefill4k with L=131072.
* ``decode``      64 sequences, one query each, context lengths uniform in
                  [8192, 131072]; packed FP8 key cache (d_I=128) and bf16
                  latent cache (576); H_I=8, Hq=128, k=2048, d_v=512.

Every tensor has its own seed, derived from (base seed, config, tensor name,
chunk), so a tensor can be regenerated independently of the others and of the
chunking used on the device.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0

CONFIGS = {
    "tiny": dict(kind="prefill", L=256, H_I=4, d_I=32, k=32, Hq=4, d_qk=80, d_v=64,
                 indexer="int"),
    "prefill4k": dict(kind="prefill", L=4096, H_I=8, d_I=128, k=2048, Hq=128, d_qk=576,
                      d_v=512, indexer="normal"),
    "prefill32k": dict(kind="prefill", L=32768, H_I=8, d_I=128, k=2048, Hq=128, d_qk=576,
                       d_v=512, indexer="normal"),
    "prefill32k_int": dict(kind="prefill", L=32768, H_I=8, d_I=128, k=2048, Hq=128,
                           d_qk=576, d_v=512, indexer="int"),
    "prefill128k": dict(kind="prefill", L=131072, H_I=8, d_I=128, k=2048, Hq=128,
                        d_qk=576, d_v=512, indexer="normal"),
    "decode": dict(kind="decode", B=64, ctx_lo=8192, ctx_hi=131072, H_I=8, d_I=128, k=2048,
                   Hq=128, d_qk=576, d_v=512, indexer="normal"),
}

# rows of a large tensor drawn per seed; keeps device temporaries bounded
_CHUNK_ELEMS = 1 << 27


def tensor_seed(base: int, config: str, name: str, chunk: int = 0) -> int:
    return zlib.crc32(f"{base}:{config}:{name}:{chunk}".encode()) & 0x7FFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _rows_per_chunk(row_elems: int) -> int:
    return max(1, _CHUNK_ELEMS // max(1, row_elems))


def normal(shape, base, config, name, device, dtype=torch.float32, scale=1.0):
    """N(0, scale^2) samples, drawn in fp32 chunk by chunk along dim 0, cast to dtype."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype, device=device)
    if out.numel() == 0:
        return out
    row = int(math.prod(shape[1:])) if len(shape) > 1 else 1
    step = _rows_per_chunk(row)
    for c, r0 in enumerate(range(0, shape[0], step)):
        r1 = min(shape[0], r0 + step)
        g = _gen(device, tensor_seed(base, config, name, c))
        x = torch.randn((r1 - r0,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out[r0:r1] = x.to(dtype)
    return out


def integers(shape, lo, hi, base, config, name, device):
    """Integers uniform in [lo, hi] (inclusive), returned as fp32."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.float32, device=device)
    if out.numel() == 0:
        return out
    row = int(math.prod(shape[1:])) if len(shape) > 1 else 1
    step = _rows_per_chunk(row)
    for c, r0 in enumerate(range(0, shape[0], step)):
        r1 = min(shape[0], r0 + step)
        g = _gen(device, tensor_seed(base, config, name, c))
        out[r0:r1] = torch.randint(lo, hi + 1, (r1 - r0,) + shape[1:], generator=g,
                                   device=device, dtype=torch.int32).float()
    return out


def to_e4m3_bytes(x: torch.Tensor) -> torch.Tensor:
    """Encode fp32 as OCP FP8 E4M3 (round to nearest even, saturated to +-448) -> uint8."""
    return x.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


@dataclass
class DSAInputs:
    """One batch of DSA inputs. FP8 tensors hold raw e4m3 bytes (uint8)."""
    config: str
    q_idx: torch.Tensor      # uint8 (e4m3) [T, H_I, d_I]
    w: torch.Tensor          # fp32 [T, H_I]
    k_idx: torch.Tensor      # uint8 (e4m3) [S, d_I]
    q: torch.Tensor          # bf16 [T, Hq, d_qk]
    kv: torch.Tensor         # bf16 [S, d_qk]
    pos: Optional[torch.Tensor]     # int32 [T] or None (suffix-aligned causal)
    k_base: Optional[torch.Tensor]  # int32 [T] or None (single sequence)
    k: int
    scale: float
    d_v: int
    meta: dict = field(default_factory=dict)

    @property
    def T(self):
        return self.q_idx.shape[0]

    @property
    def S(self):
        return self.k_idx.shape[0]

    def positions(self) -> torch.Tensor:
        """Explicit pos[t] (last visible key of row t, relative to k_base[t])."""
        if self.pos is not None:
            return self.pos
        return torch.arange(self.T, dtype=torch.int32, device=self.q_idx.device) + (self.S - self.T)

    def bases(self) -> torch.Tensor:
        if self.k_base is not None:
            return self.k_base
        return torch.zeros(self.T, dtype=torch.int32, device=self.q_idx.device)

    def to(self, device) -> "DSAInputs":
        mv = lambda t: None if t is None else t.to(device)
        return DSAInputs(self.config, mv(self.q_idx), mv(self.w), mv(self.k_idx), mv(self.q),
                         mv(self.kv), mv(self.pos), mv(self.k_base), self.k, self.scale,
                         self.d_v, dict(self.meta))


def _indexer_tensors(cfg, name, T, S, base, device, with_main=True):
    H_I, d_I = cfg["H_I"], cfg["d_I"]
    if cfg["indexer"] == "int":
        q_idx = to_e4m3_bytes(integers((T, H_I, d_I), -4, 4, base, name, "q_idx", device))
        k_idx = to_e4m3_bytes(integers((S, d_I), -4, 4, base, name, "k_idx", device))
        w = integers((T, H_I), -2, 2, base, name, "w", device)
    else:
        q_idx = to_e4m3_bytes(normal((T, H_I, d_I), base, name, "q_idx", device))
        k_idx = to_e4m3_bytes(normal((S, d_I), base, name, "k_idx", device))
        w = normal((T, H_I), base, name, "w", device, scale=1.0 / math.sqrt(H_I))
    return q_idx, w, k_idx


def prefill_inputs(name: str = "prefill4k", device="cpu", seed: int = 0, L: int = None,
                   overrides: dict = None, T: int = None) -> DSAInputs:
    """One causal prefill sequence of L tokens: S = L keys; the queries are its
    last T tokens (T = L by default; T < L is a chunked prefill of the tail),
    pos[t] = t + L - T, k_base = 0."""
    cfg = dict(CONFIGS[name])
    if overrides:
        cfg.update(overrides)
    if L is not None:
        cfg["L"] = L
    L = cfg["L"]
    T = L if T is None else int(T)
    assert 0 < T <= L
    q_idx, w, k_idx = _indexer_tensors(cfg, name, T, L, seed, device)
    q = normal((T, cfg["Hq"], cfg["d_qk"]), seed, name, "q", device, dtype=torch.bfloat16)
    kv = normal((L, cfg["d_qk"]), seed, name, "kv", device, dtype=torch.bfloat16)
    return DSAInputs(name, q_idx, w, k_idx, q, kv, None, None, cfg["k"],
                     1.0 / math.sqrt(cfg["d_qk"]), cfg["d_v"], meta=cfg)


def varlen_prefill_inputs(name: str = "prefill4k", device="cpu", seed: int = 0, lens=(700, 1500),
                          overrides: dict = None) -> DSAInputs:
    """A packed batch of causal prefill sequences (full prefill: each sequence's
    queries are all of its tokens). Sequence b owns rows [cu[b], cu[b+1]) of the
    query tensors and of the key caches; pos[t] is the row's index within its
    sequence and k_base[t] = cu[b]. meta["cu"] holds the offsets."""
    cfg = dict(CONFIGS[name])
    if overrides:
        cfg.update(overrides)
    lens = [int(v) for v in lens]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    total = cu[-1]
    q_idx, w, k_idx = _indexer_tensors(cfg, name + ":varlen", total, total, seed, device)
    q = normal((total, cfg["Hq"], cfg["d_qk"]), seed, name + ":varlen", "q", device, dtype=torch.bfloat16)
    kv = normal((total, cfg["d_qk"]), seed, name + ":varlen", "kv", device, dtype=torch.bfloat16)
    pos = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens]).to(device)
    k_base = torch.cat([torch.full((n,), c, dtype=torch.int32) for n, c in zip(lens, cu)]).to(device)
    meta = dict(cfg, cu=cu)
    return DSAInputs(name + ":varlen", q_idx, w, k_idx, q, kv, pos, k_base, cfg["k"],
                     1.0 / math.sqrt(cfg["d_qk"]), cfg["d_v"], meta=meta)


def page_caches(x: DSAInputs, page_size: int, seed: int = 0, spare_pages: int = 3):
    """Scatter the per-sequence caches of decode/packed inputs x (rows
    [k_base, k_base + pos + 1) per query row, one row per sequence) into a
    shuffled pool of pages. Returns (k_pages, kv_pages, block_table [n_seqs,
    max_pages], seq [T]); unused block-table entries are -1."""
    base = x.bases().cpu().long().tolist()
    n = (x.positions().cpu().long() + 1).tolist()
    pages = [(c + page_size - 1) // page_size for c in n]
    total = sum(pages) + spare_pages
    g = _gen("cpu", tensor_seed(seed, x.config, f"pages{page_size}"))
    perm = torch.randperm(total, generator=g).tolist()
    dev = x.k_idx.device
    k_pages = torch.zeros((total * page_size, x.k_idx.shape[1]), dtype=x.k_idx.dtype, device=dev)
    kv_pages = torch.zeros((total * page_size, x.kv.shape[1]), dtype=x.kv.dtype, device=dev)
    max_pages = max(pages)
    table = torch.full((len(n), max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b, (b0, c, npg) in enumerate(zip(base, n, pages)):
        for j in range(npg):
            pid = perm[nxt]
            nxt += 1
            table[b, j] = pid
            lo, hi = j * page_size, min(c, (j + 1) * page_size)
            k_pages[pid * page_size: pid * page_size + hi - lo] = x.k_idx[b0 + lo: b0 + hi]
            kv_pages[pid * page_size: pid * page_size + hi - lo] = x.kv[b0 + lo: b0 + hi]
    seq = torch.arange(len(n), dtype=torch.int32, device=dev)
    return k_pages, kv_pages, table.to(dev), seq


def decode_inputs(name: str = "decode", device="cpu", seed: int = 0, B: int = None,
                  ctx: list = None, overrides: dict = None) -> DSAInputs:
    """B sequences with one query each, keys packed per sequence in one cache.

    Sequence b owns cache rows [k_base[b], k_base[b] + ctx[b]); its query sees
    all of them: pos[b] = ctx[b] - 1.
    """
    cfg = dict(CONFIGS[name])
    if overrides:
        cfg.update(overrides)
    if B is not None:
        cfg["B"] = B
    B = cfg["B"]
    if ctx is None:
        g = _gen("cpu", tensor_seed(seed, name, "ctx"))
        ctx = torch.randint(cfg["ctx_lo"], cfg["ctx_hi"] + 1, (B,), generator=g).tolist()
    ctx = [int(c) for c in ctx]
    base = [0]
    for c in ctx[:-1]:
        base.append(base[-1] + c)
    S = sum(ctx)
    q_idx, w, k_idx = _indexer_tensors(cfg, name, B, S, seed, device)
    q = normal((B, cfg["Hq"], cfg["d_qk"]), seed, name, "q", device, dtype=torch.bfloat16)
    kv = normal((S, cfg["d_qk"]), seed, name, "kv", device, dtype=torch.bfloat16)
    pos = torch.tensor([c - 1 for c in ctx], dtype=torch.int32, device=device)
    k_base = torch.tensor(base, dtype=torch.int32, device=device)
    meta = dict(cfg)
    meta["ctx"] = ctx
    return DSAInputs(name, q_idx, w, k_idx, q, kv, pos, k_base, cfg["k"],
                     1.0 / math.sqrt(cfg["d_qk"]), cfg["d_v"], meta=meta)


def make_inputs(name: str, device="cpu", seed: int = 0, **kw) -> DSAInputs:
    if CONFIGS[name]["kind"] == "decode":
        return decode_inputs(name, device, seed, **kw)
    return prefill_inputs(name, device, seed, **kw)


def sample_rows(T: int, k: int, n: int, seed: int = 0) -> list:
    """Query rows checked at large L: 0, k-1, k, T-1 plus a seeded random set."""
    fixed = [r for r in (0, k - 1, k, T - 1) if 0 <= r < T]
    g = _gen("cpu", tensor_seed(seed, "rows", str(T)))
    rest = torch.randperm(T, generator=g)[: max(0, n)].tolist()
    out = []
    for r in fixed + rest:
        if r not in out:
            out.append(r)
        if len(out) >= max(n, len(fixed)):
            break
    return sorted(out)


def selection(pos, k: int, seed: int = 0) -> torch.Tensor:
    """A valid selection for every query row that depends on no score: int32
    [T, k] (CPU) holding min(k, n_t) distinct s in [0, n_t) first and -1 after,
    n_t = pos[t] + 1. Row t takes s_i = (a_t * i + b_t) mod n_t, i = 0, 1, ...,
    with a_t drawn coprime to n_t (so the s_i are distinct) and b_t uniform."""
    pos = np.asarray(pos.cpu() if hasattr(pos, "cpu") else pos, dtype=np.int64)
    T = pos.shape[0]
    out = np.full((T, k), -1, np.int32)
    rng = np.random.default_rng(tensor_seed(seed, "selection", str(k)))
    n = np.maximum(pos + 1, 0)
    a = rng.integers(1, np.maximum(n, 1) + 1)
    bad = np.gcd(a, np.maximum(n, 1)) != 1
    while bad.any():
        a[bad] = rng.integers(1, n[bad] + 1)
        bad = np.gcd(a, np.maximum(n, 1)) != 1
    b = rng.integers(0, np.maximum(n, 1))
    i = np.arange(k, dtype=np.int64)
    step = max(1, (1 << 24) // max(k, 1))
    for r0 in range(0, T, step):
        r1 = min(T, r0 + step)
        nn = n[r0:r1, None]
        s = (a[r0:r1, None] * i[None, :] + b[r0:r1, None]) % np.maximum(nn, 1)
        out[r0:r1] = np.where(i[None, :] < nn, s, -1)
    return torch.from_numpy(out)


def grad_out(x: DSAInputs, seed: int = 0) -> torch.Tensor:
    """dL/dout of the attention output: bf16 N(0, 1) [T, Hq, d_v] on x's device."""
    return normal((x.T, x.q.shape[1], x.d_v), seed, x.config, "dout", x.q.device, dtype=torch.bfloat16)


# MLA in MHA mode: per-head query/key dims 192 (128 expanded from the latent
# row + the 64 rope dims) and value dims 128, for a short prefill (L <= k).
MHA_CONFIGS = {
    "mha_short": dict(L=2048, Hq=128, d_h=192, d_hv=128),
    "mha_small": dict(L=300, Hq=4, d_h=64, d_hv=64),
}


def mha_inputs(name: str = "mha_short", device="cpu", seed: int = 0, L: int = None, T: int = None,
               Hq: int = None):
    """(q [T, Hq, d_h], k [L, Hq, d_h], v [L, Hq, d_hv], scale): bf16 N(0, 1),
    the queries being the last T of the L tokens; scale 1/sqrt(d_h)."""
    cfg = dict(MHA_CONFIGS[name])
    if L is not None:
        cfg["L"] = L
    if Hq is not None:
        cfg["Hq"] = Hq
    L, H, dh, dv = cfg["L"], cfg["Hq"], cfg["d_h"], cfg["d_hv"]
    T = L if T is None else int(T)
    q = normal((T, H, dh), seed, name, "q", device, dtype=torch.bfloat16)
    k = normal((L, H, dh), seed, name, "k", device, dtype=torch.bfloat16)
    v = normal((L, H, dv), seed, name, "v", device, dtype=torch.bfloat16)
    return q, k, v, 1.0 / math.sqrt(dh)
