"""The bound the decode-form Top-k select rests on, checked on the host in
order-key space ("Paper Breakdown: DeepSeek-V3.2", section 2, "Top-k
selector"): with the scores cut into groups, the k-th largest group maximum
is reached by at least k groups, so by at least k scores. Rounding it down
to the lower edge of a histogram bin, then a sub-bin (as the kernel does,
restated here), keeps that property, so the scores at or above the
threshold hold the row's exact Top-k. Groups are the score kernel's: 16
consecutive keys, or 4 keys (rows gid, gid + 1, gid + 8, gid + 9 of a warp's
16) inside each 128-key tile; an empty group (past the row's end) has key 0.
No GPU."""
import zlib

import numpy as np
import pytest

BINS = 2048


def order_keys(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return np.where(b & 0x80000000, (~b) & 0xFFFFFFFF, b | 0x80000000).astype(np.uint64)


def kth_bin(idx, k):
    """Bin holding the k-th entry from the top, and k minus the entries above it."""
    counts = np.bincount(idx, minlength=BINS)
    above = 0
    for b in range(len(counts) - 1, -1, -1):
        if above + counts[b] >= k:
            return b, k - above
        above += counts[b]
    raise AssertionError("fewer than k entries")


def range_floor(v, k):
    v = v[v != 0]
    if len(v) < k:
        return 0
    lo, hi = int(v.min()), int(v.max())
    if lo == hi:
        return lo
    shift = max(0, (hi - lo).bit_length() - 11)
    kb, need = kth_bin(((v - lo) >> shift).astype(np.int64), k)
    b0 = lo + (kb << shift)
    if shift == 0:
        return b0
    shift2 = max(0, shift - 11)
    inb = v[((v - lo) >> shift) == kb]
    kb2, _ = kth_bin(((inb - b0) >> shift2).astype(np.int64), need)
    return b0 + (kb2 << shift2)


def group_maxima(keys, size):
    n = len(keys)
    tiles = (n + 127) // 128
    pad = np.zeros(tiles * 128, dtype=np.uint64)
    pad[:n] = keys
    t = pad.reshape(tiles, 8, 16)            # tile, scoring warp, row of the warp's 16
    if size == 16:
        return t.max(axis=2).reshape(-1)
    g = np.stack([t[:, :, [2 * p, 2 * p + 1, 2 * p + 8, 2 * p + 9]].max(axis=2) for p in range(4)], axis=2)
    return g.reshape(-1)


ROWS = [
    ("normal", 40000, lambda r, n: r.standard_normal(n)),
    ("relu_sum", 70000, lambda r, n: np.maximum(r.standard_normal((n, 8)), 0) @ r.uniform(-0.2, 1, 8)),
    ("ties", 50000, lambda r, n: r.integers(-3, 4, n).astype(np.float64)),
    ("sorted_runs", 33000, lambda r, n: np.sort(r.standard_normal(n))),
    ("ragged", 9001, lambda r, n: r.standard_normal(n) * 100),
]


@pytest.mark.parametrize("name,n,draw", ROWS)
@pytest.mark.parametrize("size", [16, 4])
@pytest.mark.parametrize("k", [2048, 256])
def test_group_maximum_threshold_keeps_the_top_k(name, n, draw, size, k):
    rng = np.random.default_rng(zlib.crc32(f"{name}/{size}/{k}".encode()))
    keys = order_keys(draw(rng, n))
    gm = group_maxima(keys, size)
    if np.count_nonzero(gm) < k:
        pytest.skip("fewer than k groups: the kernel keeps every score")
    tau = range_floor(gm, k)
    kth = np.sort(keys)[::-1][k - 1]
    assert tau <= kth                                  # a lower bound of the k-th largest score
    assert np.count_nonzero(keys >= tau) >= k
    # and no looser than the group bound it rounds: the bin edge is within
    # one sub-bin of the k-th largest group maximum
    gk = np.sort(gm)[::-1][k - 1]
    assert tau <= gk


def test_four_key_groups_cover_each_key_once():
    keys = np.arange(1, 257, dtype=np.uint64)
    g = group_maxima(keys, 4)
    assert len(g) == 64 and sorted(g.tolist()) == sorted(
        [int(keys[t * 128 + w * 16 + 2 * p + 9]) for t in range(2) for w in range(8) for p in range(4)])
