"""The streaming top-k policy of the fused indexer kernel, replayed on the CPU
and checked against brute force.

The model takes the kernel's decisions in the kernel's order: appends that
pass (tau, tau_idx), a check every CHECK_TILES tiles of 128 keys, shrinks by
the highest sample pivot with at least k entries at or above it (128 evenly
spaced samples, the same rank ladder), the exact cut when a shrink frees too
little, and the final selection (k largest, ties to the lower index). It
shares no code with the kernel. What it pins is the policy: the kept set can
never lose a member of the true top-k, on inputs built to stress it (long
tie runs, rising and falling scores, few distinct values).
"""
import zlib

import numpy as np
import pytest

CAP, M, CHECK_TILES = 4352, 128, 2
HEADROOM = CHECK_TILES * M
LADDER = (-4, -1, 2, 5, 9, 14, 22, 200)


def order_key(f):
    u = np.asarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = np.where(np.asarray(f, dtype=np.float32) == 0, 0, u)            # -0 -> +0
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def k_largest(keys, idx, k):
    """Exact: sort by (key desc, index asc), keep k."""
    order = np.lexsort((idx, -keys.astype(np.int64)))
    return order[:k]


def pivots(keys, k):
    n = len(keys)
    samp = keys[(np.arange(128) * n) >> 7]
    # rank by (key desc, slot asc)
    order = np.lexsort((np.arange(128), -samp.astype(np.int64)))
    rank = np.empty(128, dtype=np.int64)
    rank[order] = np.arange(128)
    t0 = (k * 128) // n
    piv = [int(samp[rank == min(127, max(0, t0 + d))][0]) for d in LADDER]
    counts = [int((keys >= p).sum()) for p in piv]
    lo, c_lo, hi, c_hi, has_hi = 0, n, 0, 0, False
    for p, c in zip(piv, counts):
        if c >= k:
            lo, c_lo = p, c
            break
        hi, c_hi, has_hi = p, c, True
    return lo, c_lo, hi, c_hi, has_hi


def stream_select(keys_row, k):
    """Replay one row; returns the selected key indices."""
    n_keys = len(keys_row)
    buf_u, buf_i = [], []
    tau, tau_idx = 0, 0xFFFFFFFF
    n_tiles = (n_keys + M - 1) // M
    for t in range(n_tiles):
        s = np.arange(t * M, min(n_keys, (t + 1) * M))
        u = keys_row[s]
        take = (u > tau) | ((u == tau) & (s <= tau_idx))
        buf_u.extend(u[take].tolist())
        buf_i.extend(s[take].tolist())
        assert len(buf_u) <= CAP, "buffer overflow"
        if t % CHECK_TILES == CHECK_TILES - 1 and t + 1 < n_tiles and len(buf_u) > CAP - HEADROOM:
            bu, bi = np.array(buf_u, dtype=np.uint64), np.array(buf_i, dtype=np.int64)
            lo, c_lo, *_ = pivots(bu, k)
            keep = bu >= lo
            tau, tau_idx = lo, 0xFFFFFFFF
            if keep.sum() > CAP - 2 * HEADROOM:      # exact cut
                sel = k_largest(bu, bi, k)
                kth = bu[sel].min()
                tied = bi[sel][bu[sel] == kth]
                tau, tau_idx = int(kth), (int(tied.max()) if (bu == kth).sum() > len(tied) else 0xFFFFFFFF)
                keep = np.zeros(len(bu), dtype=bool)
                keep[sel] = True
            buf_u, buf_i = bu[keep].tolist(), bi[keep].tolist()
    bu, bi = np.array(buf_u, dtype=np.uint64), np.array(buf_i, dtype=np.int64)
    if len(bu) <= k:
        return np.sort(bi)
    return np.sort(bi[k_largest(bu, bi, k)])


def brute(keys_row, k):
    return np.sort(k_largest(keys_row, np.arange(len(keys_row)), k))


def _rows(kind, n, rng):
    if kind == "normal":
        return rng.standard_normal(n).astype(np.float32)
    if kind == "hot":
        x = rng.standard_normal(n).astype(np.float32)
        x[rng.choice(n, n // 20, replace=False)] += 3.0
        return x
    if kind == "rising":
        return np.linspace(-1, 1, n, dtype=np.float32) + rng.standard_normal(n).astype(np.float32) * 1e-3
    if kind == "falling":
        return np.linspace(1, -1, n, dtype=np.float32)
    if kind == "few_values":
        return rng.integers(0, 5, n).astype(np.float32)
    if kind == "all_equal":
        return np.full(n, 0.5, dtype=np.float32)
    if kind == "signed_zeros":
        x = np.where(rng.random(n) < 0.5, -0.0, 0.0).astype(np.float32)
        x[rng.choice(n, 100, replace=False)] = 1.0
        return x
    if kind == "tie_runs":
        x = np.round(rng.standard_normal(n) * 3).astype(np.float32)   # long runs of equal scores
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "hot", "rising", "falling", "few_values", "all_equal",
                                  "signed_zeros", "tie_runs"])
@pytest.mark.parametrize("n,k", [(3000, 2048), (20000, 2048), (65536, 2048), (9000, 100)])
def test_streaming_policy_is_exact(kind, n, k):
    rng = np.random.default_rng(zlib.crc32(f"{kind}/{n}/{k}".encode()))
    keys = order_key(_rows(kind, n, rng))
    got = stream_select(keys, k)
    want = brute(keys, k)
    assert np.array_equal(got, want)


def test_order_key_is_monotone_and_folds_signed_zero():
    x = np.array([-np.inf, -3.0, -1e-30, -0.0, 0.0, 1e-30, 2.0, np.inf], dtype=np.float32)
    u = order_key(x)
    assert (np.diff(u.astype(np.int64)) >= 0).all() and u[3] == u[4]
