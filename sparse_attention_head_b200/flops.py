"""Work counts of the hybrid prefill, used to turn times into TFLOP/s.

Effective work counts only visible (query, key) pairs: each costs d
multiply-adds in Q K^T and d in P V, i.e. 4 d flops.  The tile-granular count
is the work of every 128 x 128 score tile that holds at least one visible
pair, which is what the tensor cores actually execute.
"""
from __future__ import annotations

import numpy as np


def attn_visible_pairs(N: int, sparse: bool, sink: int, window: int) -> int:
    """Visible (i, j) pairs of one head: FA = causal; SA = sink + window."""
    if not sparse:
        return N * (N + 1) // 2
    i = np.arange(N, dtype=np.int64)
    win = np.minimum(i + 1, window)
    sink_left = np.minimum(sink, np.maximum(0, i - window + 1))
    return int(np.sum(win + sink_left))


def effective_flops(mask, N: int, d: int, sink: int, window: int) -> float:
    m = np.asarray(mask).reshape(-1)
    n_sa = int(np.count_nonzero(m))
    n_fa = m.size - n_sa
    pairs = n_fa * attn_visible_pairs(N, False, sink, window) + \
        n_sa * attn_visible_pairs(N, True, sink, window)
    return 4.0 * d * pairs


def _visible_tiles(N: int, sparse: bool, sink: int, window: int, bm: int = 128,
                   bn: int = 128) -> int:
    nt = (N + bm - 1) // bm
    total = 0
    for m in range(nt):
        r0 = m * bm
        imax = min(r0 + bm - 1, N - 1)
        c0 = np.arange(0, imax + 1, bn)
        if sparse:
            seen = (c0 < sink) | ((r0 - (c0 + bn - 1)) < window)
            total += int(np.count_nonzero(seen))
        else:
            total += len(c0)
    return total


def tile_flops(mask, N: int, d: int, sink: int, window: int) -> float:
    m = np.asarray(mask).reshape(-1)
    n_sa = int(np.count_nonzero(m))
    n_fa = m.size - n_sa
    tiles = n_fa * _visible_tiles(N, False, sink, window) + \
        n_sa * _visible_tiles(N, True, sink, window)
    return 4.0 * d * 128 * 128 * tiles


# ---------------------------------------------------------------- decode
def decode_group_rows(t: int, all_sparse: bool, sink: int, window: int) -> int:
    """Cache rows one kv group reads for the query at position t: every
    position 0..t when some query head of the group is FA, else the sink and
    window positions (j < S or t - j < W)."""
    if not all_sparse:
        return t + 1
    lo = max(0, t - window + 1)
    return min(sink, lo) + (t - lo + 1)


def decode_bytes(mask, pos, hkv: int, d: int, sink: int, window: int) -> dict:
    """Algorithmic HBM bytes of one decode step (bf16 everywhere):
    kv   = K and V rows every kv group reads once for all its query heads;
    io   = q read + out write + the new k, v rows read and appended."""
    m = np.asarray(mask, dtype=np.uint8)
    B, hq = m.shape
    g = hq // hkv
    all_sa = np.all(m.reshape(B, hkv, g) != 0, axis=2)
    row = 2 * d                                    # bytes of one bf16 row
    kv = 0
    for b in range(B):
        t = int(pos[b])
        for hk in range(hkv):
            kv += 2 * row * decode_group_rows(t, bool(all_sa[b, hk]), sink, window)
    io = 2 * B * hq * row + 2 * 2 * B * hkv * row
    return {"kv": kv, "io": io, "total": kv + io, "n_sa_groups": int(all_sa.sum()),
            "n_groups": int(B * hkv)}
