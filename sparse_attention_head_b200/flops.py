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
