"""Host mirror of the backward kernels' work schedule (the per-CTA unit
lists that ea_bwd_sched_kernel writes into the backward workspace), for the
tests: unit costs, the sort by decreasing cost bin (ties by unit index), the
least-loaded assignment for dK/dV and the snake deal for dQ."""
import numpy as np

BN = 128
BINS = 4096
MAX_GRID = 1024


def _cdiv(a, b):
    return (a + b - 1) // b


def unit_of(kdkdv, u, B, Hq, Hkv, nT):
    if kdkdv:
        per = B * Hkv
        return (u % per) // Hkv, (u % per) % Hkv, u // per
    per = B * Hq
    return (u % per) // Hq, (u % per) % Hq, nT - 1 - u // per


def unit_cost(kdkdv, u, mask, B, Hq, Hkv, N, S, W):
    """Steps of unit u plus one (its fixed work)."""
    nT = _cdiv(N, BN)
    b, hx, tile = unit_of(kdkdv, u, B, Hq, Hkv, nT)
    if kdkdv:
        G = Hq // Hkv
        c = 1
        for g in range(G):
            sa = bool(mask[b][hx * G + g])
            if not sa or tile * BN < S:
                last = nT - 1
            else:
                last = min(nT - 1, (tile * BN + BN - 1 + W - 1) // BN)
            c += last - tile + 1
        return c
    if not bool(mask[b][hx]):
        return 1 + tile + 1
    lo = max(0, tile * BN - W + 1) // BN
    a = min(_cdiv(S, BN), lo)
    return 1 + a + (tile - lo + 1)


def schedule(kdkdv, mask, B, Hq, Hkv, N, S, W, grid):
    """(offs [grid + 1], list [units]) exactly as the device builds them."""
    nT = _cdiv(N, BN)
    units = B * (Hkv if kdkdv else Hq) * nT
    max_cost = 1 + (Hq // Hkv if kdkdv else 1) * nT
    shift = 0
    while (max_cost >> shift) >= BINS:
        shift += 1
    cost = np.array([unit_cost(kdkdv, u, mask, B, Hq, Hkv, N, S, W) for u in range(units)])
    order = sorted(range(units), key=lambda u: (-(cost[u] >> shift), u))
    cta = np.zeros(units, dtype=np.int64)
    if kdkdv:
        load = np.zeros(grid, dtype=np.int64)
        for r, u in enumerate(order):
            i = int(np.argmin(load))          # first index of the minimum
            cta[r] = i
            load[i] += cost[u]
    else:
        for r in range(units):
            k, c = divmod(r, grid)
            cta[r] = grid - 1 - c if k & 1 else c
    offs = np.zeros(grid + 1, dtype=np.int64)
    for i in range(grid):
        offs[i + 1] = offs[i] + int(np.sum(cta == i))
    lists = [[] for _ in range(grid)]
    for r, u in enumerate(order):
        lists[cta[r]].append(u)
    flat = [u for lst in lists for u in lst]
    return offs, np.array(flat, dtype=np.int64), cost


def per_cta_load(offs, lst, cost):
    return np.array([cost[lst[offs[i]:offs[i + 1]]].sum() for i in range(len(offs) - 1)])
