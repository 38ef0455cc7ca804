"""Host logic of the fused kernel's schedule (no GPU): every selected
(b, h, query row) is covered by exactly one unit slot, every tile a slot
needs is visited with the right masking code, units are ordered longest
first, and the snake deal gives each rank to exactly one CTA."""
import numpy as np
import pytest

import oracle
from sparse_attention_head_b200 import flops
from sparse_attention_head_b200.api import (ea_schedule_unit_tiles, ea_schedule_units,
                                            make_params)


def brute_codes(N, sparse, S, W, r0, tile):
    """0/1/2 code of (128-row slot at r0, 128-key tile) from the definition."""
    rows = [i for i in range(r0, r0 + 128)]
    keys = range(tile * 128, tile * 128 + 128)
    any_vis = False
    all_vis = True
    for i in rows:
        for j in keys:
            v = oracle.visible(i, j, sparse, S, W)
            if i < N and v:
                any_vis = True
            if not v:
                all_vis = False
    if not any_vis:
        return 0
    return 1 if all_vis else 2


CASES = [
    # B, Hq, Hkv, N, d, S, W, select
    (1, 4, 2, 512, 64, 16, 128, 0),
    (1, 4, 2, 300, 64, 0, 1, 0),
    (2, 4, 1, 700, 128, 130, 200, 0),
    (1, 2, 2, 1, 64, 5, 3, 0),
    (1, 4, 4, 1000, 128, 64, 1024, 0),
    (1, 4, 2, 640, 64, 1, 129, 1),
    (1, 4, 2, 640, 64, 1, 129, 2),
    (2, 6, 3, 257, 64, 300, 5, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W,sel", CASES)
def test_units_cover_rows_once(B, Hq, Hkv, N, d, S, W, sel):
    rng = np.random.default_rng(N + S + W + sel)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    p = make_params(B, Hq, Hkv, N, d, S, W, select=sel)
    units = ea_schedule_units(mask, p)
    covered = np.zeros((B, Hq, N), dtype=np.int32)
    for sparse, b, h, pair, ntiles in units:
        assert sparse == mask[b, h]
        assert sel == 0 or (sel == 1 and not sparse) or (sel == 2 and sparse)
        r0 = 256 * pair
        covered[b, h, r0:min(N, r0 + 256)] += 1
    for b in range(B):
        for h in range(Hq):
            selected = sel == 0 or (sel == 1) == (mask[b, h] == 0)
            want = 1 if selected else 0
            assert np.all(covered[b, h] == want)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W,sel", CASES)
def test_unit_tiles_match_definition(B, Hq, Hkv, N, d, S, W, sel):
    rng = np.random.default_rng(7 * N + S)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    p = make_params(B, Hq, Hkv, N, d, S, W, select=sel)
    units = ea_schedule_units(mask, p)
    ntiles_total = (N + 127) // 128
    seen_kinds = set()
    for rank, (sparse, b, h, pair, n) in enumerate(units):
        key = (sparse, pair)
        if key in seen_kinds:
            continue
        seen_kinds.add(key)
        tiles, codes = ea_schedule_unit_tiles(mask, p, rank)
        assert len(tiles) == n
        assert len(set(tiles.tolist())) == n and list(tiles) == sorted(tiles)
        r0 = 256 * pair
        for slot in range(2):
            rs = r0 + 128 * slot
            for t in range(ntiles_total):
                want = brute_codes(N, bool(sparse), S, W, rs, t) if rs < N else 0
                if t in tiles:
                    got = codes[list(tiles).index(t), slot]
                    assert got == want, (rank, slot, t)
                else:
                    assert want == 0, (rank, slot, t)
        # every listed tile is needed by some slot
        assert np.all(codes.max(axis=1) > 0)


def test_order_longest_first_and_snake_deal():
    B, Hq, Hkv, N, d, S, W = 1, 32, 8, 32768, 128, 64, 1024
    mask = np.zeros((B, Hq), np.uint8)
    mask[0, [1, 2, 5, 7, 9, 11, 12, 13, 15, 17, 18, 19, 20, 22, 23, 24, 25, 26, 28, 29, 30, 31]] = 1
    p = make_params(B, Hq, Hkv, N, d, S, W)
    units = ea_schedule_units(mask, p)
    cost = units[:, 4]
    sa_cap = max(cost[units[:, 0] == 1])
    nfa = int((mask == 0).sum())
    # long FA units first, strictly non-increasing
    long_fa = units[: nfa * (128 - sa_cap // 2)]
    assert np.all(long_fa[:, 0] == 0)
    assert np.all(np.diff(long_fa[:, 4]) <= 0)
    assert np.all(long_fa[:, 4] > sa_cap)
    # then SA units, then the short FA units
    rest = units[len(long_fa):]
    assert np.all(rest[: 22 * 128, 0] == 1)
    assert np.all(rest[22 * 128:, 0] == 0)
    assert np.all(rest[22 * 128:, 4] <= sa_cap)
    # snake deal: each rank exactly once, loads within one longest unit
    G = 148
    total = len(units)
    owner = -np.ones(total, dtype=np.int64)
    load = np.zeros(G, dtype=np.int64)
    for c in range(G):
        k = 0
        while True:
            r = k * G + ((G - 1 - c) if (k & 1) else c)
            if r >= total:
                break
            assert owner[r] == -1
            owner[r] = c
            load[c] += cost[r]
            k += 1
    assert np.all(owner >= 0)
    assert load.max() - load.min() <= cost.max()


@pytest.mark.parametrize("N,S,W", [(1, 0, 1), (77, 3, 5), (512, 16, 128), (300, 400, 2)])
def test_pair_counts_match_oracle(N, S, W):
    for sparse in (False, True):
        assert flops.attn_visible_pairs(N, sparse, S, W) == \
            oracle.count_visible_pairs(N, sparse, S, W)


def test_effective_and_tile_flops():
    mask = np.array([[0, 1, 0, 1]], np.uint8)
    eff = flops.effective_flops(mask, 512, 64, 16, 128)
    pairs = 2 * oracle.count_visible_pairs(512, False, 16, 128) + \
        2 * oracle.count_visible_pairs(512, True, 16, 128)
    assert eff == 4 * 64 * pairs
    # tile-granular: FA 512 rows -> 1+2+3+4 tiles; SA (S=16, W=128): tiles per
    # row tile m are {0, m-1, m} -> 1, 2, 3, 3
    assert flops.tile_flops(mask, 512, 64, 16, 128) == 4 * 64 * 128 * 128 * (2 * 10 + 2 * 9)


@pytest.mark.parametrize("t,S,W", [(0, 4, 16), (5, 4, 16), (19, 4, 16), (20, 4, 16),
                                   (1000, 64, 256), (7, 0, 1), (300, 500, 8)])
def test_decode_group_rows_match_oracle(t, S, W):
    assert flops.decode_group_rows(t, False, S, W) == len(oracle.visible_keys(t, False, S, W))
    assert flops.decode_group_rows(t, True, S, W) == len(oracle.visible_keys(t, True, S, W))


def test_decode_bytes():
    mask = np.array([[1, 1, 0, 1], [1, 1, 1, 1]], np.uint8)
    pos = [100, 9]
    got = flops.decode_bytes(mask, pos, 2, 64, 2, 8)
    row = 128
    # b0: group 0 all SA (2 + 8 rows), group 1 mixed (101 rows); b1: both SA (2 + 8)
    assert got["kv"] == 2 * row * (10 + 101 + 10 + 10)
    assert got["io"] == 2 * 2 * 4 * row + 4 * 2 * 2 * row
    assert got["n_sa_groups"] == 3 and got["n_groups"] == 4


# ---------------------------------------------------------------- packed batches
from sparse_attention_head_b200.api import ea_schedule_units_varlen, make_varlen_params  # noqa: E402

VARLEN_CASES = [
    # cu_seqlens, Hq, Hkv, d, S, W, select
    ([0, 300, 300, 1000, 1077, 1600], 4, 2, 64, 16, 128, 0),
    ([0, 1, 2, 515, 4611], 4, 1, 128, 64, 1024, 0),
    ([0, 256, 512, 768], 2, 2, 64, 0, 1, 0),
    ([0, 700, 900, 2000], 4, 2, 128, 130, 200, 1),
    ([0, 700, 900, 2000], 4, 2, 128, 130, 200, 2),
    ([0, 0, 0, 129], 2, 1, 64, 5, 3, 0),
]


def _units_cover(units, cu, mask, sel):
    B, Hq = mask.shape
    lens = np.diff(cu)
    covered = [np.zeros((Hq, n), np.int32) for n in lens]
    for sparse, b, h, pair, ntiles in units:
        assert sparse == mask[b, h]
        assert sel == 0 or (sel == 1 and not sparse) or (sel == 2 and sparse)
        r0 = 256 * pair
        assert r0 < lens[b]
        covered[b][h, r0:min(lens[b], r0 + 256)] += 1
    for b in range(B):
        for h in range(Hq):
            selected = sel == 0 or (sel == 1) == (mask[b, h] == 0)
            assert np.all(covered[b][h] == (1 if selected else 0)), (b, h)


@pytest.mark.parametrize("cu,Hq,Hkv,d,S,W,sel", VARLEN_CASES)
def test_varlen_units_cover_rows_once(cu, Hq, Hkv, d, S, W, sel):
    B = len(cu) - 1
    rng = np.random.default_rng(cu[-1] + S)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    p = make_varlen_params(B, Hq, Hkv, cu[-1], max(np.diff(cu)), d, S, W, select=sel)
    units = ea_schedule_units_varlen(mask, p, cu)
    _units_cover(units, cu, mask, sel)
    # each unit's tile count is that of its own sequence's shape
    for sparse, b, h, pair, n in units:
        N_b = cu[b + 1] - cu[b]
        tiles = [t for t in range((N_b + 127) // 128)
                 if any(brute_codes(N_b, bool(sparse), S, W, 256 * pair + 128 * s, t)
                        for s in range(2) if 256 * pair + 128 * s < N_b)]
        assert n == len(tiles), (b, pair, n, tiles)


def test_varlen_equal_lengths_schedule_like_the_padded_batch():
    B, Hq, Hkv, N, d, S, W = 3, 4, 2, 1000, 128, 64, 256
    rng = np.random.default_rng(5)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    padded = ea_schedule_units(mask, make_params(B, Hq, Hkv, N, d, S, W))
    packed = ea_schedule_units_varlen(mask, make_varlen_params(B, Hq, Hkv, B * N, N, d, S, W),
                                      [0, N, 2 * N, 3 * N])
    np.testing.assert_array_equal(padded, packed)


def test_varlen_order_longest_first_and_balance():
    cu = np.cumsum([0, 32768, 1000, 9000, 300, 20000, 0, 4096]).tolist()
    B, Hq, Hkv, d, S, W = len(cu) - 1, 32, 8, 128, 64, 1024
    rng = np.random.default_rng(11)
    mask = (rng.random((B, Hq)) < 0.7).astype(np.uint8)
    p = make_varlen_params(B, Hq, Hkv, cu[-1], max(np.diff(cu)), d, S, W)
    units = ea_schedule_units_varlen(mask, p, cu)
    _units_cover(units, cu, mask, 0)
    cost = units[:, 4]
    sa_cap = int(np.ceil(S / 128)) + 2 + int(np.ceil((W - 1) / 128))
    pA = sa_cap // 2
    # long FA units first by pair, descending; then every SA unit; then short FA
    nlong = int(np.sum((units[:, 0] == 0) & (units[:, 3] >= pA)))
    assert np.all(units[:nlong, 0] == 0) and np.all(np.diff(units[:nlong, 3]) <= 0)
    nsa = int(np.sum(units[:, 0] == 1))
    assert np.all(units[nlong:nlong + nsa, 0] == 1)
    assert np.all(units[nlong + nsa:, 0] == 0) and np.all(units[nlong + nsa:, 3] < pA)
    # snake deal over 148 CTAs: loads within one longest unit
    G = 148
    load = np.zeros(G, np.int64)
    for r in range(len(units)):
        k = r // G
        c = (r % G) if k % 2 == 0 else G - 1 - (r % G)
        load[c] += cost[r]
    assert load.max() - load.min() <= cost.max()


def test_varlen_schedule_rejects_inconsistent_offsets():
    mask = np.zeros((2, 2), np.uint8)
    p = make_varlen_params(2, 2, 1, 10, 10, 64, 1, 4)
    with pytest.raises(ValueError):
        ea_schedule_units_varlen(mask, p, [1, 5, 10])
    with pytest.raises(ValueError):
        ea_schedule_units_varlen(mask, p, [0, 6, 4])
    with pytest.raises(ValueError):
        ea_schedule_units_varlen(mask, p, [0, 5, 9])


def test_backward_schedule_mirror_balances():
    """The backward kernels' unit lists (host mirror of the device schedule):
    every unit exactly once, each CTA's units longest first, and the busiest
    CTA within 2% of the mean load on a llama8b-shaped layer with mixed
    modes, where ordering units by tile index alone leaves it 41% above."""
    import numpy as np
    import bwd_sched_mirror as m
    rng = np.random.default_rng(1)
    B, Hq, Hkv, N, S, W = 1, 32, 8, 32768, 64, 1024
    mask = (rng.random((B, Hq)) < 0.44).astype(np.uint8)
    for kdkdv in (True, False):
        offs, lst, cost = m.schedule(kdkdv, mask, B, Hq, Hkv, N, S, W, 148)
        assert sorted(lst.tolist()) == list(range(len(cost)))
        for i in range(148):
            c = cost[lst[offs[i]:offs[i + 1]]]
            assert np.all(c[:-1] >= c[1:])
        load = m.per_cta_load(offs, lst, cost)
        assert load.max() / load.mean() < 1.02, (kdkdv, load.max() / load.mean())
