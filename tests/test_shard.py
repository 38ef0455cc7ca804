"""The head-sharded multi-GPU path's host logic, on the CPU.

- Pooling ownership: every (b, kv head) row pooled by exactly one rank, in
  contiguous equal chunks.
- Group costs: the score tiles of each group's heads, against a count made
  tile by tile from the visibility definition.
- LPT assignment: a partition, deterministic, and within the LPT bound; the
  split assignment splits exactly the groups costlier than a rank's share,
  keeps the others whole, and balances the bench's 8-group layer on 8 ranks.
- World-size 2 and 3 gloo ranks: each rank pools only its own rows (the
  oracle's pooling stands in for the pooling kernel), the package's
  all-gather assembles the pooled vector, and the router MLP on it gives
  every rank the single-rank oracle's x and mask bit for bit; every rank
  computes the same assignment, and the ranks' head sets cover every head
  exactly once."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_attention_head_b200 import shard


@pytest.mark.parametrize("B,Hkv,world", [(1, 8, 1), (1, 8, 2), (1, 8, 3), (2, 8, 4), (3, 2, 4),
                                         (1, 2, 8), (4, 8, 8)])
def test_pool_rows_partition(B, Hkv, world):
    seen = []
    chunk = shard.pool_chunk(B, Hkv, world)
    for r in range(world):
        row0, n = shard.pool_rows(B, Hkv, world, r)
        assert 0 <= n <= chunk
        if n:
            assert row0 == r * chunk
        seen.extend(range(row0, row0 + n))
    assert seen == list(range(B * Hkv))


def _tiles_by_definition(N, sparse, S, W, bm=128):
    """Tiles of one head holding at least one visible pair, by enumeration."""
    nt = -(-N // bm)
    count = 0
    for m in range(nt):
        rows = range(m * bm, min(N, (m + 1) * bm))
        for t in range(m + 1):
            cols = range(t * bm, min(N, (t + 1) * bm))
            if any(oracle.visible(i, j, sparse, S, W) for i in rows for j in cols):
                count += 1
    return count


@pytest.mark.parametrize("N,S,W", [(300, 4, 100), (1000, 0, 1), (513, 130, 257)])
def test_group_costs_count_visible_tiles(N, S, W):
    rng = np.random.default_rng(N)
    B, Hq, Hkv = 2, 8, 2
    mask = (rng.random((B, Hq)) < 0.5).astype(np.uint8)
    costs = shard.group_costs(mask, Hkv, N, S, W)
    t_fa, t_sa = _tiles_by_definition(N, False, S, W), _tiles_by_definition(N, True, S, W)
    for b in range(B):
        for hk in range(Hkv):
            heads = mask[b, hk * 4:(hk + 1) * 4]
            assert costs[b, hk] == sum(t_sa if x else t_fa for x in heads)


def test_lpt_assignment_partition_and_bound():
    rng = np.random.default_rng(9)
    for world in (1, 2, 3, 4, 8):
        for _ in range(20):
            costs = rng.integers(1, 1000, size=(int(rng.integers(1, 5)), 8))
            owner = shard.lpt_assign(costs, world)
            assert owner.shape == costs.shape
            assert set(np.unique(owner)) <= set(range(world))
            # deterministic: the same costs give the same owners
            assert np.array_equal(owner, shard.lpt_assign(costs.copy(), world))
            loads = shard.rank_loads(costs, owner, world)
            assert sum(loads) == int(costs.sum())
            # greedy list scheduling bound: max load <= mean load + largest item
            assert max(loads) <= costs.sum() / world + costs.max()
    # a hand-worked case, costs 7, 5, 4, 3, 1 on two ranks: 7 -> r0; 5 -> r1;
    # 4 -> r1 (load 5 < 7); 3 -> r0 (7 < 9); 1 -> r1 (9 < 10)
    owner = shard.lpt_assign(np.array([[7, 5, 4, 3, 1]]), 2)
    assert owner.tolist() == [[0, 1, 1, 0, 1]]


@pytest.mark.parametrize("N,S,W", [(300, 4, 100), (1000, 0, 1)])
def test_head_costs_count_visible_tiles(N, S, W):
    rng = np.random.default_rng(N + 1)
    mask = (rng.random((2, 8)) < 0.5).astype(np.uint8)
    hc = shard.head_costs(mask, N, S, W)
    t_fa, t_sa = _tiles_by_definition(N, False, S, W), _tiles_by_definition(N, True, S, W)
    np.testing.assert_array_equal(hc, np.where(mask != 0, t_sa, t_fa))
    np.testing.assert_array_equal(hc.reshape(2, 2, 4).sum(axis=2), shard.group_costs(mask, 2, N, S, W))


def test_split_assignment_splits_only_heavy_groups():
    rng = np.random.default_rng(3)
    N, S, W = 8192, 64, 512
    for world in (1, 2, 3, 4, 8):
        for _ in range(10):
            B, Hkv, G = int(rng.integers(1, 4)), int(rng.choice([2, 4, 8])), int(rng.choice([1, 2, 4]))
            Hq = Hkv * G
            mask = (rng.random((B, Hq)) < 0.6).astype(np.uint8)
            owner = shard.lpt_assign_split(mask, Hkv, N, S, W, world)
            assert owner.shape == (B, Hq) and set(np.unique(owner)) <= set(range(world))
            np.testing.assert_array_equal(owner, shard.lpt_assign_split(mask.copy(), Hkv, N, S, W,
                                                                        world))
            gc = shard.group_costs(mask, Hkv, N, S, W)
            share = gc.sum() / world
            g_owner = owner.reshape(B, Hkv, G)
            for b in range(B):
                for hk in range(Hkv):
                    whole = len(set(g_owner[b, hk].tolist())) == 1
                    if gc[b, hk] <= share or world == 1 or G == 1:
                        assert whole, (world, b, hk)
            hc = shard.head_costs(mask, N, S, W)
            loads = shard.rank_loads(hc, owner, world)
            assert sum(loads) == int(hc.sum())
            # LPT bound over the items: mean load + the largest item
            assert max(loads) <= hc.sum() / world + max(int(hc.max()), int(gc[gc <= share].max())
                                                          if np.any(gc <= share) else 0)


def test_split_assignment_balances_eight_groups_on_eight_ranks():
    # the bench's 256K layer shape: FA heads per kv group 2 1 2 0 1 1 0 1
    fa = [2, 1, 2, 0, 1, 1, 0, 1]
    mask = np.ones((1, 32), np.uint8)
    for g, n in enumerate(fa):
        mask[0, 4 * g:4 * g + n] = 0
    N, S, W = 262144, 128, 4096
    whole = shard.lpt_assign(shard.group_costs(mask, 8, N, S, W), 8)
    hc = shard.head_costs(mask, N, S, W)
    loads_whole = shard.rank_loads(shard.group_costs(mask, 8, N, S, W), whole, 8)
    split = shard.lpt_assign_split(mask, 8, N, S, W, 8)
    loads_split = shard.rank_loads(hc, split, 8)
    mean = hc.sum() / 8
    assert mean / max(loads_whole) < 0.6
    assert mean / max(loads_split) > 0.95
    # each rank runs one full-attention head
    for r in range(8):
        assert sum(1 for h in range(32) if split[0, h] == r and mask[0, h] == 0) == 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(21)
    B, Hkv, N, d, hidden, Hq = 2, 4, 96, 16, 24, 16
    k = (torch.randn((B, Hkv, N, d), generator=g) +
         torch.randn((1, Hkv, 1, d), generator=g)).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.1
    b1 = torch.randn((hidden,), generator=g) * 0.1
    w2 = torch.randn((Hq, hidden), generator=g) * 0.3
    b2 = torch.randn((Hq,), generator=g) * 0.1
    return k.float().double().numpy(), w1.double().numpy(), b1.double().numpy(), \
        w2.double().numpy(), b2.double().numpy()


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        k, w1, b1, w2, b2 = _inputs()
        B, Hkv, N, d = k.shape
        Hq = w2.shape[0]
        row0, nrows = shard.pool_rows(B, Hkv, world, rank)
        chunk = shard.pool_chunk(B, Hkv, world)
        # this rank pools only its own rows of K (the oracle's pooling)
        x_local = np.zeros((chunk, d))
        if nrows:
            rows = k.reshape(B * Hkv, N, d)[row0:row0 + nrows]
            x_local[:nrows] = oracle.router_pool(rows[None]).reshape(nrows, d)
        x = shard.gather_pooled(torch.as_tensor(x_local.reshape(-1)), B, Hkv, d, world)
        z = oracle.router_mlp(x.numpy(), w1, b1, w2, b2)
        mask = (z > 0.0).astype(np.uint8)
        owner = shard.lpt_assign_split(mask, Hkv, N, 8, 20, world)
        heads = shard.heads_of(owner, rank)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), x=x.numpy(), z=z, mask=mask,
                 owner=owner, heads=np.array(heads, dtype=np.int64).reshape(-1, 2))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_reproduce_single_rank_router_and_cover_every_head(world, tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    k, w1, b1, w2, b2 = _inputs()
    B, Hkv, N, d = k.shape
    Hq = w2.shape[0]
    mask_ref, z_ref = oracle.router_decide(k, w1, b1, w2, b2)
    x_ref = oracle.router_pool(k)
    assert 0 < int(mask_ref.sum()) < mask_ref.size
    res = [np.load(os.path.join(tmp_path, f"rank{r}.npz")) for r in range(world)]
    for r in res:
        # bit for bit: the gathered pooled vector, the logits and the mask
        assert np.array_equal(r["x"].view(np.uint64), x_ref.view(np.uint64))
        assert np.array_equal(r["z"].view(np.uint64), z_ref.view(np.uint64))
        assert np.array_equal(r["mask"], mask_ref)
        assert np.array_equal(r["owner"], res[0]["owner"])
    heads = sorted(tuple(h) for r in res for h in r["heads"])
    assert heads == [(b, h) for b in range(B) for h in range(Hq)]
