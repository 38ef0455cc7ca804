"""GPU parity of the head-sharded path's entry points, with the ranks
emulated one after another on one GPU (no kernel waits on another):
- each rank's ea_router_pool_rows slice, laid side by side as the
  all-gather lays them, then ea_router_mlp, gives ea_router_decide's mask
  and logits bit for bit;
- each rank's ea_hybrid_attn_prefill_groups launch on its LPT-assigned
  groups, and each rank's ea_hybrid_attn_prefill_heads launch on its heads
  under the split assignment (a group costlier than a rank's share split by
  query head), writes exactly its heads' rows, with the bits of the
  unsharded fused launch, and leaves every other row untouched."""
import numpy as np
import pytest
import torch

from sparse_attention_head_b200 import build, shard
from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
                                            ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_groups,
                                            ea_hybrid_attn_prefill_heads, ea_router_decide,
                                            ea_router_mlp, ea_router_mlp_workspace_size,
                                            ea_router_pool_rows, ea_router_workspace_size,
                                            make_params)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _layer(B, Hq, Hkv, N, d, hidden, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = (torch.randn((B, Hkv, N, d), generator=g) +
         torch.randn((1, Hkv, 1, d), generator=g)).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.05
    b1 = torch.randn((hidden,), generator=g) * 0.05
    w2 = torch.randn((Hq, hidden), generator=g) * 0.2
    b2 = torch.randn((Hq,), generator=g) * 0.1
    return [t.to(DEV) for t in (q, k, v, w1, b1, w2, b2)]


CASES = [
    # B, Hq, Hkv, N, d, S, W
    (1, 32, 8, 4096, 128, 64, 1024),
    (2, 16, 4, 1000, 64, 16, 128),
    (3, 8, 2, 777, 128, 4, 300),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W", CASES)
@pytest.mark.parametrize("world", [2, 3, 8])
def test_sharded_router_and_attention_equal_the_single_launch(B, Hq, Hkv, N, d, S, W, world):
    q, k, v, w1, b1, w2, b2 = _layer(B, Hq, Hkv, N, d, 64, seed=B * 100 + N)
    mask_ref, z_ref = ea_router_decide(k, w1, b1, w2, b2)
    ws_ref = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
    out_ref = ea_hybrid_attn_prefill(q, k, v, mask_ref, S, W, workspace=ws_ref)

    # steps 1-2: every rank's pooled slice, side by side as the all-gather
    # lays them
    chunk = shard.pool_chunk(B, Hkv, world)
    pool_ws = torch.empty(ea_router_workspace_size(B, Hkv, N, d), dtype=torch.uint8, device=DEV)
    gathered = torch.full((world, chunk * d), float("nan"), dtype=torch.float32, device=DEV)
    for r in range(world):
        row0, nrows = shard.pool_rows(B, Hkv, world, r)
        ea_router_pool_rows(k, row0, nrows, x_out=gathered[r], workspace=pool_ws)
    x = gathered.reshape(-1)[:B * Hkv * d].view(B, Hkv * d)
    # step 3: the MLP on the gathered vector
    mask = torch.empty((B, Hq), dtype=torch.uint8, device=DEV)
    z = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    mlp_ws = torch.empty(ea_router_mlp_workspace_size(B, 64), dtype=torch.uint8, device=DEV)
    ea_router_mlp(x, w1, b1, w2, b2, route_mask=mask, logits=z, workspace=mlp_ws)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask_ref)
    assert torch.equal(z.view(torch.int32), z_ref.view(torch.int32))
    m = mask.cpu().numpy()
    assert 0 < int(m.sum()) < m.size

    # step 4: every rank's groups
    owner = shard.lpt_assign(shard.group_costs(m, Hkv, N, S, W), world)
    G = Hq // Hkv
    covered = torch.zeros((B, Hq), dtype=torch.bool)
    for r in range(world):
        sel = torch.as_tensor(shard.group_select(owner, r), device=DEV)
        out = torch.full_like(q, 7.0)
        ws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
        ea_hybrid_attn_prefill_groups(q, k, v, mask, sel, S, W, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert ea_get_device_status(ws) == 0
        mine = torch.zeros((B, Hq), dtype=torch.bool)
        for b, h in shard.head_rows_of(owner, r, G):
            mine[b, h] = True
        covered |= mine
        own = mine.to(DEV)
        assert torch.equal(out[own].view(torch.int16), out_ref[own].view(torch.int16)), r
        assert bool((out[~own] == 7.0).all()), r
    assert bool(covered.all())

    # step 4, split assignment: every rank's query heads
    owner_h = shard.lpt_assign_split(m, Hkv, N, S, W, world)
    covered = torch.zeros((B, Hq), dtype=torch.bool)
    for r in range(world):
        sel = torch.as_tensor((owner_h == r).astype(np.uint8), device=DEV)
        out = torch.full_like(q, 7.0)
        ws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
        ea_hybrid_attn_prefill_heads(q, k, v, mask, sel, S, W, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert ea_get_device_status(ws) == 0
        own = torch.as_tensor(owner_h == r)
        assert not bool((covered & own).any())
        covered |= own
        own = own.to(DEV)
        assert torch.equal(out[own].view(torch.int16), out_ref[own].view(torch.int16)), r
        assert bool((out[~own] == 7.0).all()), r
    assert bool(covered.all())
    assert ea_get_device_status(ws_ref) == 0


@pytest.mark.parametrize("split", [True, False])
def test_sharded_prefill_class_one_rank(split):
    """ShardedPrefill on one rank (no exchange: the gathered vector is the
    rank's own slice): route, assign and attend give the unsharded launch's
    mask and output bits, and host_step moves every head up and down."""
    B, Hq, Hkv, N, d, S, W = 2, 16, 4, 700, 128, 16, 128
    q, k, v, w1, b1, w2, b2 = _layer(B, Hq, Hkv, N, d, 64, seed=77)
    mask_ref, _ = ea_router_decide(k, w1, b1, w2, b2)
    out_ref = ea_hybrid_attn_prefill(q, k, v, mask_ref, S, W)
    sp = shard.ShardedPrefill(B, Hq, Hkv, N, d, w1, b1, w2, b2, S, W, 0, 1, DEV,
                              split_groups=split)
    out = torch.full_like(q, 7.0)
    sp(q, k, v, out)
    torch.cuda.synchronize()
    assert ea_get_device_status(sp.attn_ws) == 0
    assert torch.equal(sp.mask, mask_ref)
    assert np.all(sp.owner == 0)
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    # from pinned host buffers
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    qd, kd, vd, od = (torch.empty_like(t) for t in (q, k, v, q))
    up, down = sp.host_step(qh, kh, vh, oh, qd, kd, vd, od)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), out_ref.cpu().view(torch.int16))
    assert up == (q.numel() + k.numel() + v.numel()) * 2 and down == q.numel() * 2
