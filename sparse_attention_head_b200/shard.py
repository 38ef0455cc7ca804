"""Head-sharded prefill over several GPUs (one process per GPU).

The prefill splits into independent (batch, kv group) problems: a kv group
is one kv head with the G query heads that read it.  The work is therefore
sharded over (b, kv head) pairs, and the output stays head-sharded (each
rank writes the rows of its own heads).  The one exchange is the router's:
its pooled input is the mean of the keys of EVERY kv head of a batch row
(Elastic Attention blog §2.1: the router reads the layer's Key hidden
states), so each rank pools a static share of the (b, kv head) rows and one
all-gather of those fp32 slices (B * Hkv * d values) gives every rank the
same pooled vector, hence the same mask.  The mask then fixes each group's
cost, and the groups are assigned to ranks by longest-processing-time
(largest cost first, to the least-loaded rank): deterministic, so every rank
computes the same assignment without another exchange.  A group that costs
more than a rank's share (total / ranks) is split into its query heads, each
assigned on its own; the ranks holding its heads each read the group's K/V.
With few groups per rank (8 kv groups over 8 ranks) whole groups cannot
balance: one with two or three full-attention heads sets the time.

Host logic only (ownership, costs, assignment) plus the per-layer step that
strings the C ABI calls together with torch.distributed; every step of the
computation runs in libea.so's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

from .flops import _visible_tiles


def pool_chunk(B: int, Hkv: int, world: int) -> int:
    """Rows of the flattened (b, kv head) index each rank pools (the last
    rank's share may be shorter)."""
    return -(-B * Hkv // world)


def pool_rows(B: int, Hkv: int, world: int, rank: int) -> Tuple[int, int]:
    """(row0, nrows): the rank's contiguous rows r = b * Hkv + hk of the
    pooling.  Contiguous equal chunks, so an all-gather of [chunk, d] slices
    lays the pooled vector out in [B][Hkv][d] order without any permute."""
    chunk = pool_chunk(B, Hkv, world)
    row0 = min(rank * chunk, B * Hkv)
    return row0, max(0, min(B * Hkv, row0 + chunk) - row0)


def group_costs(mask, Hkv: int, N: int, sink: int, window: int) -> np.ndarray:
    """[B, Hkv] int64: the 128 x 128 score tiles the group's query heads run
    (what the fused kernel's time is proportional to), from the route mask
    [B, Hq] (nonzero = SA)."""
    m = np.asarray(mask).reshape(np.asarray(mask).shape[0], -1)
    B, Hq = m.shape
    G = Hq // Hkv
    t_fa = _visible_tiles(N, False, sink, window)
    t_sa = _visible_tiles(N, True, sink, window)
    n_sa = (m.reshape(B, Hkv, G) != 0).sum(axis=2)
    return (n_sa * t_sa + (G - n_sa) * t_fa).astype(np.int64)


def head_costs(mask, N: int, sink: int, window: int) -> np.ndarray:
    """[B, Hq] int64: the score tiles each query head runs under the mask."""
    m = np.asarray(mask)
    m = m.reshape(m.shape[0], -1)
    t_fa = _visible_tiles(N, False, sink, window)
    t_sa = _visible_tiles(N, True, sink, window)
    return np.where(m != 0, t_sa, t_fa).astype(np.int64)


def lpt_assign_split(mask, Hkv: int, N: int, sink: int, window: int, world: int) -> np.ndarray:
    """owner [B, Hq] by query head.  The items are the (b, kv group) groups,
    except that a group costing more than total / world becomes one item per
    query head; then longest processing time first over the items (ties:
    lower first head index first; least-loaded rank, ties to the lower
    rank).  Depends only on the mask, so every rank computes the same one."""
    hc = head_costs(mask, N, sink, window)
    B, Hq = hc.shape
    G = Hq // Hkv
    gc = hc.reshape(B, Hkv, G).sum(axis=2)
    share = gc.sum() / max(world, 1)
    items = []          # (cost, first head flat index, heads as flat indices)
    for b in range(B):
        for hk in range(Hkv):
            heads = [b * Hq + hk * G + j for j in range(G)]
            if world > 1 and G > 1 and gc[b, hk] > share:
                items.extend((int(hc.reshape(-1)[i]), i, [i]) for i in heads)
            else:
                items.append((int(gc[b, hk]), heads[0], heads))
    items.sort(key=lambda it: (-it[0], it[1]))
    load = [0] * world
    owner = np.empty(B * Hq, dtype=np.int64)
    for cost, _, heads in items:
        r = min(range(world), key=lambda x: (load[x], x))
        owner[heads] = r
        load[r] += cost
    return owner.reshape(B, Hq)


def lpt_assign(costs, world: int) -> np.ndarray:
    """owner [B, Hkv]: longest processing time first.  Groups are taken in
    order of decreasing cost (ties: lower flattened index first) and each
    goes to the rank with the least load so far (ties: the lower rank).  The
    result depends only on the costs, so every rank computes the same one."""
    c = np.asarray(costs, dtype=np.int64)
    flat = c.reshape(-1)
    order = sorted(range(flat.size), key=lambda i: (-int(flat[i]), i))
    load = [0] * world
    owner = np.empty(flat.size, dtype=np.int64)
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        owner[i] = r
        load[r] += int(flat[i])
    return owner.reshape(c.shape)


def heads_of(owner_h, rank: int) -> Sequence[Tuple[int, int]]:
    """(b, h) query heads a per-head assignment gives `rank`."""
    o = np.asarray(owner_h)
    return [(b, h) for b in range(o.shape[0]) for h in range(o.shape[1]) if o[b, h] == rank]


def group_select(owner, rank: int) -> np.ndarray:
    """uint8 [B, Hkv]: 1 where the group belongs to `rank`."""
    return (np.asarray(owner) == rank).astype(np.uint8)


def rank_loads(costs, owner, world: int) -> List[int]:
    c = np.asarray(costs, dtype=np.int64).reshape(-1)
    o = np.asarray(owner).reshape(-1)
    return [int(c[o == r].sum()) for r in range(world)]


def gather_pooled(x_local: torch.Tensor, B: int, Hkv: int, d: int, world: int,
                  group=None) -> torch.Tensor:
    """All-gather every rank's pooled slice ([chunk * d] fp32, rows past its
    share ignored) into x [B, Hkv * d].  With one rank it returns the slice."""
    chunk = pool_chunk(B, Hkv, world)
    if x_local.numel() != chunk * d:
        raise ValueError("x_local must hold pool_chunk(B, Hkv, world) * d values")
    if world == 1:
        return x_local[:B * Hkv * d].view(B, Hkv * d)
    full = torch.empty(world * chunk * d, dtype=x_local.dtype, device=x_local.device)
    torch.distributed.all_gather_into_tensor(full, x_local.reshape(-1), group=group)
    return full[:B * Hkv * d].view(B, Hkv * d)


class ShardedPrefill:
    """One layer's sharded prefill on this rank: router pooling of the rank's
    rows, the all-gather of the pooled slices, the router MLP, the
    assignment (by group, a group costlier than a rank's share split by
    query head; split_groups=False keeps whole groups), and the fused
    attention on the rank's query heads.

    Every rank holds the layer's full q, k, v (for instance after an
    all-gather of the projections); a rank reads the keys of its pooling
    rows and the q, k, v of its assigned groups only, and writes only its
    heads' rows of `out`.  The mask's host copy (B * Hq bytes) is the one
    synchronisation of the step: the assignment needs it."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, d: int, w1, b1, w2, b2,
                 sink: int, window: int, rank: int, world: int, device, group=None,
                 threshold: float = 0.0, mask: Optional[torch.Tensor] = None,
                 split_groups: bool = True):
        """w1..b2: the router's weights on `device`; or all None with `mask`
        (device uint8 [B, Hq]) given, for a layer whose routing is fixed (no
        router step, no exchange)."""
        from .api import attn_workspace, ea_router_mlp_workspace_size, ea_router_workspace_size
        from .api import make_params
        self.B, self.Hq, self.Hkv, self.N, self.d = B, Hq, Hkv, N, d
        self.router = (w1, b1, w2, b2)
        self.sink, self.window = sink, window
        self.rank, self.world, self.group = rank, world, group
        self.threshold = threshold
        self.dev = torch.device(device)
        self.row0, self.nrows = pool_rows(B, Hkv, world, rank)
        self.chunk = pool_chunk(B, Hkv, world)
        self.x_local = torch.zeros(self.chunk * d, dtype=torch.float32, device=self.dev)
        self.pool_ws = torch.empty(max(ea_router_workspace_size(B, Hkv, N, d), 16),
                                   dtype=torch.uint8, device=self.dev)
        hidden = w1.shape[0] if w1 is not None else 4
        self.mlp_ws = torch.empty(max(ea_router_mlp_workspace_size(B, hidden), 16),
                                  dtype=torch.uint8, device=self.dev)
        self.fixed_mask = mask is not None
        self.mask = mask if mask is not None else \
            torch.empty((B, Hq), dtype=torch.uint8, device=self.dev)
        self.mask_host = torch.empty((B, Hq), dtype=torch.uint8).pin_memory() \
            if torch.cuda.is_available() else torch.empty((B, Hq), dtype=torch.uint8)
        self.split_groups = split_groups
        self.sel = torch.empty((B, Hq), dtype=torch.uint8, device=self.dev)
        self.attn_ws = attn_workspace(make_params(B, Hq, Hkv, N, d, sink, window), self.dev)
        self.owner = None

    def route(self, k: torch.Tensor, stream=None) -> torch.Tensor:
        """Steps 1-3: the rank's pooling rows, the all-gather, the MLP.
        Returns the device mask (the same on every rank)."""
        from .api import ea_router_mlp, ea_router_pool_rows
        if self.fixed_mask:
            return self.mask
        ea_router_pool_rows(k, self.row0, self.nrows, x_out=self.x_local,
                            workspace=self.pool_ws, stream=stream)
        x = gather_pooled(self.x_local, self.B, self.Hkv, self.d, self.world, self.group)
        ea_router_mlp(x, *self.router, self.threshold, route_mask=self.mask,
                      workspace=self.mlp_ws, stream=stream)
        return self.mask

    def assign(self, stream=None) -> np.ndarray:
        """Step 4a: the host copy of the mask (synchronises the stream), the
        costs and the LPT assignment; uploads this rank's head selection.
        Returns the owner of every query head, [B, Hq]."""
        s = stream if stream is not None else torch.cuda.current_stream(self.dev)
        with torch.cuda.stream(s):
            self.mask_host.copy_(self.mask, non_blocking=True)
            s.synchronize()
            m = self.mask_host.numpy().copy()
            if self.split_groups:
                self.owner = lpt_assign_split(m, self.Hkv, self.N, self.sink, self.window,
                                              self.world)
            else:
                g = lpt_assign(group_costs(m, self.Hkv, self.N, self.sink, self.window),
                               self.world)
                self.owner = np.repeat(g, self.Hq // self.Hkv, axis=1)
            self.sel.copy_(torch.as_tensor((self.owner == self.rank).astype(np.uint8)))
        return self.owner

    def attend(self, q, k, v, out, stream=None) -> torch.Tensor:
        """Step 4b: the fused attention on this rank's query heads."""
        from .api import ea_hybrid_attn_prefill_heads
        return ea_hybrid_attn_prefill_heads(q, k, v, self.mask, self.sel, self.sink,
                                            self.window, out=out, workspace=self.attn_ws,
                                            stream=stream)

    def host_step(self, q_host, k_host, v_host, out_host, q, k, v, out, stream=None):
        """The step from pinned host buffers: the keys of the rank's pooling
        rows go up first; after the assignment, the q rows of the rank's
        heads and the k, v of their kv groups; its heads' output rows come
        back into out_host (valid after the stream synchronises).  q, k, v,
        out: full-size device buffers of which the rank uses its parts.
        Returns (bytes up, bytes down)."""
        s = stream if stream is not None else torch.cuda.current_stream(self.dev)
        G = self.Hq // self.Hkv
        up = down = 0
        with torch.cuda.stream(s):
            for r in range(self.row0, self.row0 + self.nrows):
                b, hk = divmod(r, self.Hkv)
                k[b, hk].copy_(k_host[b, hk], non_blocking=True)
                up += k[b, hk].numel() * k.element_size()
            self.route(k, s)
            owner = self.assign(s)
            mine = owner == self.rank
            for b in range(self.B):
                for hk in range(self.Hkv):
                    hs = [hk * G + j for j in range(G) if mine[b, hk * G + j]]
                    if not hs:
                        continue
                    for h in hs:
                        q[b, h].copy_(q_host[b, h], non_blocking=True)
                        up += q[b, h].numel() * q.element_size()
                    v[b, hk].copy_(v_host[b, hk], non_blocking=True)
                    up += v[b, hk].numel() * v.element_size()
                    if not (self.row0 <= b * self.Hkv + hk < self.row0 + self.nrows):
                        k[b, hk].copy_(k_host[b, hk], non_blocking=True)
                        up += k[b, hk].numel() * k.element_size()
            self.attend(q, k, v, out, s)
            for b, h in heads_of(owner, self.rank):
                out_host[b, h].copy_(out[b, h], non_blocking=True)
                down += out[b, h].numel() * out.element_size()
        return up, down

    def __call__(self, q, k, v, out, stream=None) -> torch.Tensor:
        self.route(k, stream)
        self.assign(stream)
        return self.attend(q, k, v, out, stream)


def head_rows_of(owner, rank: int, G: int) -> Sequence[Tuple[int, int]]:
    """(b, h) query heads whose rows `rank` writes."""
    o = np.asarray(owner)
    return [(b, hk * G + j) for b in range(o.shape[0]) for hk in range(o.shape[1])
            if o[b, hk] == rank for j in range(G)]
