"""The per-unit trace of the fused prefill (ea_hybrid_attn_prefill_traced):
the output equals the untraced call's bits, and the trace holds one record
per unit of the host schedule view, with that unit's mode, heads, rows and
tile count; units are dispatched dynamically, so each CTA runs the ranks it
took from the ticket counter in increasing order, one after another."""
import numpy as np
import pytest
import torch

from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (attn_workspace, ea_attn_grid_size,
                                            ea_get_device_status, ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_traced, ea_schedule_units,
                                            make_params)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W", [
    (1, 8, 2, 2048, 128, 64, 256),
    (2, 16, 4, 700, 64, 8, 100),
    (1, 8, 2, 131072, 128, 64, 1024),    # long FA units kv group by kv group
    (1, 48, 16, 600, 64, 8, 64),         # G = 3: groups over the prologue's 30-lane chunks
    (1, 64, 2, 300, 64, 8, 64),          # G = 32 over two chunks
])
def test_trace_matches_the_schedule(B, Hq, Hkv, N, d, S, W):
    g = torch.Generator().manual_seed(N)
    q, k, v = (torch.randn(s, generator=g).to(torch.bfloat16).to(DEV) for s in
               ((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d)))
    m = np.random.default_rng(N).integers(0, 2, size=(B, Hq)).astype(np.uint8)
    m[:, 0] = 0                                     # at least one FA head per sequence
    mask = torch.from_numpy(m).to(DEV)
    p = make_params(B, Hq, Hkv, N, d, S, W)
    ws = attn_workspace(p, DEV)
    plain = ea_hybrid_attn_prefill(q, k, v, mask, S, W, workspace=ws)
    traced, rec, total = ea_hybrid_attn_prefill_traced(q, k, v, mask, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    assert torch.equal(plain, traced)
    units = ea_schedule_units(m, p)       # rows: sparse, b, h0, h1, row0, n_kv_tiles
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    grid = ea_attn_grid_size(p, sms)
    assert total == len(units) == len(rec)
    # a second traced call on the same workspace: the ticket counter was
    # reset by the first launch's last CTA
    _, rec2, total2 = ea_hybrid_attn_prefill_traced(q, k, v, mask, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert total2 == total and sorted(rec2[:, 5].tolist()) == list(range(total))
    start, first_s, last_p, end, cta, rank, sparse, tiles = (rec[:, i] for i in range(8))
    assert sorted(rank.tolist()) == list(range(total))
    assert np.all(start > 0)
    assert np.all(first_s >= start) and np.all(last_p >= first_s) and np.all(end >= last_p)
    assert set(np.unique(cta).tolist()) <= set(range(grid))
    np.testing.assert_array_equal(sparse, units[rank, 0])
    np.testing.assert_array_equal(tiles, units[rank, 5])
    # the unit each rank ran is the host view's: both slots' heads and rows
    level, head0, head1 = rec[:, 8], rec[:, 9], rec[:, 10]
    u = units[rank]
    np.testing.assert_array_equal(head0, u[:, 1] * Hq + u[:, 2])
    np.testing.assert_array_equal(head1, u[:, 1] * Hq + u[:, 3])
    paired = u[:, 2] != u[:, 3]
    np.testing.assert_array_equal(np.where(paired, level * 128, (level >> 1) * 256), u[:, 4])
    if Hq // Hkv >= 2:
        assert np.any(paired)
    # a CTA runs its units one after another, in the increasing rank order of
    # its tickets
    for c in np.unique(cta):
        sel = np.where(cta == c)[0]
        order = sel[np.argsort(rank[sel])]
        assert np.all(start[order][1:] >= start[order][:-1])
        assert np.all(start[order][1:] >= end[order][:-1])
