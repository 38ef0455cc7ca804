"""The backward's work schedule on the GPU: the per-CTA unit lists that
ea_bwd_sched_kernel leaves in the backward workspace equal the host mirror's
(the sort by cost and the assignment are deterministic)."""
import numpy as np
import pytest
import torch

import bwd_sched_mirror as m
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_backward,
                                            ea_hybrid_attn_prefill_lse)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _read_lists(ws, B, Hq, Hkv, N):
    """Workspace: 256-byte status block, D (fp32 [B][Hq][N], padded to 256
    bytes), the dK/dV kernel's two padded vectors (fp32 [B*Hq][128 nT] each),
    then int32 offs_kv[1025], offs_q[1025], list/sorted/cta of dK/dV,
    list/sorted/cta of dQ."""
    nT = -(-N // m.BN)
    ukv, uq = B * Hkv * nT, B * Hq * nT
    base = 256 + (B * Hq * N * 4 + 255) // 256 * 256 + 2 * B * Hq * nT * 128 * 4
    ints = ws[base:].view(torch.int32).cpu().numpy().astype(np.int64)
    g = m.MAX_GRID + 1
    offs_kv, offs_q = ints[:g], ints[g:2 * g]
    w = 2 * g
    list_kv = ints[w:w + ukv]
    w += 3 * ukv
    list_q = ints[w:w + uq]
    return offs_kv, list_kv, offs_q, list_q


@pytest.mark.parametrize("B,Hq,Hkv,N,S,W,seed", [
    (1, 8, 2, 2048, 64, 256, 3),
    (2, 16, 4, 1000, 16, 300, 4),
])
def test_device_schedule_equals_mirror(B, Hq, Hkv, N, S, W, seed):
    d = 128
    rng = np.random.default_rng(seed)
    mask_np = (rng.random((B, Hq)) < 0.5).astype(np.uint8)
    mask_np[0, 0], mask_np[-1, -1] = 0, 1
    g = torch.Generator().manual_seed(seed)
    q, k, v, dout = (torch.randn(s, generator=g).to(torch.bfloat16).to(DEV)
                     for s in ((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, Hq, N, d)))
    mask = torch.from_numpy(mask_np).to(DEV)
    out, lse = ea_hybrid_attn_prefill_lse(q, k, v, mask, S, W)
    import ctypes
    from sparse_attention_head_b200 import _lib
    from sparse_attention_head_b200.api import make_params
    p = make_params(B, Hq, Hkv, N, d, S, W)
    n = int(_lib.load().ea_hybrid_attn_backward_workspace_size(ctypes.byref(p)))
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    ea_hybrid_attn_backward(q, k, v, out, dout, lse, mask, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    offs_kv, list_kv, offs_q, list_q = _read_lists(ws, B, Hq, Hkv, N)
    nT = -(-N // m.BN)
    for kdkdv, offs, lst in ((True, offs_kv, list_kv), (False, offs_q, list_q)):
        units = B * (Hkv if kdkdv else Hq) * nT
        grid = min(units, sms)
        want_offs, want_list, _ = m.schedule(kdkdv, mask_np, B, Hq, Hkv, N, S, W, grid)
        np.testing.assert_array_equal(offs[:grid + 1], want_offs)
        np.testing.assert_array_equal(lst, want_list)
