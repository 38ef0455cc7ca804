"""GPU: router and attention in one (cooperative) launch.  The routed launch
must give, bit for bit, what the router followed by the attention gives, and
its masks must match the oracle's routing exactly."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import LOGIT_ABS, compare, f64, few_key_rows_packed, margin_controlled_b2
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_routed,
                                            ea_hybrid_attn_prefill_varlen,
                                            ea_hybrid_attn_prefill_varlen_routed,
                                            ea_router_decide, ea_router_decide_varlen)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _weights(in_dim, hidden, Hq, seed):
    g = torch.Generator().manual_seed(seed)
    w1 = (torch.randn((hidden, in_dim), generator=g) * 0.05).float()
    b1 = (torch.randn((hidden,), generator=g) * 0.1).float()
    w2 = (torch.randn((Hq, hidden), generator=g) * 0.05).float()
    b2 = (torch.randn((Hq,), generator=g) * 0.05).float()
    return w1, b1, w2, b2


def _keys_with_offsets(shape, seq_axis_slices, seed):
    """Random keys plus a per-sequence channel offset, so each sequence's
    pooled keys (and its routing) differ."""
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(shape, generator=g)
    for sl in seq_axis_slices:
        k[sl] += torch.randn(shape[-1], generator=g)
    return k.to(torch.bfloat16)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W", [(2, 8, 2, 1000, 128, 16, 128),
                                               (1, 32, 8, 4096, 128, 64, 1024),
                                               (3, 4, 4, 300, 64, 0, 7)])
def test_routed_equals_router_then_attention(B, Hq, Hkv, N, d, S, W):
    g = torch.Generator().manual_seed(N + d)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = _keys_with_offsets((B, Hkv, N, d), [(b,) for b in range(B)], seed=N)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    w1, b1, w2, b2 = _weights(Hkv * d, 256, Hq, seed=N + 1)
    b2 = torch.as_tensor(margin_controlled_b2(f64(k), w1.double().numpy(), b1.double().numpy(),
                                              w2.double().numpy(), b2.double().numpy()),
                         dtype=torch.float32)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    wd = [t.to(DEV) for t in (w1, b1, w2, b2)]
    mask2, z2 = ea_router_decide(kd, *wd)
    out2 = ea_hybrid_attn_prefill(qd, kd, vd, mask2, S, W)
    logits = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device=DEV)
    for rep in range(3):          # the grid barrier is reused launch after launch
        out1, mask1, _ = ea_hybrid_attn_prefill_routed(qd, kd, vd, *wd, S, W, logits=logits,
                                                       workspace=ws)
        torch.cuda.synchronize()
        assert ea_get_device_status(ws) == 0
        assert torch.equal(mask1, mask2) and torch.equal(logits, z2), rep
        assert torch.equal(out1, out2), rep
    ref_mask, ref_z = oracle.router_decide(f64(k), w1.double().numpy(), b1.double().numpy(),
                                           w2.double().numpy(), b2.double().numpy())
    np.testing.assert_array_equal(mask1.cpu().numpy(), ref_mask)
    assert np.abs(logits.cpu().double().numpy() - ref_z).max() <= LOGIT_ABS
    if N <= 1000:
        ref = oracle.attention(f64(q), f64(k), f64(v), ref_mask, S, W)
        compare(out1, ref, "routed", few_keys=W <= 2)


def test_routed_packed_equals_router_then_attention():
    lens = [1200, 0, 77, 3000, 513]
    cu = np.cumsum([0] + lens).tolist()
    T, Hq, Hkv, d, S, W = cu[-1], 16, 4, 128, 32, 256
    g = torch.Generator().manual_seed(5)
    q = torch.randn((T, Hq, d), generator=g).to(torch.bfloat16)
    k = _keys_with_offsets((T, Hkv, d), [slice(cu[b], cu[b + 1]) for b in range(len(lens))], 6)
    v = torch.randn((T, Hkv, d), generator=g).to(torch.bfloat16)
    w1, b1, w2, b2 = _weights(Hkv * d, 256, Hq, seed=7)
    b2 = torch.as_tensor(margin_controlled_b2(f64(k), w1.double().numpy(), b1.double().numpy(),
                                              w2.double().numpy(), b2.double().numpy(), cu=cu),
                         dtype=torch.float32)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    wd = [t.to(DEV) for t in (w1, b1, w2, b2)]
    cud = torch.as_tensor(cu, dtype=torch.int32, device=DEV)
    L = max(lens)
    mask2, z2 = ea_router_decide_varlen(kd, cud, L, *wd)
    out2 = ea_hybrid_attn_prefill_varlen(qd, kd, vd, cud, mask2, L, S, W)
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device=DEV)
    logits = torch.empty((len(lens), Hq), dtype=torch.float32, device=DEV)
    out1, mask1, _ = ea_hybrid_attn_prefill_varlen_routed(qd, kd, vd, cud, L, *wd, S, W,
                                                          logits=logits, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    assert torch.equal(mask1, mask2) and torch.equal(logits, z2)
    assert torch.equal(out1, out2)
    ref_mask, _ = oracle.router_decide_varlen(f64(k), cu, w1.double().numpy(),
                                              b1.double().numpy(), w2.double().numpy(),
                                              b2.double().numpy())
    np.testing.assert_array_equal(mask1.cpu().numpy(), ref_mask)
    ref = oracle.attention_varlen(f64(q), f64(k), f64(v), cu, ref_mask, S, W)
    compare(out1, ref, "routed packed", few_rows=few_key_rows_packed(cu, ref_mask, Hq, S, W))
