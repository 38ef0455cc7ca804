"""The device entry points inside CUDA graphs: a router + fused prefill
step, and a decode step, captured once (after a warm-up call, which sets
the kernels' shared-memory attributes outside the capture) and replayed on
new inputs copied into the captured buffers, give the same bits as eager
calls."""
import numpy as np
import pytest
import torch

from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (attn_workspace, decode_workspace,
                                            ea_decode_kv_policy, ea_get_device_status,
                                            ea_hybrid_attn_decode, ea_hybrid_attn_prefill,
                                            ea_router_decide, ea_router_workspace_size,
                                            make_decode_params, make_params)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _rand(shape, seed, offset=0.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) + offset).to(torch.bfloat16).to(DEV)


def test_prefill_step_in_a_graph():
    B, Hq, Hkv, N, d, S, W, hidden = 2, 8, 4, 700, 128, 16, 200, 32
    g = torch.Generator().manual_seed(3)
    w1 = (torch.randn((hidden, Hkv * d), generator=g) * 0.05).to(DEV)
    b1 = torch.zeros(hidden, device=DEV)
    w2 = torch.randn((Hq, hidden), generator=g).to(DEV)
    b2 = torch.tensor([3.0, -3.0] * (Hq // 2), device=DEV)
    q, k, v = (torch.empty(s, dtype=torch.bfloat16, device=DEV) for s in
               ((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d)))
    mask = torch.empty((B, Hq), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    rws = torch.empty(ea_router_workspace_size(B, Hkv, N, d), dtype=torch.uint8, device=DEV)
    aws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)

    def step():
        ea_router_decide(k, w1, b1, w2, b2, workspace=rws, route_mask=mask, want_logits=False)
        ea_hybrid_attn_prefill(q, k, v, mask, S, W, out=out, workspace=aws)

    inputs = [[_rand(t.shape, 10 * i + j, 0.5 if j == 1 else 0.0) for j, t in
               enumerate((q, k, v))] for i in range(3)]
    for dst, src in zip((q, k, v), inputs[0]):
        dst.copy_(src)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for qkv in inputs:
        for dst, src in zip((q, k, v), qkv):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        got_out, got_mask = out.clone(), mask.clone()
        step()                                   # eager, same buffers
        torch.cuda.synchronize()
        assert torch.equal(got_mask, mask)
        assert torch.equal(got_out, out)
    assert ea_get_device_status(aws) == 0


def test_decode_step_in_a_graph():
    B, Hq, Hkv, d, S, W, max_len = 2, 8, 4, 128, 4, 100, 600
    mask_np = np.array([[1, 1, 0, 1, 1, 1, 1, 1], [0, 0, 1, 1, 1, 1, 1, 1]], dtype=np.uint8)
    slots, n_full, n_sa = ea_decode_kv_policy(mask_np, Hkv)
    mask = torch.as_tensor(mask_np, device=DEV)
    slot_t = torch.as_tensor(slots, dtype=torch.int32, device=DEV)

    def caches():
        z = dict(dtype=torch.bfloat16, device=DEV)
        return (torch.zeros((n_full, max_len, d), **z), torch.zeros((n_full, max_len, d), **z),
                torch.zeros((n_sa, S + W, d), **z), torch.zeros((n_sa, S + W, d), **z))

    ws_e = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    ws_g = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    ce, cg = caches(), caches()
    q, kn, vn = (torch.empty(s, dtype=torch.bfloat16, device=DEV) for s in
                 ((B, Hq, d), (B, Hkv, d), (B, Hkv, d)))
    pos = torch.zeros(B, dtype=torch.int32, device=DEV)
    out_g = torch.empty_like(q)

    def step_graph():
        ea_hybrid_attn_decode(q, kn, vn, pos, mask, slot_t, *cg, S, W, max_len, out=out_g,
                              workspace=ws_g)

    # positions 0..2 run eagerly on both cache sets (the first is the warm-up);
    # the graph, captured at position 3, then runs the remaining steps
    graph = None
    for t in range(12):
        q.copy_(_rand((B, Hq, d), 100 + t))
        kn.copy_(_rand((B, Hkv, d), 200 + t))
        vn.copy_(_rand((B, Hkv, d), 300 + t))
        pos.fill_(t)
        want = ea_hybrid_attn_decode(q, kn, vn, pos, mask, slot_t, *ce, S, W, max_len,
                                     workspace=ws_e)
        if t < 3:
            step_graph()
        elif graph is None:
            graph = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.graph(graph, stream=s):
                step_graph()                     # the capture does not run it
            torch.cuda.current_stream().wait_stream(s)
            graph.replay()
        else:
            graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, want), f"position {t}"
    for a, b in zip(ce, cg):
        assert torch.equal(a, b)
    assert ea_get_device_status(ws_g) == 0
