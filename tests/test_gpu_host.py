"""GPU tests of ea_hybrid_attn_prefill_host (prefill from host buffers with
the uploads and downloads split into kv-head chunks).  The chunked host path
must give, bit for bit, what the device path (ea_router_decide, then
ea_hybrid_attn_prefill on device copies) gives, for every chunk size, and
match the oracle within the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import compare, f64, margin_controlled_b2
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (HostPrefill, attn_workspace, ea_get_device_status,
                                            ea_hybrid_attn_host_chunks,
                                            ea_hybrid_attn_host_workspace_size,
                                            ea_hybrid_attn_prefill, ea_hybrid_attn_prefill_host,
                                            ea_router_decide, make_params)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _qkv(B, Hq, Hkv, N, d, seed, pin=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = (torch.randn((B, Hkv, N, d), generator=g) +
         torch.randn((1, Hkv, 1, d), generator=g)).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    if pin:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    return q, k, v


def _router(k, Hq, hidden, seed):
    """Router weights with every oracle logit at least the margin away from
    the threshold (so the mask is unique), and both modes present."""
    B, Hkv, N, d = k.shape
    g = torch.Generator().manual_seed(seed)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.05
    b1 = torch.randn((hidden,), generator=g) * 0.05
    w2 = torch.randn((Hq, hidden), generator=g) * 0.2
    kf = f64(k)
    b2 = margin_controlled_b2(kf, w1.double().numpy(), b1.double().numpy(),
                              w2.double().numpy(), np.zeros(Hq))
    mask_ref, _ = oracle.router_decide(kf, w1.double().numpy(), b1.double().numpy(),
                                       w2.double().numpy(), b2)
    return (w1, b1, w2, torch.from_numpy(b2).float()), mask_ref


def _device_path(q, k, v, S, W, router=None, mask=None):
    """ea_router_decide (or the given mask) then ea_hybrid_attn_prefill on
    device copies: the reference for the host path's bits."""
    B, Hq, N, d = q.shape
    kd = k.to(DEV)
    if router is not None:
        mask, _ = ea_router_decide(kd, *(t.to(DEV) for t in router))
    else:
        mask = mask.to(DEV)
    ws = attn_workspace(make_params(B, Hq, k.shape[1], N, d, S, W), DEV)
    out = ea_hybrid_attn_prefill(q.to(DEV), kd, v.to(DEV), mask, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    return out.cpu(), mask.cpu()


def _host_path(q, k, v, S, W, chunk, router=None, mask=None, stream=None):
    B, Hq, N, d = q.shape
    p = make_params(B, Hq, k.shape[1], N, d, S, W)
    hidden = router[0].shape[0] if router is not None else 0
    ws = torch.zeros(ea_hybrid_attn_host_workspace_size(p, hidden), dtype=torch.uint8,
                     device=DEV)
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    mask_out = torch.full((B, Hq), 7, dtype=torch.uint8)
    dev_router = tuple(t.to(DEV) for t in router) if router is not None else None
    ea_hybrid_attn_prefill_host(q, k, v, S, W, out_host=out, workspace=ws, router=dev_router,
                                route_mask_host=None if router is not None else mask.reshape(-1),
                                route_mask_out_host=mask_out, kv_heads_per_chunk=chunk,
                                stream=stream)
    (stream or torch.cuda.current_stream()).synchronize()
    assert ea_get_device_status(ws) == 0
    return out, mask_out


def test_tiny_workload_fixed_mask():
    """The tiny workload (fixed mask, d = 64): bit-identical to the device
    path, within the tolerance of the oracle, and the mask copied back."""
    w = workloads.get("tiny")
    seed = workloads.layer_seed(w)
    q, k, v = workloads.make_qkv(w, seed)
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    mask = workloads.make_fixed_mask(w, seed)
    ref_out, _ = _device_path(q, k, v, w.sink, w.window, mask=mask)
    for chunk in (0, 1, 2):
        out, mask_out = _host_path(q, k, v, w.sink, w.window, chunk, mask=mask)
        assert torch.equal(out, ref_out), f"chunk {chunk}"
        assert torch.equal(mask_out, mask)
    ref = oracle.attention(f64(q), f64(k), f64(v), mask.numpy(), w.sink, w.window)
    compare(out, ref, "tiny host path")


@pytest.mark.parametrize("chunk", [0, 1, 3, 4, 9])
def test_router_chunks_bit_identical(chunk):
    """Router path, B = 2, a ragged length and chunk sizes that do and do not
    divide Hkv: the mask equals the oracle's and the output equals the
    device path's bit for bit."""
    B, Hq, Hkv, N, d, S, W = 2, 8, 4, 700, 128, 16, 200
    q, k, v = _qkv(B, Hq, Hkv, N, d, seed=31)
    router, mask_ref = _router(k, Hq, 64, seed=32)
    assert 0 < mask_ref.sum() < mask_ref.size
    ref_out, ref_mask = _device_path(q, k, v, S, W, router=router)
    np.testing.assert_array_equal(ref_mask.numpy(), mask_ref)
    out, mask_out = _host_path(q, k, v, S, W, chunk, router=router)
    np.testing.assert_array_equal(mask_out.numpy(), mask_ref)
    assert torch.equal(out, ref_out)
    p = make_params(B, Hq, Hkv, N, d, S, W)
    c = min(chunk, Hkv) if chunk > 0 else max(1, (B * Hkv + 7) // 8)
    assert ea_hybrid_attn_host_chunks(p, chunk) == B * -(-Hkv // c)


def test_oracle_rows_router_path():
    """The host path against the oracle directly (sampled rows of every
    head), with the router deciding the modes."""
    B, Hq, Hkv, N, d, S, W = 1, 8, 2, 1536, 128, 64, 256
    q, k, v = _qkv(B, Hq, Hkv, N, d, seed=41)
    router, mask_ref = _router(k, Hq, 32, seed=42)
    out, mask_out = _host_path(q, k, v, S, W, 1, router=router)
    np.testing.assert_array_equal(mask_out.numpy(), mask_ref)
    rows = [0, 1, 63, 64, 255, 256, 319, 320, 700, 1024, N - 1]
    qf, kf, vf = f64(q), f64(k), f64(v)
    ref = np.stack([oracle.attention_rows(qf, kf, vf, mask_ref, 0, h, rows, S, W)
                    for h in range(Hq)])[None]
    compare(out[:, :, rows], ref, "host path sampled rows")


def test_pageable_buffers_and_side_stream():
    """Pageable host memory gives the same bits (without the overlap), and
    the call orders itself on a side stream."""
    B, Hq, Hkv, N, d, S, W = 1, 4, 2, 600, 64, 8, 100
    q, k, v = _qkv(B, Hq, Hkv, N, d, seed=51, pin=False)
    mask = torch.tensor([[1, 0, 0, 1]], dtype=torch.uint8)
    ref_out, _ = _device_path(q, k, v, S, W, mask=mask)
    side = torch.cuda.Stream()
    out, _ = _host_path(q, k, v, S, W, 1, mask=mask, stream=side)
    assert torch.equal(out, ref_out)


def test_host_prefill_reuse():
    """HostPrefill reuses its workspace: two calls on different inputs each
    match the device path."""
    B, Hq, Hkv, N, d, S, W = 1, 8, 4, 1000, 128, 32, 300
    q0, k0, v0 = _qkv(B, Hq, Hkv, N, d, seed=61)
    router, _ = _router(k0, Hq, 64, seed=161)
    hp = HostPrefill(B, Hq, Hkv, N, d, *router, S, W, device=DEV)
    outs = []
    for q, k, v in ((q0, k0, v0), _qkv(B, Hq, Hkv, N, d, seed=62)):
        hp(q, k, v)
        torch.cuda.synchronize()
        ref_out, _ = _device_path(q, k, v, S, W, router=router)
        assert torch.equal(hp.out_host, ref_out)
        outs.append(hp.out_host.clone())
    assert not torch.equal(outs[0], outs[1])
    assert ea_get_device_status(hp.workspace) == 0


def test_llama8b_full_size_matches_device_path():
    """The bench's e2e configuration (llama8b layer, router, automatic
    chunks): the host path's mask and output equal the device path's bit for
    bit, and its rows match the oracle on a sample of every head."""
    w = workloads.get("llama8b")
    seed = workloads.layer_seed(w)
    q, k, v = workloads.make_qkv(w, seed)
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    heads = workloads.sparse_head_set(w.hq, w.sparse_frac, seed)
    router = workloads.make_router_weights(w.hkv * w.d, w.router_hidden, w.hq, heads, seed)
    hp = HostPrefill(w.batch, w.hq, w.hkv, w.seq, w.d, *router, w.sink, w.window, device=DEV)
    assert hp.chunks == 8
    hp(q, k, v)
    torch.cuda.synchronize()
    assert ea_get_device_status(hp.workspace) == 0
    ref_out, ref_mask = _device_path(q, k, v, w.sink, w.window, router=router)
    assert int(ref_mask.sum()) == 22
    assert torch.equal(hp.out_host, ref_out)
    qf, kf, vf = f64(q), f64(k), f64(v)
    rows = [0, 1, 63, 64, 1023, 1024, 1087, 1088, 20000, w.seq - 1]
    for h in range(0, w.hq, 5):
        ref = oracle.attention_rows(qf, kf, vf, ref_mask.numpy(), 0, h, rows, w.sink, w.window)
        compare(hp.out_host[0, h, rows], ref, f"llama8b host path head {h}")


def test_shutdown_then_call_again():
    """ea_shutdown releases the copy streams; the next call recreates them
    and gives the same bits."""
    from sparse_attention_head_b200.api import ea_shutdown
    B, Hq, Hkv, N, d, S, W = 1, 4, 2, 400, 64, 8, 100
    q, k, v = _qkv(B, Hq, Hkv, N, d, seed=71)
    mask = torch.tensor([[0, 1, 1, 0]], dtype=torch.uint8)
    first, _ = _host_path(q, k, v, S, W, 1, mask=mask)
    ea_shutdown()
    again, _ = _host_path(q, k, v, S, W, 1, mask=mask)
    assert torch.equal(first, again)
    ea_shutdown()
    ea_shutdown()


def test_two_calls_in_flight_on_two_streams():
    """Two host-buffer calls with their own workspaces, enqueued on two
    streams before either is synchronised, share the library's copy streams;
    each still equals the device path."""
    B, Hq, Hkv, N, d, S, W = 1, 8, 4, 900, 128, 16, 200
    calls = []
    for seed in (81, 82):
        q, k, v = _qkv(B, Hq, Hkv, N, d, seed=seed)
        router, _ = _router(k, Hq, 32, seed=seed + 100)
        hp = HostPrefill(B, Hq, Hkv, N, d, *router, S, W, device=DEV, kv_heads_per_chunk=1)
        calls.append((hp, (q, k, v), router, torch.cuda.Stream()))
    torch.cuda.synchronize()
    for hp, (q, k, v), _, stream in calls:
        hp(q, k, v, stream=stream)
    torch.cuda.synchronize()
    for hp, (q, k, v), router, _ in calls:
        ref_out, _ = _device_path(q, k, v, S, W, router=router)
        assert torch.equal(hp.out_host, ref_out)
        assert ea_get_device_status(hp.workspace) == 0
