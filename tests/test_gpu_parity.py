"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded bf16 inputs.  Masks bit-exact; attention outputs within
max-abs 1e-2 and mean-abs 1e-3."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import compare, f64, margin_controlled_b2, sample_rows
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (EA_SELECT_FA, EA_SELECT_SA, attn_workspace,
                                            ea_get_device_status, ea_hybrid_attn_prefill,
                                            ea_router_decide, make_params)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _qkv(B, Hq, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _run(q, k, v, mask, S, W, **kw):
    ws = attn_workspace(make_params(*q.shape[:2], k.shape[1], q.shape[2], q.shape[3], S, W),
                        DEV)
    out = ea_hybrid_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), mask.to(DEV), S, W,
                                 workspace=ws, **kw)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    return out


def test_tiny_workload():
    w = workloads.get("tiny")
    seed = workloads.layer_seed(w)
    q, k, v = workloads.make_qkv(w, seed)
    mask = workloads.make_fixed_mask(w, seed)
    assert mask.tolist() == [[0, 1, 0, 1]]
    out = _run(q, k, v, mask, w.sink, w.window)
    ref = oracle.attention(f64(q), f64(k), f64(v), mask.numpy(), w.sink, w.window)
    compare(out, ref, "tiny")


EDGE = [
    # B, Hq, Hkv, N, d, S, W, mask kind
    (1, 2, 1, 1, 64, 0, 1, "rand"),
    (1, 2, 2, 17, 128, 3, 5, "rand"),
    (1, 4, 2, 128, 64, 16, 128, "rand"),
    (1, 4, 2, 129, 128, 16, 128, "rand"),
    (1, 2, 1, 255, 64, 0, 1, "sa"),
    (2, 4, 2, 256, 128, 1, 1, "sa"),
    (1, 4, 1, 257, 64, 130, 200, "rand"),
    (2, 8, 2, 640, 128, 64, 100, "rand"),
    (1, 4, 4, 1000, 64, 0, 300, "rand"),
    (1, 4, 2, 1000, 128, 40, 1200, "sa"),        # S + W >= N: SA equals FA
    (1, 4, 2, 777, 128, 5, 64, "fa"),
    (1, 2, 1, 1536, 128, 128, 512, "rand"),
    (2, 6, 3, 513, 64, 250, 2, "rand"),
    (1, 3, 1, 384, 128, 0, 129, "sa"),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W,kind", EDGE)
def test_edge_shapes(B, Hq, Hkv, N, d, S, W, kind):
    q, k, v = _qkv(B, Hq, Hkv, N, d, seed=N * 31 + S * 7 + W)
    rng = np.random.default_rng(N + W)
    if kind == "rand":
        m = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    elif kind == "sa":
        m = np.ones((B, Hq), np.uint8)
    else:
        m = np.zeros((B, Hq), np.uint8)
    mask = torch.from_numpy(m)
    out = _run(q, k, v, mask, S, W)
    ref = oracle.attention(f64(q), f64(k), f64(v), m, S, W)
    compare(out, ref, f"edge {B},{Hq},{Hkv},{N},{d},{S},{W},{kind}", few_keys=W <= 2)


def test_explicit_softmax_scale():
    q, k, v = _qkv(1, 4, 2, 300, 128, seed=5)
    m = np.array([[0, 1, 1, 0]], np.uint8)
    out = _run(q, k, v, torch.from_numpy(m), 8, 40, softmax_scale=0.05)
    ref = oracle.attention(f64(q), f64(k), f64(v), m, 8, 40, scale=0.05)
    compare(out, ref, "scale")


def test_split_pass_equals_fused_and_is_deterministic():
    q, k, v = _qkv(2, 8, 2, 1100, 128, seed=9)
    m = torch.from_numpy(np.random.default_rng(3).integers(0, 2, size=(2, 8)).astype(np.uint8))
    fused = _run(q, k, v, m, 32, 256)
    again = _run(q, k, v, m, 32, 256)
    assert torch.equal(fused, again)
    split = torch.full_like(fused, float("nan"))
    ws = attn_workspace(make_params(2, 8, 2, 1100, 128, 32, 256), DEV)
    qd, kd, vd, md = q.to(DEV), k.to(DEV), v.to(DEV), m.to(DEV)
    ea_hybrid_attn_prefill(qd, kd, vd, md, 32, 256, select=EA_SELECT_FA, out=split, workspace=ws)
    fa_only = split.clone()
    ea_hybrid_attn_prefill(qd, kd, vd, md, 32, 256, select=EA_SELECT_SA, out=split, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    assert torch.equal(split, fused)
    # the FA-only call leaves SA heads untouched
    for b in range(2):
        for h in range(8):
            if m[b, h]:
                assert torch.isnan(fa_only[b, h]).all()
            else:
                assert torch.equal(fa_only[b, h], fused[b, h])


def test_router_mask_bit_exact_data_driven():
    """Keys with a per-channel offset make the pooled vector O(1), so the
    logits depend on the data; the mask must match the oracle bit for bit."""
    B, Hkv, N, d, hidden, Hq = 3, 8, 4096 + 77, 128, 256, 32
    g = torch.Generator().manual_seed(21)
    mu = torch.randn((1, Hkv, 1, d), generator=g)
    k = (torch.randn((B, Hkv, N, d), generator=g) + mu).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.05
    b1 = torch.randn((hidden,), generator=g) * 0.05
    w2 = torch.randn((Hq, hidden), generator=g) * 0.2
    b2 = torch.zeros(Hq)
    kf = f64(k)
    b2 = torch.from_numpy(margin_controlled_b2(kf, w1.double().numpy(), b1.double().numpy(),
                                               w2.double().numpy(), b2.double().numpy()))
    b2 = b2.float()
    mask_ref, z_ref = oracle.router_decide(kf, w1.double().numpy(), b1.double().numpy(),
                                           w2.double().numpy(), b2.double().numpy())
    assert 0 < mask_ref.sum() < mask_ref.size      # both modes present
    mask, z = ea_router_decide(k.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(mask.cpu().numpy(), mask_ref)
    np.testing.assert_allclose(f64(z), z_ref, rtol=0, atol=1e-4)
    mask2, _ = ea_router_decide(k.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV))
    assert torch.equal(mask, mask2)


@pytest.mark.parametrize("d,N", [(64, 1), (64, 300), (128, 1000)])
def test_router_small_shapes(d, N):
    B, Hkv, hidden, Hq = 2, 2, 16, 4
    g = torch.Generator().manual_seed(N + d)
    k = (torch.randn((B, Hkv, N, d), generator=g) + 1.0).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.1
    b1 = torch.randn((hidden,), generator=g) * 0.1
    w2 = torch.randn((Hq, hidden), generator=g)
    kf = f64(k)
    b2 = torch.from_numpy(margin_controlled_b2(kf, w1.double().numpy(), b1.double().numpy(),
                                               w2.double().numpy(), np.zeros(Hq))).float()
    mask_ref, z_ref = oracle.router_decide(kf, w1.double().numpy(), b1.double().numpy(),
                                           w2.double().numpy(), b2.double().numpy())
    mask, z = ea_router_decide(k.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(mask.cpu().numpy(), mask_ref)
    np.testing.assert_allclose(f64(z), z_ref, rtol=0, atol=1e-4)


@pytest.mark.parametrize("d", [64, 128])
def test_output_only_16_byte_aligned(d):
    """The C ABI asks 16-byte alignment of out; the epilogue uses 32-byte
    stores only on a 32-byte aligned base.  An out buffer 16 bytes past a
    32-byte boundary gives the same bits as an aligned one."""
    B, Hq, Hkv, N, S, W = 1, 4, 2, 300, 8, 64
    q, k, v = (t.to(DEV) for t in _qkv(B, Hq, Hkv, N, d, 31 + d))
    mask = torch.tensor([[0, 1, 1, 0]], dtype=torch.uint8, device=DEV)
    ws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
    aligned = ea_hybrid_attn_prefill(q, k, v, mask, S, W, workspace=ws)
    n = q.numel()
    buf = torch.empty(n + 64, dtype=torch.bfloat16, device=DEV)
    base = buf.data_ptr()
    skip = ((32 - base % 32) % 32 + 16) // 2     # elements to a 16-mod-32 address
    out16 = buf[skip:skip + n].view(q.shape)
    assert out16.data_ptr() % 32 == 16
    ea_hybrid_attn_prefill(q, k, v, mask, S, W, workspace=ws, out=out16)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    assert torch.equal(aligned, out16)
    ref = oracle.attention(f64(q.cpu()), f64(k.cpu()), f64(v.cpu()), mask.cpu().numpy(), S, W)
    compare(out16, ref, "out16")


@pytest.mark.parametrize("B,Hq,Hkv,N,d", [
    (2, 3, 1, 300, 64),      # G = 3: a pair and a single per mode at most
    (1, 16, 2, 261, 128),    # G = 8
    (1, 32, 1, 200, 64),     # G = 32: the largest group that pairs
    (1, 64, 1, 130, 64),     # G = 64: every head runs single
    (1, 6, 6, 257, 128),     # G = 1: nothing to pair
    (1, 48, 16, 140, 64),    # G = 3 over two 30-lane chunks of the prologue's ballots
    (2, 40, 8, 129, 64),     # G = 5 over two chunks
])
def test_group_sizes_pairing(B, Hq, Hkv, N, d):
    """Query heads of one kv group and one route share paired units; every
    group size and odd-one-out case matches the oracle, and the split pass
    (one mode per launch) gives the same bits."""
    S, W = 16, 96
    q, k, v = _qkv(B, Hq, Hkv, N, d, 700 + Hq)
    mask = torch.from_numpy(np.random.default_rng(Hq + N).integers(0, 2, size=(B, Hq))
                            .astype(np.uint8))
    out = _run(q, k, v, mask, S, W)
    ref = oracle.attention(f64(q), f64(k), f64(v), mask.numpy(), S, W)
    compare(out, ref, f"G={Hq // Hkv}")
    fa = _run(q, k, v, mask, S, W, select=EA_SELECT_FA)
    sa = _run(q, k, v, mask, S, W, select=EA_SELECT_SA)
    m = mask.to(DEV).bool()[:, :, None, None]
    assert torch.equal(torch.where(m, sa, fa), out)
