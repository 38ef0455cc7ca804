"""Parity at the limits the entry points accept: B * Hq = 4096 schedule
entries, a packed batch of 1024 sequences, eight query heads per kv head,
and the router at its largest input, hidden and head sizes."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import LOGIT_ABS, compare, f64, margin_controlled_b2
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
                                            ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_varlen, ea_router_decide,
                                            make_params)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,S,W", [
    (64, 64, 8, 130, 64, 4, 64),      # B * Hq = 4096 entries, eight heads per kv head
    (1, 8, 1, 700, 128, 32, 256),     # one kv head for eight query heads, d = 128
])
def test_entry_limit_and_eight_heads_per_kv_head(B, Hq, Hkv, N, d, S, W):
    q, k, v = _rand((B, Hq, N, d), 1), _rand((B, Hkv, N, d), 2), _rand((B, Hkv, N, d), 3)
    m = np.random.default_rng(B + N).integers(0, 2, size=(B, Hq)).astype(np.uint8)
    ws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
    out = ea_hybrid_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(m).to(DEV),
                                 S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    ref = oracle.attention(f64(q), f64(k), f64(v), m, S, W)
    compare(out, ref, f"limits B{B} Hq{Hq} Hkv{Hkv} N{N} d{d}")


def test_packed_batch_of_1024_sequences():
    B, Hq, Hkv, d, S, W = 1024, 4, 2, 64, 3, 16
    lens = np.random.default_rng(7).integers(1, 41, size=B)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = _rand((T, Hq, d), 11), _rand((T, Hkv, d), 12), _rand((T, Hkv, d), 13)
    m = np.random.default_rng(8).integers(0, 2, size=(B, Hq)).astype(np.uint8)
    out = ea_hybrid_attn_prefill_varlen(q.to(DEV), k.to(DEV), v.to(DEV),
                                        torch.from_numpy(cu).to(DEV), torch.from_numpy(m).to(DEV),
                                        int(lens.max()), S, W)
    torch.cuda.synchronize()
    ref = oracle.attention_varlen(f64(q), f64(k), f64(v), cu, m, S, W)
    # the first rows of a sequence see one to four keys: the bf16 output rounding
    # allowance of the few-key rows applies there
    few = np.zeros((T, Hq, 1), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            for i in range(min(4, int(lens[b]))):
                few[cu[b] + i, h, 0] = len(oracle.visible_keys(i, bool(m[b, h]), S, W)) <= 4
    compare(out, ref, "1024 packed sequences", few_rows=few)


def test_router_at_its_largest_sizes():
    """Hkv * d = 8192 pooled inputs, hidden = 4096, Hq = 1024 heads."""
    B, Hkv, N, d, hidden, Hq = 2, 64, 100, 128, 4096, 1024
    g = torch.Generator().manual_seed(21)
    mu = torch.randn((1, Hkv, 1, d), generator=g)
    k = (torch.randn((B, Hkv, N, d), generator=g) + mu).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.02
    b1 = torch.randn((hidden,), generator=g) * 0.02
    w2 = torch.randn((Hq, hidden), generator=g) * 0.05
    kf = f64(k)
    b2 = torch.from_numpy(margin_controlled_b2(kf, w1.double().numpy(), b1.double().numpy(),
                                               w2.double().numpy(), np.zeros(Hq))).float()
    mask_ref, z_ref = oracle.router_decide(kf, w1.double().numpy(), b1.double().numpy(),
                                           w2.double().numpy(), b2.double().numpy())
    assert 0 < mask_ref.sum() < mask_ref.size
    mask, z = ea_router_decide(k.to(DEV), w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(mask.cpu().numpy(), mask_ref)
    # fp32 sums of 8192 and 4096 terms: measured max |z - z_ref| ~5e-6 on a B200
    np.testing.assert_allclose(f64(z), z_ref, rtol=0, atol=LOGIT_ABS)


def test_decode_step_at_the_group_limit():
    """B * Hkv = 4096 (sequence, kv head) groups, every kind of group (all
    SA with a compact cache, mixed, all FA), ragged positions."""
    from test_gpu_decode import _caches, _history, _mask, _prefill_caches, _step
    from sparse_attention_head_b200.api import (decode_workspace, ea_decode_kv_policy,
                                                make_decode_params)
    B, Hq, Hkv, d, S, W, max_len = 512, 32, 8, 64, 4, 32, 80
    pos = np.random.default_rng(5).integers(0, max_len, size=B).tolist()
    L = max(pos) + 1
    q, k, v = _history(B, Hq, Hkv, L, d, seed=99)
    mask = _mask(B, Hq, Hkv, seed=98)
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    caches = _caches(slots, n_full, n_sa, max_len, S, W, d)
    _prefill_caches(caches, slots, k, v, pos, S, W)
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    idx = torch.as_tensor(pos, dtype=torch.long)
    bi = torch.arange(B)
    q_t, k_t, v_t = q[bi, :, idx], k[bi, :, idx], v[bi, :, idx]
    out = _step(q_t, k_t, v_t, pos, mask, slots, caches, S, W, max_len, ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    ref = oracle.decode_step(f64(q_t), f64(k), f64(v), pos, mask, S, W)
    # position 0 sees one key and positions 1-3 at most four: the few-key
    # allowance of bf16 output rounding applies to those rows
    few = np.array([p <= 3 for p in pos], dtype=bool)[:, None, None]
    compare(out, ref, "decode at 4096 groups", few_rows=few)


def test_backward_with_many_heads():
    """2048 (batch, head) entries with eight query heads per kv head, two key
    tiles: the backward's cost-sorted schedule over 512 dK/dV units and 4096
    dQ units, against the oracle."""
    from sparse_attention_head_b200.api import (ea_hybrid_attn_backward,
                                                ea_hybrid_attn_prefill_lse)
    B, Hq, Hkv, N, d, S, W = 32, 64, 8, 150, 128, 8, 64
    q, k, v, dout = (_rand(s, 30 + i) for i, s in
                     enumerate(((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, Hq, N, d))))
    mn = np.random.default_rng(31).integers(0, 2, size=(B, Hq)).astype(np.uint8)
    m = torch.as_tensor(mn, device=DEV)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    out, lse = ea_hybrid_attn_prefill_lse(qd, kd, vd, m, S, W)
    dq, dk, dv = ea_hybrid_attn_backward(qd, kd, vd, out, dod, lse, m, S, W)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attention_backward(f64(q), f64(k), f64(v), f64(dout), mn, S, W)
    # the normwise bound of the backward tests: P and dS enter the tensor cores
    # as bf16 and the results are bf16 (2^-6 of the max, 2^-7 of the mean)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = np.abs(f64(got) - ref)
        assert np.all(np.isfinite(f64(got))), name
        assert err.max() <= 2.0 ** -6 * np.abs(ref).max(), (name, float(err.max()))
        assert err.mean() <= 2.0 ** -7 * np.abs(ref).mean(), (name, float(err.mean()))
