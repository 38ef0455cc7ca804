"""GPU parity of the packed variable-length prefill (through the C ABI)
against the oracle: every sequence of the batch is its own causal prefill,
positions restarting at its first token."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import compare, f64, few_key_rows_packed, sample_rows
from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import (EA_SELECT_FA, EA_SELECT_SA, ea_get_device_status,
                                            ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_varlen)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _packed(cu, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    T = cu[-1]
    q = torch.randn((T, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((T, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((T, Hkv, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _run(q, k, v, cu, mask, S, W, **kw):
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    cu_d = torch.as_tensor(cu, dtype=torch.int32, device=DEV)
    out = ea_hybrid_attn_prefill_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_d,
                                        torch.as_tensor(mask, device=DEV),
                                        int(max(np.diff(cu))), S, W, workspace=ws, **kw)
    torch.cuda.synchronize()
    return out, ws


CASES = [
    # cu_seqlens, Hq, Hkv, d, S, W
    ([0, 300, 300, 1000, 1077, 2600], 8, 2, 128, 16, 128),     # empty, short, ragged tails
    ([0, 1, 129, 130, 640], 4, 4, 64, 0, 1),                    # 1-token sequences, W = 1
    ([0, 2048, 2049, 2561], 8, 2, 64, 64, 300),                 # one long, one single token
    ([0, 513, 1026, 1539], 4, 1, 128, 130, 257),                # MQA, sinks span two tiles
]


@pytest.mark.parametrize("cu,Hq,Hkv,d,S,W", CASES)
def test_varlen_matches_oracle(cu, Hq, Hkv, d, S, W):
    B = len(cu) - 1
    q, k, v = _packed(cu, Hq, Hkv, d, seed=cu[-1] + d)
    rng = np.random.default_rng(cu[-1])
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    mask[0, 0], mask[-1, -1] = 0, 1
    out, ws = _run(q, k, v, cu, mask, S, W)
    assert ea_get_device_status(ws) == 0
    ref = oracle.attention_varlen(f64(q), f64(k), f64(v), cu, mask, S, W)
    compare(out, ref, f"varlen cu={cu}", few_keys=W <= 2,
            few_rows=None if W <= 2 else few_key_rows_packed(cu, mask, Hq, S, W))


def test_varlen_equal_lengths_match_the_padded_kernel_bitwise():
    B, Hq, Hkv, N, d, S, W = 3, 8, 2, 777, 128, 64, 256
    g = torch.Generator().manual_seed(3)
    q4 = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k4 = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    v4 = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    mask = np.array([[0, 1, 1, 0, 1, 0, 0, 1], [1] * 8, [0] * 8], np.uint8)
    padded = ea_hybrid_attn_prefill(q4.to(DEV), k4.to(DEV), v4.to(DEV),
                                    torch.as_tensor(mask, device=DEV), S, W)
    pack = (lambda t: t.permute(0, 2, 1, 3).reshape(B * N, t.shape[1], d).contiguous())
    cu = [0, N, 2 * N, 3 * N]
    out, ws = _run(pack(q4), pack(k4), pack(v4), cu, mask, S, W)
    assert ea_get_device_status(ws) == 0
    assert torch.equal(out.view(B, N, Hq, d).permute(0, 2, 1, 3), padded)


@pytest.mark.parametrize("select", [EA_SELECT_FA, EA_SELECT_SA])
def test_varlen_select_leaves_other_heads_untouched(select):
    cu, Hq, Hkv, d, S, W = [0, 400, 1200], 4, 2, 64, 8, 64
    q, k, v = _packed(cu, Hq, Hkv, d, seed=17)
    mask = np.array([[0, 1, 0, 1], [1, 1, 0, 0]], np.uint8)
    sentinel = torch.full((cu[-1], Hq, d), 7.0, dtype=torch.bfloat16, device=DEV)
    out, ws = _run(q, k, v, cu, mask, S, W, select=select, out=sentinel)
    assert ea_get_device_status(ws) == 0
    ref = oracle.attention_varlen(f64(q), f64(k), f64(v), cu, mask, S, W)
    got = f64(out)
    for b in range(2):
        for h in range(Hq):
            rows = slice(cu[b], cu[b + 1])
            chosen = (select == EA_SELECT_SA) == bool(mask[b, h])
            if chosen:
                assert np.abs(got[rows, h] - ref[rows, h]).max() <= 1e-2
            else:
                assert np.all(got[rows, h] == 7.0)


@pytest.mark.parametrize("cu", [[1, 5, 10], [0, 6, 4], [0, 5, 9]])
def test_varlen_inconsistent_offsets_are_reported(cu):
    Hq, Hkv, d = 2, 1, 64
    T = 10
    q, k, v = _packed([0, T], Hq, Hkv, d, seed=1)
    mask = np.zeros((2, Hq), np.uint8)
    sentinel = torch.full((T, Hq, d), 3.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    out = ea_hybrid_attn_prefill_varlen(q.to(DEV), k.to(DEV), v.to(DEV),
                                        torch.as_tensor(cu, dtype=torch.int32, device=DEV),
                                        torch.as_tensor(mask, device=DEV), 10, 1, 4,
                                        out=sentinel, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == _lib.EA_ERR_INVALID_ARG
    assert torch.all(out == 3.0)


def test_varlen_large_ragged_batch_sampled_rows():
    """A serving-like packed batch (llama8b layer shape), rows sampled per
    sequence and checked against the oracle row by row."""
    lens = [8192, 3000, 17, 12000, 256]
    cu = np.cumsum([0] + lens).tolist()
    Hq, Hkv, d, S, W = 32, 8, 128, 64, 1024
    q, k, v = _packed(cu, Hq, Hkv, d, seed=99)
    rng = np.random.default_rng(7)
    mask = (rng.random((len(lens), Hq)) < 0.68).astype(np.uint8)
    out, ws = _run(q, k, v, cu, mask, S, W)
    assert ea_get_device_status(ws) == 0
    got = f64(out)
    for b, n in enumerate(lens):
        t0 = cu[b]
        qs = f64(q[t0:t0 + n]).transpose(1, 0, 2)[None]
        ks = f64(k[t0:t0 + n]).transpose(1, 0, 2)[None]
        vs = f64(v[t0:t0 + n]).transpose(1, 0, 2)[None]
        rows = sample_rows(n, S, W, 12, seed=b)
        for h in (0, 5, 17, 31):
            ref = oracle.attention_rows(qs, ks, vs, mask[b:b + 1], 0, h, rows, S, W)
            err = np.abs(got[[t0 + r for r in rows], h] - ref)
            assert err.max() <= 1e-2, (b, h, float(err.max()))


# ---------------------------------------------------------------- router
from gpu_common import LOGIT_ABS, margin_controlled_b2  # noqa: E402
from sparse_attention_head_b200.api import ea_router_decide, ea_router_decide_varlen  # noqa: E402


def _router_weights(in_dim, hidden, Hq, seed):
    g = torch.Generator().manual_seed(seed)
    w1 = (torch.randn((hidden, in_dim), generator=g) * 0.05).float()
    b1 = (torch.randn((hidden,), generator=g) * 0.1).float()
    w2 = (torch.randn((Hq, hidden), generator=g) * 0.05).float()
    b2 = (torch.randn((Hq,), generator=g) * 0.05).float()
    return w1, b1, w2, b2


@pytest.mark.parametrize("cu,Hkv,d", [([0, 300, 300, 1000, 1077, 5000], 8, 128),
                                      ([0, 1, 4097, 4100], 4, 64)])
def test_varlen_router_matches_oracle(cu, Hkv, d):
    B, Hq, hidden = len(cu) - 1, 32, 256
    T = cu[-1]
    g = torch.Generator().manual_seed(T)
    # per-sequence channel offsets make the pooled vectors (and so the
    # routing) depend on each sequence's own keys
    offs = torch.randn((B, Hkv, d), generator=g)
    k = torch.randn((T, Hkv, d), generator=g)
    for b in range(B):
        k[cu[b]:cu[b + 1]] += offs[b]
    k = k.to(torch.bfloat16)
    w1, b1, w2, b2 = _router_weights(Hkv * d, hidden, Hq, seed=T + 1)
    b2 = torch.as_tensor(margin_controlled_b2(f64(k), w1.double().numpy(), b1.double().numpy(),
                                              w2.double().numpy(), b2.double().numpy(), cu=cu),
                         dtype=torch.float32)
    mask, z = ea_router_decide_varlen(k.to(DEV), torch.as_tensor(cu, dtype=torch.int32,
                                                                  device=DEV),
                                      int(max(np.diff(cu))), w1.to(DEV), b1.to(DEV), w2.to(DEV),
                                      b2.to(DEV))
    torch.cuda.synchronize()
    ref_mask, ref_z = oracle.router_decide_varlen(f64(k), cu, w1.double().numpy(),
                                                  b1.double().numpy(), w2.double().numpy(),
                                                  b2.double().numpy())
    np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask)
    assert np.abs(z.cpu().double().numpy() - ref_z).max() <= LOGIT_ABS
    assert len(set(map(tuple, ref_mask.tolist()))) > 1      # sequences route differently


def test_varlen_router_equal_lengths_match_the_padded_router_bitwise():
    B, Hkv, N, d, Hq, hidden = 3, 8, 2000, 128, 32, 256
    g = torch.Generator().manual_seed(12)
    k4 = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    w1, b1, w2, b2 = (t.to(DEV) for t in _router_weights(Hkv * d, hidden, Hq, seed=13))
    m_pad, z_pad = ea_router_decide(k4.to(DEV), w1, b1, w2, b2)
    packed = k4.permute(0, 2, 1, 3).reshape(B * N, Hkv, d).contiguous().to(DEV)
    cu = torch.as_tensor([0, N, 2 * N, 3 * N], dtype=torch.int32, device=DEV)
    m_var, z_var = ea_router_decide_varlen(packed, cu, N, w1, b1, w2, b2)
    torch.cuda.synchronize()
    assert torch.equal(m_pad, m_var) and torch.equal(z_pad, z_var)
