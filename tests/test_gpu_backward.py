"""GPU parity of the training path (through the C ABI) against the oracle:
the forward's log-sum-exp and the backward's dQ, dK, dV for mixed FA/SA
heads under GQA."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import f64, sample_rows
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


# log-sum-exp: the forward's row sum adds bf16-rounded probabilities; bf16
# keeps 8 significand bits, so each is off by at most 2^-8 of itself (unit
# roundoff) and log(l) moves by at most -log(1 - 2^-8) = 3.91e-3.
LSE_ABS = 4.0e-3
# Gradients: P and dS enter the tensor cores as bf16 (relative 2^-8 each),
# sums are fp32, results are rounded to bf16 (relative 2^-8).  dS mixes signs,
# so the bound is normwise: max |err| <= 2^-6 max |ref| (4 unit roundoffs) and
# mean |err| <= 2^-7 mean |ref|.
GRAD_MAX_REL = 2.0 ** -6
GRAD_MEAN_REL = 2.0 ** -7


def _inputs(B, Hq, Hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    dout = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    return q, k, v, dout


def _grad_report(got, ref):
    err = np.abs(f64(got) - ref)
    return float(err.max()), float(err.mean()), float(np.abs(ref).max()), float(np.abs(ref).mean())


CASES = [
    # B, Hq, Hkv, N, S, W, mask
    (1, 4, 2, 300, 16, 64, [[0, 1, 1, 0]]),
    (2, 8, 2, 513, 4, 200, [[1, 1, 1, 1, 0, 0, 0, 0], [0, 1, 0, 1, 0, 1, 0, 1]]),
    (1, 2, 2, 128, 0, 1, [[1, 0]]),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,S,W,mask", CASES)
def test_backward_matches_oracle(B, Hq, Hkv, N, S, W, mask):
    d = 128
    q, k, v, dout = _inputs(B, Hq, Hkv, N, d, seed=N + Hq)
    m = torch.as_tensor(np.array(mask, np.uint8), device=DEV)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    out, lse = ea_hybrid_attn_prefill_lse(qd, kd, vd, m, S, W)
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device=DEV)
    dq, dk, dv = ea_hybrid_attn_backward(qd, kd, vd, out, dod, lse, m, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    mn = np.array(mask, np.uint8)
    ref_lse = oracle.attention_lse(f64(q), f64(k), mn, S, W)
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() <= LSE_ABS
    rq, rk, rv = oracle.attention_backward(f64(q), f64(k), f64(v), f64(dout), mn, S, W)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        mx, mean, rmax, rmean = _grad_report(got, ref)
        print(name, mx, mean, rmax, rmean)
        assert np.all(np.isfinite(f64(got))), name
        assert mx <= GRAD_MAX_REL * rmax and mean <= GRAD_MEAN_REL * rmean, \
            (name, mx, mean, rmax, rmean)


def test_backward_llama_layer_shape():
    """llama8b layer shape (32 query heads, 8 kv heads, d 128) at N = 2048,
    router-like mask with most heads SA and mixed GQA groups."""
    B, Hq, Hkv, N, S, W, d = 1, 32, 8, 2048, 64, 1024, 128
    q, k, v, dout = _inputs(B, Hq, Hkv, N, d, seed=2048)
    rng = np.random.default_rng(3)
    mn = (rng.random((B, Hq)) < 0.68).astype(np.uint8)
    m = torch.as_tensor(mn, device=DEV)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    out, lse = ea_hybrid_attn_prefill_lse(qd, kd, vd, m, S, W)
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device=DEV)
    dq, dk, dv = ea_hybrid_attn_backward(qd, kd, vd, out, dod, lse, m, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    rq, rk, rv = oracle.attention_backward(f64(q), f64(k), f64(v), f64(dout), mn, S, W)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        mx, mean, rmax, rmean = _grad_report(got, ref)
        assert mx <= GRAD_MAX_REL * rmax and mean <= GRAD_MEAN_REL * rmean, \
            (name, mx, mean, rmax, rmean)


def test_backward_full_schedule_sampled_n16k():
    """The llama8b layer shape at N = 16384 (128 query tiles per head, so the
    sink key tiles gather every query tile of all G heads of their group in
    the dK/dV schedule): all heads run on the GPU; the oracle checks sampled
    dQ rows of two kv groups (one mixing FA and SA heads, one all SA) and
    three whole key tiles of dK and dV (the first, holding the sinks, one in
    the middle and the last), each from the gradients' definition."""
    B, Hq, Hkv, N, S, W, d = 1, 32, 8, 16384, 64, 1024, 128
    q, k, v, dout = _inputs(B, Hq, Hkv, N, d, seed=16384)
    rng = np.random.default_rng(16)
    mn = (rng.random((B, Hq)) < 0.68).astype(np.uint8)
    mn[0, 0:4] = [0, 1, 1, 1]      # group 0: one FA head, three SA heads
    mn[0, 20:24] = 1               # group 5: all SA
    m = torch.as_tensor(mn, device=DEV)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    out, lse = ea_hybrid_attn_prefill_lse(qd, kd, vd, m, S, W)
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device=DEV)
    dq, dk, dv = ea_hybrid_attn_backward(qd, kd, vd, out, dod, lse, m, S, W, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    q_rows = sample_rows(N, S, W, 6, seed=5)
    key_rows = list(range(0, 128)) + list(range(8192, 8320)) + list(range(N - 128, N))
    q64, k64, v64, do64 = f64(q), f64(k), f64(v), f64(dout)
    dq_h, dk_h, dv_h = dq.cpu(), dk.cpu(), dv.cpu()
    for hk in (0, 5):
        rq, rk, rv = oracle.attention_backward_sampled(q64, k64, v64, do64, mn, 0, hk, q_rows,
                                                       key_rows, S, W)
        got_q = f64(dq_h[0, 4 * hk:4 * hk + 4][:, q_rows])
        got_k = f64(dk_h[0, hk, key_rows])
        got_v = f64(dv_h[0, hk, key_rows])
        for name, got, ref in (("dq", got_q, rq), ("dk", got_k, rk), ("dv", got_v, rv)):
            assert np.all(np.isfinite(got)), name
            err = np.abs(got - ref)
            mx, mean = float(err.max()), float(err.mean())
            rmax, rmean = float(np.abs(ref).max()), float(np.abs(ref).mean())
            assert mx <= GRAD_MAX_REL * rmax and mean <= GRAD_MEAN_REL * rmean, \
                (hk, name, mx, mean, rmax, rmean)
