"""Out-of-bounds writes, without a sanitizer: every entry point writes into
the middle of a canary-filled buffer, at ragged sizes (sequence lengths that
are not multiples of the 128-row tile, batches of several sequences), and
the canaries before and after must be untouched afterwards.  The outputs
are also scanned for NaN and Inf."""
import math

import numpy as np
import pytest
import torch

from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (HostPrefill, attn_workspace, decode_workspace,
                                            ea_decode_kv_policy, ea_get_device_status,
                                            ea_hybrid_attn_backward, ea_hybrid_attn_decode,
                                            ea_hybrid_attn_prefill, ea_hybrid_attn_prefill_fp8,
                                            ea_hybrid_attn_prefill_lse,
                                            ea_hybrid_attn_prefill_routed,
                                            ea_hybrid_attn_prefill_varlen, ea_quantize_fp8,
                                            ea_router_decide, make_decode_params, make_params)

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096          # elements on each side; a multiple of 16 bytes for every dtype used


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


class Guarded:
    """A tensor of `shape` in the middle of a buffer whose GUARD elements on
    either side hold a canary (on the device, or in pinned host memory)."""

    def __init__(self, shape, dtype, canary, device=DEV):
        self.n = math.prod(shape)
        self.buf = torch.full((GUARD + self.n + GUARD,), canary, dtype=dtype, device=device)
        if device == "cpu":
            self.buf = self.buf.pin_memory()
        self.canary = self.buf[:1].clone()
        self.t = self.buf[GUARD:GUARD + self.n].view(shape)

    def check(self, label):
        before, after = self.buf[:GUARD], self.buf[GUARD + self.n:]
        assert torch.equal(before, self.canary.expand_as(before)), f"{label}: write before"
        assert torch.equal(after, self.canary.expand_as(after)), f"{label}: write after"


def _finite(t, label):
    assert torch.isfinite(t.float()).all(), f"{label}: NaN or Inf in the output"


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("d,N", [(64, 300), (128, 300), (128, 1)])
def test_prefill_and_router(d, N):
    B, Hq, Hkv, S, W, hidden = 2, 4, 2, 16, 100, 32
    q, k, v = (_rand(s, d + N + i).to(DEV) for i, s in
               enumerate(((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d))))
    g = torch.Generator().manual_seed(5)
    w1 = (torch.randn((hidden, Hkv * d), generator=g) * 0.1).to(DEV)
    b1 = torch.zeros(hidden, device=DEV)
    w2 = torch.randn((Hq, hidden), generator=g).to(DEV)
    b2 = torch.zeros(Hq, device=DEV)
    mask = Guarded((B, Hq), torch.uint8, 0xA5)
    logits = Guarded((B, Hq), torch.float32, -777.0)
    ea_router_decide(k, w1, b1, w2, b2, route_mask=mask.t, logits=logits.t)
    out = Guarded((B, Hq, N, d), torch.bfloat16, -1000.0)
    ws = attn_workspace(make_params(B, Hq, Hkv, N, d, S, W), DEV)
    ea_hybrid_attn_prefill(q, k, v, mask.t, S, W, out=out.t, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    for gd, name in ((mask, "route mask"), (logits, "logits"), (out, "out")):
        gd.check(name)
    _finite(out.t, "out")
    # the routed one-launch path
    mask2 = Guarded((B, Hq), torch.uint8, 0x5A)
    out2 = Guarded((B, Hq, N, d), torch.bfloat16, -1000.0)
    ea_hybrid_attn_prefill_routed(q, k, v, w1, b1, w2, b2, S, W, route_mask=mask2.t,
                                  out=out2.t)
    torch.cuda.synchronize()
    mask2.check("routed mask")
    out2.check("routed out")
    assert torch.equal(out2.t, out.t)


def test_packed_batch():
    Hq, Hkv, d, S, W = 4, 2, 128, 8, 64
    lens = [1, 129, 300, 128]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    T = int(sum(lens))
    q, k, v = (_rand(s, 40 + i).to(DEV) for i, s in
               enumerate(((T, Hq, d), (T, Hkv, d), (T, Hkv, d))))
    mask = torch.tensor([[0, 1, 1, 0]] * len(lens), dtype=torch.uint8, device=DEV)
    out = Guarded((T, Hq, d), torch.bfloat16, -1000.0)
    ea_hybrid_attn_prefill_varlen(q, k, v, cu, mask, max(lens), S, W, out=out.t)
    torch.cuda.synchronize()
    out.check("packed out")
    _finite(out.t, "packed out")


def test_backward():
    B, Hq, Hkv, N, d, S, W = 1, 4, 2, 300, 128, 16, 100
    q, k, v, dout = (_rand(s, 60 + i).to(DEV) for i, s in
                     enumerate(((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, Hq, N, d))))
    mask = torch.tensor([[1, 0, 0, 1]], dtype=torch.uint8, device=DEV)
    o, lse = ea_hybrid_attn_prefill_lse(q, k, v, mask, S, W)
    dq = Guarded((B, Hq, N, d), torch.bfloat16, -1000.0)
    dk = Guarded((B, Hkv, N, d), torch.bfloat16, -1000.0)
    dv = Guarded((B, Hkv, N, d), torch.bfloat16, -1000.0)
    ea_hybrid_attn_backward(q, k, v, o, dout, lse, mask, S, W, dq=dq.t, dk=dk.t, dv=dv.t)
    torch.cuda.synchronize()
    for gd, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        gd.check(name)
        _finite(gd.t, name)


def test_fp8():
    B, Hq, Hkv, N, d, S, W = 1, 4, 2, 300, 128, 16, 100
    q, k, v = (_rand(s, 80 + i).to(DEV) for i, s in
               enumerate(((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d))))
    q8, qs = ea_quantize_fp8(q)
    k8, ks = ea_quantize_fp8(k)
    vt8, vs = ea_quantize_fp8(v, transpose=True)
    mask = torch.tensor([[0, 1, 1, 0]], dtype=torch.uint8, device=DEV)
    out = Guarded((B, Hq, N, d), torch.bfloat16, -1000.0)
    ea_hybrid_attn_prefill_fp8(q8, k8, vt8, qs, ks, vs, mask, S, W, out=out.t)
    torch.cuda.synchronize()
    out.check("fp8 out")
    _finite(out.t, "fp8 out")


def test_decode_step_and_caches():
    B, Hq, Hkv, d, S, W, max_len = 2, 8, 4, 128, 4, 100, 700
    mask = np.array([[1, 1, 0, 1, 1, 1, 0, 0], [0, 0, 1, 1, 1, 1, 1, 1]], dtype=np.uint8)
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    kf = Guarded((n_full, max_len, d), torch.bfloat16, 3.0)
    vf = Guarded((n_full, max_len, d), torch.bfloat16, 3.0)
    ks = Guarded((n_sa, S + W, d), torch.bfloat16, 3.0)
    vs = Guarded((n_sa, S + W, d), torch.bfloat16, 3.0)
    out = Guarded((B, Hq, d), torch.bfloat16, -1000.0)
    for t in (kf, vf, ks, vs):
        t.t.zero_()
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    pos = torch.tensor([max_len - 1, 250], dtype=torch.int32, device=DEV)
    q_t, k_t, v_t = (_rand(s, 90 + i).to(DEV) for i, s in
                     enumerate(((B, Hq, d), (B, Hkv, d), (B, Hkv, d))))
    ea_hybrid_attn_decode(q_t, k_t, v_t, pos, torch.as_tensor(mask, device=DEV),
                          torch.as_tensor(slots, dtype=torch.int32, device=DEV), kf.t, vf.t,
                          ks.t, vs.t, S, W, max_len, out=out.t, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    for gd, name in ((kf, "k_full"), (vf, "v_full"), (ks, "k_sa"), (vs, "v_sa"), (out, "out")):
        gd.check(name)
    _finite(out.t, "decode out")


def test_host_buffer_path():
    B, Hq, Hkv, N, d, S, W = 2, 8, 4, 300, 128, 16, 100
    q, k, v = (_rand(s, 100 + i).pin_memory() for i, s in
               enumerate(((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d))))
    mask = torch.tensor([[0, 1] * 4, [1, 1, 0, 0] * 2], dtype=torch.uint8)
    hp = HostPrefill(B, Hq, Hkv, N, d, None, None, None, None, S, W, device=DEV,
                     kv_heads_per_chunk=3)
    out = Guarded((B, Hq, N, d), torch.bfloat16, -1000.0, device="cpu")
    hp.out_host = out.t
    hp(q, k, v, mask)
    torch.cuda.synchronize()
    assert ea_get_device_status(hp.workspace) == 0
    out.check("host out")
    _finite(out.t, "host out")
