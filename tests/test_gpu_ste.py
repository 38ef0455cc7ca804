"""GPU: router training through the C ABI against the oracle -- the
Gumbel-Softmax decision (hard routes bit-exact, soft routes within the
logits' bound) and the straight-through gradients of the router's weights and
of the keys through the pooling.

Tolerances.  Everything on the GPU is fp32 (unit roundoff u = 2^-24).  The
longest chain of dependent additions in any reduction here stays below
2^10 at these sizes (the dr reduction: about N*d / (splits * 256) products
per thread, then 5 shuffle levels, 8 warps and the splits), so by the
standard summation bound each fp32 reduction is within 2^10 u = 2^-14 of the
sum of its terms' magnitudes.  The logits carry the router's own bound
LOGIT_ABS, which moves u = (z + g1 - g0) / tau by LOGIT_ABS / tau and so
r (1 - r) by at most that much relatively.  A gradient G = A^T B built from
dz is therefore compared elementwise against EPS * (|A|^T |B|) with
EPS = 4 (2^-14 + LOGIT_ABS / tau): the componentwise matmul error bound with
a factor 4 for the chained stages."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import LOGIT_ABS, f64
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import ea_router_decide, ea_router_decide_gumbel, \
    ea_router_ste_backward

pytestmark = pytest.mark.gpu

DEV = "cuda"
SUM_REL = 2.0 ** -14


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _inputs(B, Hkv, N, d, Hq, hidden, seed, mix=False):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((B, Hkv, N, d), generator=g)
    k += torch.randn((B, Hkv, 1, d), generator=g)          # per-sequence offsets
    k = k.to(torch.bfloat16)
    w1 = (torch.randn((hidden, Hkv * d), generator=g) * 0.05).float()
    b1 = (torch.randn((hidden,), generator=g) * 0.1).float()
    w2 = (torch.randn((Hq, hidden), generator=g) * 0.05).float()
    b2 = (torch.randn((Hq,), generator=g) * 0.05).float()
    # keep every ReLU input clear of zero so both sides gate the same units
    x = oracle.router_pool(f64(k))
    pre = x @ w1.double().numpy().T + b1.double().numpy()
    for j in range(hidden):
        while np.abs(pre[:, j]).min() < 1e-3:
            b1[j] += 2e-3
            pre[:, j] += float(np.float32(2e-3))
    # Gumbel noise g = -log(-log U); pushed so |z + g1 - g0| clears the
    # logits' bound and both sides take the same hard decision
    U = torch.rand((2, B, Hq), generator=g, dtype=torch.float64).clamp(1e-12, 1 - 1e-12)
    gum = (-torch.log(-torch.log(U))).float()
    g0, g1 = gum[0].clone(), gum[1].clone()
    _, _, z = oracle.router_gumbel_forward(f64(k), w1.double().numpy(), b1.double().numpy(),
                                           w2.double().numpy(), b2.double().numpy(),
                                           g0.double().numpy(), g1.double().numpy(), 1.0)
    u = z + g1.double().numpy() - g0.double().numpy()
    close = np.abs(u) < 20 * LOGIT_ABS
    g1[torch.as_tensor(close)] += torch.as_tensor(np.where(u[close] >= 0, 1e-2, -1e-2),
                                                  dtype=torch.float32)
    if mix:     # head 0 of the first sequence to SA, head 1 to FA
        g1[0, 0] = float(g0[0, 0] - z[0, 0] + 1.0)
        g1[0, 1] = float(g0[0, 1] - z[0, 1] - 1.0)
    return k, w1, b1, w2, b2, g0, g1


def _np(*ts):
    return [t.double().numpy() for t in ts]


SHAPES = [
    # B, Hkv, N, d, Hq, hidden, tau
    (2, 2, 300, 128, 8, 64, 1.0),
    (3, 4, 77, 64, 4, 32, 0.5),                 # ragged N, d = 64, more splits than work
    (1, 8, 2048, 128, 32, 256, 1.0),            # llama8b layer shape
]


@pytest.mark.parametrize("B,Hkv,N,d,Hq,hidden,tau", SHAPES)
def test_gumbel_decision_matches_oracle(B, Hkv, N, d, Hq, hidden, tau):
    k, w1, b1, w2, b2, g0, g1 = _inputs(B, Hkv, N, d, Hq, hidden, seed=N + d)
    dev = [t.to(DEV) for t in (k, w1, b1, w2, b2, g0, g1)]
    r_hard, r_soft, z = ea_router_decide_gumbel(*dev, tau)
    torch.cuda.synchronize()
    ref_hard, ref_soft, ref_z = oracle.router_gumbel_forward(f64(k), *_np(w1, b1, w2, b2, g0, g1),
                                                             tau)
    np.testing.assert_array_equal(r_hard.cpu().numpy(), ref_hard)
    assert np.abs(z.cpu().double().numpy() - ref_z).max() <= LOGIT_ABS
    # d r / d z <= 1 / (4 tau): the logits' bound moves r by LOGIT_ABS / (4 tau)
    assert np.abs(r_soft.cpu().double().numpy() - ref_soft).max() <= LOGIT_ABS / (4 * tau) + 1e-6
    # the logits are the router's, bit for bit
    _, z_plain = ea_router_decide(dev[0], *dev[1:5])
    assert torch.equal(z, z_plain)


@pytest.mark.parametrize("B,Hkv,N,d,Hq,hidden,tau", SHAPES)
def test_ste_backward_matches_oracle(B, Hkv, N, d, Hq, hidden, tau):
    k, w1, b1, w2, b2, g0, g1 = _inputs(B, Hkv, N, d, Hq, hidden, seed=N + d + 1)
    g = torch.Generator().manual_seed(N)
    dout, o_fa, o_sa = (torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
                        for _ in range(3))
    dk_before = (torch.randn((B, Hkv, N, d), generator=g) * 0.01).to(torch.bfloat16)
    dk_accum = dk_before.to(DEV)
    dev = [t.to(DEV) for t in (k, w1, b1, w2, b2, g0, g1)]
    dr, dw1, db1, dw2, db2, dk_pool = ea_router_ste_backward(
        *dev, tau, dout.to(DEV), o_fa.to(DEV), o_sa.to(DEV), dk_accum=dk_accum)
    torch.cuda.synchronize()
    W1, B1, W2, B2, G0, G1 = _np(w1, b1, w2, b2, g0, g1)
    r_dr, r_dz, r_dw1, r_db1, r_dw2, r_db2, r_dk = oracle.router_ste_backward(
        f64(k), W1, B1, W2, B2, G0, G1, tau, f64(dout), f64(o_fa), f64(o_sa))
    # dr: one fp32 reduction of N*d products
    terms = np.sum(np.abs(f64(dout) * (f64(o_sa) - f64(o_fa))), axis=(2, 3))
    assert np.all(np.abs(dr.cpu().double().numpy() - r_dr) <= SUM_REL * terms)
    # the rest: componentwise bounds built from absolute values
    eps = 4 * (SUM_REL + LOGIT_ABS / tau)
    x = oracle.router_pool(f64(k))
    pre = x @ W1.T + B1
    h = np.maximum(pre, 0.0)
    adz = np.abs(r_dz) + SUM_REL * terms * 0.25 / tau
    adpre = np.where(pre > 0, adz @ np.abs(W2), 0.0)
    checks = [("dw2", dw2, r_dw2, adz.T @ h), ("db2", db2, r_db2, adz.sum(0)),
              ("dw1", dw1, r_dw1, adpre.T @ np.abs(x)), ("db1", db1, r_db1, adpre.sum(0)),
              ("dk_pool", dk_pool, r_dk[:, :, 0, :].reshape(B, Hkv * d),
               (adpre @ np.abs(W1)) / N)]
    for name, got, ref, mag in checks:
        err = np.abs(got.cpu().double().numpy() - ref)
        bad = err > eps * mag + 1e-30
        assert not bad.any(), (name, float(err.max()), float((eps * mag)[bad].min()))
    assert np.abs(r_dz).max() > 0                          # the gradients are not trivial
    # dk_accum: the attention's dk plus the pooled share, rounded once to bf16
    want = (dk_before.float() + dk_pool.cpu().view(B, Hkv, 1, d)).to(torch.bfloat16)
    assert torch.equal(dk_accum.cpu(), want)


def test_ste_backward_is_deterministic():
    B, Hkv, N, d, Hq, hidden, tau = 2, 8, 1500, 128, 32, 256, 1.0
    k, w1, b1, w2, b2, g0, g1 = _inputs(B, Hkv, N, d, Hq, hidden, seed=3)
    g = torch.Generator().manual_seed(4)
    dout, o_fa, o_sa = (torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16).to(DEV)
                        for _ in range(3))
    dev = [t.to(DEV) for t in (k, w1, b1, w2, b2, g0, g1)]
    a = ea_router_ste_backward(*dev, tau, dout, o_fa, o_sa)
    b = ea_router_ste_backward(*dev, tau, dout, o_fa, o_sa)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- a training step
from gpu_common import compare  # noqa: E402
from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_backward,  # noqa: E402
                                            ea_hybrid_attn_prefill,
                                            ea_hybrid_attn_prefill_lse,
                                            ea_hybrid_attn_prefill_train)

LSE_ABS = 4.0e-3          # as for the forward's log-sum-exp (bf16 row-sum terms)


@pytest.mark.parametrize("B,Hq,Hkv,N,S,W", [(2, 8, 2, 640, 16, 128), (1, 4, 4, 300, 0, 37)])
def test_training_step_composes(B, Hq, Hkv, N, S, W):
    """Gumbel decision -> both-mode forward -> attention backward -> router
    gradients through the straight-through estimator, all on the GPU."""
    d, hidden, tau = 128, 64, 1.0
    k, w1, b1, w2, b2, g0, g1 = _inputs(B, Hkv, N, d, Hq, hidden, seed=N + S, mix=True)
    g = torch.Generator().manual_seed(N + 1)
    q = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g).to(torch.bfloat16)
    dout = torch.randn((B, Hq, N, d), generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), dout.to(DEV)
    rw = [t.to(DEV) for t in (w1, b1, w2, b2, g0, g1)]
    mask, _, _ = ea_router_decide_gumbel(kd, *rw, tau)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    out, lse, other = ea_hybrid_attn_prefill_train(qd, kd, vd, mask, S, W, workspace=ws[:256])
    torch.cuda.synchronize()
    assert ea_get_device_status(ws[:256]) == 0
    hm = mask.cpu().numpy()
    assert 0 < hm.sum() < hm.size, "the step should mix both modes"
    # each mode is the single-mode kernel's result, bit for bit
    out1, lse1 = ea_hybrid_attn_prefill_lse(qd, kd, vd, mask, S, W)
    other1 = ea_hybrid_attn_prefill(qd, kd, vd, (1 - mask).contiguous(), S, W)
    assert torch.equal(out, out1) and torch.equal(lse, lse1) and torch.equal(other, other1)
    # and against the oracle
    qf, kf, vf = f64(q), f64(k), f64(v)
    compare(out, oracle.attention(qf, kf, vf, hm, S, W), "train chosen mode")
    compare(other, oracle.attention(qf, kf, vf, 1 - hm, S, W), "train other mode")
    assert np.abs(f64(lse) - oracle.attention_lse(qf, kf, hm, S, W)).max() <= LSE_ABS
    # attention backward of the chosen mode, then the router's share added to dk
    dq, dk, dv = ea_hybrid_attn_backward(qd, kd, vd, out, dod, lse, mask, S, W, workspace=ws)
    dk_attn = dk.clone()
    grads = ea_router_ste_backward(kd, *rw, tau, dod, out, other, mask, dk_accum=dk)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    # the training layout gives exactly what the (O_FA, O_SA) layout gives
    m4 = mask.bool()[:, :, None, None]
    o_fa, o_sa = torch.where(m4, other, out), torch.where(m4, out, other)
    plain = ea_router_ste_backward(kd, *rw, tau, dod, o_fa, o_sa)
    torch.cuda.synchronize()
    for a, b in zip(grads, plain):
        assert torch.equal(a, b)
    want = (dk_attn.float() + grads[5].view(B, Hkv, 1, d)).to(torch.bfloat16)
    assert torch.equal(dk, want)
    # the router gradients against the oracle, on the GPU's own outputs
    r_dr, r_dz, r_dw1, r_db1, r_dw2, r_db2, r_dk = oracle.router_ste_backward(
        f64(k), *_np(w1, b1, w2, b2, g0, g1), tau, f64(dout), f64(o_fa), f64(o_sa))
    terms = np.sum(np.abs(f64(dout) * (f64(o_sa) - f64(o_fa))), axis=(2, 3))
    assert np.all(np.abs(grads[0].cpu().double().numpy() - r_dr) <= SUM_REL * terms)
    eps = 4 * (SUM_REL + LOGIT_ABS / tau)
    scale = np.abs(r_dw2).max()
    assert np.abs(grads[3].cpu().double().numpy() - r_dw2).max() <= eps * 4 * scale
