"""Parity at the full workload sizes, in the launch configuration bench.py
times: every router mask is compared in full (bit-exact) and attention rows
are sampled per head (special rows near the sink/window/tile edges plus
seeded random rows), each computed one by one by the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import LOGIT_ABS, MARGIN, compare, f64, sample_rows
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
                                            ea_hybrid_attn_prefill, ea_router_decide,
                                            make_params)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _layer(w, layer, heads_to_check, n_random):
    seed = workloads.layer_seed(w, layer)
    q, k, v = workloads.make_qkv(w, seed, device=DEV)
    kf = f64(k)
    if w.use_router:
        frac = workloads.layer_sparse_frac(w, layer)
        sheads = workloads.sparse_head_set(w.hq, frac, seed)
        w1, b1, w2, b2 = workloads.make_router_weights(w.hkv * w.d, w.router_hidden, w.hq,
                                                       sheads, seed)
        ref_mask, z_ref = oracle.router_decide(kf, w1.double().numpy(), b1.double().numpy(),
                                               w2.double().numpy(), b2.double().numpy())
        assert np.min(np.abs(z_ref)) >= MARGIN
        mask, z = ea_router_decide(k, w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask)
        np.testing.assert_allclose(f64(z), z_ref, rtol=0, atol=LOGIT_ABS)
        # the chosen heads route sparse, the others full
        want = np.zeros((w.batch, w.hq), np.uint8)
        want[:, sheads] = 1
        np.testing.assert_array_equal(ref_mask, want)
    else:
        mask = workloads.make_fixed_mask(w, seed).to(DEV)
        ref_mask = mask.cpu().numpy()
    p = make_params(w.batch, w.hq, w.hkv, w.seq, w.d, w.sink, w.window)
    ws = attn_workspace(p, DEV)
    out = ea_hybrid_attn_prefill(q, k, v, mask, w.sink, w.window, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    qf, vf = f64(q), f64(v)
    for (b, h) in heads_to_check(ref_mask):
        rows = sample_rows(w.seq, w.sink, w.window, n_random, seed=1000 * b + h)
        ref = oracle.attention_rows(qf, kf, vf, ref_mask, b, h, rows, w.sink, w.window)
        compare(out[b, h, rows], ref, f"{w.name} layer {layer} b{b} h{h}")
    return ref_mask


def _some_heads(k_fa, k_sa):
    def pick(m):
        out = []
        for b in range(m.shape[0]):
            fa = [h for h in range(m.shape[1]) if not m[b, h]][:k_fa]
            sa = [h for h in range(m.shape[1]) if m[b, h]][:k_sa]
            out += [(b, h) for h in fa + sa]
        return out
    return pick


def test_llama8b_layer():
    w = workloads.get("llama8b")
    m = _layer(w, 0, lambda m: [(0, h) for h in range(w.hq)], 24)
    assert int(m.sum()) == 22


def test_qwen4b_layer():
    w = workloads.get("qwen4b")
    m = _layer(w, 0, _some_heads(2, 3), 24)
    assert all(int(m[b].sum()) == 27 for b in range(w.batch))


def test_qwen8b36_two_layers():
    w = workloads.get("qwen8b36")
    for layer in (0, 17):
        m = _layer(w, layer, _some_heads(1, 2), 16)
        frac = workloads.layer_sparse_frac(w, layer)
        assert int(m[0].sum()) == int(round(frac * w.hq))


def test_ext256k_layer():
    w = workloads.get("ext256k")
    m = _layer(w, 0, _some_heads(2, 2), 12)
    assert int(m.sum()) == 24
