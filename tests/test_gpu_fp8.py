"""GPU: the FP8 (e4m3) variant through the C ABI.  Quantization is byte work
and must equal the oracle's bit for bit; the attention is compared with the
oracle's attention of the dequantized inputs (quantized by the oracle itself)
within the bound of rounding the probabilities to e4m3
(oracle.fp8_p_rounding_bound), plus the bf16 rounding of the output (2^-8 of
it) and 1e-3 for the fp32 arithmetic around it."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import f64
from sparse_attention_head_b200 import build
from sparse_attention_head_b200.api import (EA_SELECT_ALL, EA_SELECT_FA, EA_SELECT_SA,
                                            ea_fp8_vt_stride, ea_get_device_status,
                                            ea_hybrid_attn_prefill_fp8, ea_quantize_fp8)

pytestmark = pytest.mark.gpu

DEV = "cuda"
SLACK_ABS = 1e-3
OUT_REL = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _bf16(shape, seed, mult=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * mult).to(torch.bfloat16)


@pytest.mark.parametrize("B,H,N", [(1, 2, 300), (2, 3, 77), (1, 1, 1030), (1, 2, 16)])
def test_quantize_matches_oracle_bitwise(B, H, N):
    x = _bf16((B, H, N, 128), seed=N, mult=3.0)
    x[0, 0, : min(N, 5)] *= 40.0                        # a head with outliers
    if H > 2:
        x[-1, 2] = 0.0                                  # an all-zero head
    ref_codes, ref_scale = oracle.quantize_e4m3_per_head(x.float().numpy())
    codes, scale = ea_quantize_fp8(x.to(DEV))
    codes_t, scale_t = ea_quantize_fp8(x.to(DEV), transpose=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_scale)
    np.testing.assert_array_equal(scale_t.cpu().numpy(), ref_scale)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    npad = ea_fp8_vt_stride(N)
    assert codes_t.shape == (B, H, 128, npad)
    ct = codes_t.cpu().numpy()
    np.testing.assert_array_equal(ct[..., :N], ref_codes.transpose(0, 1, 3, 2))
    assert not ct[..., N:].any()


def _case(B, Hq, Hkv, N, seed):
    q = _bf16((B, Hq, N, 128), seed)
    k = _bf16((B, Hkv, N, 128), seed + 1)
    v = _bf16((B, Hkv, N, 128), seed + 2)
    return q, k, v


def _run_fp8(q, k, v, mask, S, W, select=EA_SELECT_ALL, out=None):
    q8, qs = ea_quantize_fp8(q.to(DEV))
    k8, ks = ea_quantize_fp8(k.to(DEV))
    vt8, vs = ea_quantize_fp8(v.to(DEV), transpose=True)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    o = ea_hybrid_attn_prefill_fp8(q8, k8, vt8, qs, ks, vs, torch.as_tensor(mask, device=DEV), S,
                                   W, select=select, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    return o


def _oracle_fp8(q, k, v, mask, S, W):
    (qc, qs), (kc, ks), (vc, vs) = (oracle.quantize_e4m3_per_head(t.float().numpy())
                                    for t in (q, k, v))
    qd, kd, vd = (oracle.dequantize_e4m3(c, s) for c, s in ((qc, qs), (kc, ks), (vc, vs)))
    ref = oracle.attention_fp8(qc, qs, kc, ks, vc, vs, mask, S, W)
    bound = oracle.fp8_p_rounding_bound(qd, kd, vd, mask, S, W)
    return ref, bound


CASES = [
    # B, Hq, Hkv, N, S, W
    (1, 4, 2, 640, 16, 128),
    (2, 8, 2, 300, 0, 37),          # ragged N (not a multiple of 16), no sinks
    (1, 2, 1, 1030, 64, 256),       # MQA, sinks span a tile
    (1, 2, 2, 17, 4, 8),            # a single short tile
]


@pytest.mark.parametrize("B,Hq,Hkv,N,S,W", CASES)
def test_fp8_attention_within_the_rounding_bound(B, Hq, Hkv, N, S, W):
    q, k, v = _case(B, Hq, Hkv, N, seed=N + S)
    rng = np.random.default_rng(N)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    mask[0, 0], mask[-1, -1] = 0, 1
    out = _run_fp8(q, k, v, mask, S, W)
    ref, bound = _oracle_fp8(q, k, v, mask, S, W)
    err = np.abs(f64(out) - ref)
    tol = bound + OUT_REL * np.abs(ref) + SLACK_ABS
    bad = err > tol
    assert not bad.any(), (int(bad.sum()), float(err.max()), float(tol[bad].min()))
    # far from the worst case on random data
    assert err.mean() < 0.25 * bound.mean()


@pytest.mark.parametrize("select", [EA_SELECT_FA, EA_SELECT_SA])
def test_fp8_select_leaves_other_heads_untouched(select):
    B, Hq, Hkv, N, S, W = 1, 4, 2, 384, 8, 64
    q, k, v = _case(B, Hq, Hkv, N, seed=5)
    mask = np.array([[0, 1, 1, 0]], np.uint8)
    sentinel = torch.full((B, Hq, N, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    out = _run_fp8(q, k, v, mask, S, W, select=select, out=sentinel)
    ref, bound = _oracle_fp8(q, k, v, mask, S, W)
    got = f64(out)
    for h in range(Hq):
        if (select == EA_SELECT_SA) == bool(mask[0, h]):
            tol = bound[0, h] + OUT_REL * np.abs(ref[0, h]) + SLACK_ABS
            assert np.all(np.abs(got[0, h] - ref[0, h]) <= tol)
        else:
            assert np.all(got[0, h] == 7.0)


def test_fp8_llama8b_layer_sampled_rows():
    """The llama8b layer (B1 N32768 Hq32 Hkv8 d128, S64 W1024, the router's
    22 SA heads) in the configuration the FP8 bench line times: the oracle
    quantizes the checked heads itself (bytes equal to the GPU's) and checks
    sampled rows of two FA and two SA heads one by one."""
    import workloads
    from gpu_common import sample_rows
    w = workloads.get("llama8b")
    seed = workloads.layer_seed(w, 0)
    q, k, v = workloads.make_qkv(w, seed, device=DEV)
    sheads = workloads.sparse_head_set(w.hq, workloads.layer_sparse_frac(w, 0), seed)
    mask = np.zeros((1, w.hq), np.uint8)
    mask[0, sheads] = 1
    q8, qs = ea_quantize_fp8(q)
    k8, ks = ea_quantize_fp8(k)
    vt8, vs = ea_quantize_fp8(v, transpose=True)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    out = ea_hybrid_attn_prefill_fp8(q8, k8, vt8, qs, ks, vs, torch.as_tensor(mask, device=DEV),
                                     w.sink, w.window, workspace=ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    g = w.hq // w.hkv
    fa = [h for h in range(w.hq) if not mask[0, h]][:2]
    sa = [h for h in range(w.hq) if mask[0, h]][:2]
    for h in fa + sa:
        hk = h // g
        (qc, qsc), (kc, ksc), (vc, vsc) = (
            oracle.quantize_e4m3_per_head(t[0:1, hh:hh + 1].float().cpu().numpy())
            for t, hh in ((q, h), (k, hk), (v, hk)))
        np.testing.assert_array_equal(q8[0:1, h:h + 1].cpu().numpy(), qc)
        np.testing.assert_array_equal(k8[0:1, hk:hk + 1].cpu().numpy(), kc)
        np.testing.assert_array_equal(qs[0, h].item(), qsc[0, 0])
        qd, kd, vd = (oracle.dequantize_e4m3(c, s) for c, s in ((qc, qsc), (kc, ksc), (vc, vsc)))
        m1 = mask[:, h:h + 1]
        rows = sample_rows(w.seq, w.sink, w.window, 16, seed=h)
        ref = oracle.attention_rows(qd, kd, vd, m1, 0, 0, rows, w.sink, w.window)
        bound = oracle.fp8_p_rounding_bound_rows(qd, kd, vd, m1, 0, 0, rows, w.sink, w.window)
        err = np.abs(f64(out[0, h, rows]) - ref)
        tol = bound + OUT_REL * np.abs(ref) + SLACK_ABS
        assert np.all(err <= tol), (h, float(err.max()), float((err - tol).max()))
