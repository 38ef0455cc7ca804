"""ea_router_decide_noalloc: the router for callers that cannot allocate
device memory when they route a layer, for instance a plug-in whose host
framework owns all device memory, or a serving loop that must not call
cudaMalloc/cudaFree after warm-up because those calls can synchronise the
device.  Its scratch is a fixed array inside libea.so.  It runs the same
kernels with the same split as ea_router_decide, so it must give the same
masks and the same logit bits, call after call, and masks equal to the
oracle's.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import (ea_router_decide, ea_router_decide_noalloc,
                                            ea_router_workspace_size)

from gpu_common import LOGIT_ABS, f64, margin_controlled_b2


def _inputs(seed, B=2, Hkv=8, N=4099, d=128, hidden=256, Hq=32):
    """Keys with a per-channel offset, so the pooled vector and the routing
    are data-driven; b2 margin-controlled by the oracle (every oracle logit at
    least 1e-3 from the threshold), so the masks are unique."""
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn((B, Hkv, N, d), generator=g) +
         torch.randn((1, Hkv, 1, d), generator=g)).to(torch.bfloat16)
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.05
    b1 = torch.randn((hidden,), generator=g) * 0.05
    w2 = torch.randn((Hq, hidden), generator=g) * 0.2
    b2 = torch.randn((Hq,), generator=g) * 0.1
    b2 = torch.as_tensor(margin_controlled_b2(f64(k), w1.double().numpy(), b1.double().numpy(),
                                              w2.double().numpy(), b2.double().numpy()),
                         dtype=torch.float32)
    return k, w1, b1, w2, b2


def test_noalloc_rejects_problems_beyond_its_scratch():
    build.build()
    lib = _lib.load()
    # B*Hkv*d*4 bytes > 1 MiB of scratch even with a single split per row;
    # the pointers are aligned stand-ins (nothing is launched)
    B, Hkv, N, d = 300, 8, 64, 128
    assert lib.ea_router_workspace_size(B, Hkv, N, d) > _lib.EA_ROUTER_NOALLOC_MAX_BYTES
    rc = lib.ea_router_decide_noalloc(16, B, Hkv, N, d, 16, 16, 256, 16, 16, 32, 0.0, 16, None,
                                      None)
    assert rc == _lib.EA_ERR_SCRATCH_LIMIT
    assert "no-allocation" in _lib.status_string(rc)


def test_noalloc_checks_arguments_before_the_scratch_limit():
    """The same codes as ea_router_decide for the same bad arguments, even when
    the problem is also too large for the scratch."""
    lib = _lib.load()
    B, Hkv, N, d = 300, 8, 64, 128
    cases = [
        (dict(k=None), _lib.EA_ERR_INVALID_ARG),
        (dict(w1=None), _lib.EA_ERR_INVALID_ARG),
        (dict(mask=None), _lib.EA_ERR_INVALID_ARG),
        (dict(d=96), _lib.EA_ERR_UNSUPPORTED),
        (dict(hidden=8192), _lib.EA_ERR_UNSUPPORTED),
        (dict(k=24), _lib.EA_ERR_MISALIGNED),
        (dict(threshold=float("nan")), _lib.EA_ERR_INVALID_ARG),
    ]
    for over, code in cases:
        a = dict(k=16, B=B, Hkv=Hkv, N=N, d=d, w1=16, b1=16, hidden=256, w2=16, b2=16, Hq=32,
                 threshold=0.0, mask=16)
        a.update(over)
        args = (a["k"], a["B"], a["Hkv"], a["N"], a["d"], a["w1"], a["b1"], a["hidden"],
                a["w2"], a["b2"], a["Hq"], a["threshold"], a["mask"], None)
        got = lib.ea_router_decide_noalloc(*args, None)
        ref = lib.ea_router_decide(*args, 16, 1 << 40, None)
        assert got == code == ref, (over, got, ref)


def test_noalloc_wrapper_checks_shapes_before_touching_memory():
    k = torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16)
    w1, b1 = torch.zeros((16, 128)), torch.zeros(16)
    w2, b2 = torch.zeros((4, 16)), torch.zeros(4)
    mask = torch.zeros((1, 4), dtype=torch.uint8)
    with pytest.raises(ValueError, match="weight shapes"):
        ea_router_decide_noalloc(k, torch.zeros((16, 64)), b1, w2, b2, route_mask=mask)
    with pytest.raises(ValueError, match="weight shapes"):
        ea_router_decide_noalloc(k, w1, b1, torch.zeros((4, 8)), b2, route_mask=mask)
    with pytest.raises(ValueError, match="route_mask"):
        ea_router_decide_noalloc(k, w1, b1, w2, b2, route_mask=torch.zeros((1, 3),
                                                                          dtype=torch.uint8))
    with pytest.raises(ValueError, match="logits"):
        ea_router_decide_noalloc(k, w1, b1, w2, b2, route_mask=mask, logits=torch.zeros(4))
    # right shapes, host memory: refused before any library call
    with pytest.raises(ValueError, match="CUDA"):
        ea_router_decide_noalloc(k, w1, b1, w2, b2, route_mask=mask)


@pytest.mark.gpu
def test_noalloc_router_matches_workspace_router_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    for seed in (1, 2):     # two calls in a row, different inputs
        k_h, w1_h, b1_h, w2_h, b2_h = _inputs(seed)
        k, w1, b1, w2, b2 = (t.to(dev) for t in (k_h, w1_h, b1_h, w2_h, b2_h))
        B, Hkv, N, d = k.shape
        Hq = w2.shape[0]
        assert ea_router_workspace_size(B, Hkv, N, d) <= _lib.EA_ROUTER_NOALLOC_MAX_BYTES
        ref_mask, ref_z = ea_router_decide(k, w1, b1, w2, b2)
        # through the C ABI directly
        mask = torch.full((B, Hq), 7, dtype=torch.uint8, device=dev)
        z = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        rc = lib.ea_router_decide_noalloc(k.data_ptr(), B, Hkv, N, d, w1.data_ptr(),
                                          b1.data_ptr(), w1.shape[0], w2.data_ptr(),
                                          b2.data_ptr(), Hq, 0.0, mask.data_ptr(), z.data_ptr(),
                                          ctypes.c_void_p(int(stream.cuda_stream)))
        assert rc == _lib.EA_OK, _lib.status_string(rc)
        # and through the Python wrapper
        mask2 = torch.full((B, Hq), 7, dtype=torch.uint8, device=dev)
        z2 = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        ea_router_decide_noalloc(k, w1, b1, w2, b2, route_mask=mask2, logits=z2)
        torch.cuda.synchronize()
        # same kernels, same split: the same bits as the workspace router
        np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask.cpu().numpy())
        np.testing.assert_array_equal(z.cpu().numpy().view(np.uint32),
                                      ref_z.cpu().numpy().view(np.uint32))
        np.testing.assert_array_equal(mask2.cpu().numpy(), mask.cpu().numpy())
        np.testing.assert_array_equal(z2.cpu().numpy().view(np.uint32),
                                      z.cpu().numpy().view(np.uint32))
        # and the oracle's decisions (margin-controlled, so unique)
        mask_ref, z_ref = oracle.router_decide(f64(k_h), w1_h.double().numpy(),
                                               b1_h.double().numpy(), w2_h.double().numpy(),
                                               b2_h.double().numpy())
        np.testing.assert_array_equal(mask.cpu().numpy(), mask_ref)
        assert np.abs(z.cpu().double().numpy() - z_ref).max() <= LOGIT_ABS
        assert 0 < int(mask.sum()) < mask.numel()


@pytest.mark.gpu
def test_noalloc_refuses_host_memory():
    """A host pointer for the keys is refused before anything is enqueued."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    k_host = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16)
    w1, b1 = torch.zeros((16, 128), device=dev), torch.zeros(16, device=dev)
    w2, b2 = torch.zeros((4, 16), device=dev), torch.zeros(4, device=dev)
    mask = torch.zeros((1, 4), dtype=torch.uint8, device=dev)
    rc = lib.ea_router_decide_noalloc(k_host.data_ptr(), 1, 2, 64, 64, w1.data_ptr(),
                                      b1.data_ptr(), 16, w2.data_ptr(), b2.data_ptr(), 4, 0.0,
                                      mask.data_ptr(), None, None)
    assert rc == _lib.EA_ERR_INVALID_ARG
