"""ea_router_decide_noalloc: the router for callers that cannot allocate
device memory when they route a layer, for instance a plug-in whose host
framework owns all device memory, or a serving loop that must not call
cudaMalloc/cudaFree after warm-up because those calls can synchronise the
device.  Its scratch is a fixed array inside libea.so, so it must give the
same masks and logits as ea_router_decide with a caller workspace, call after
call.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import ea_router_decide, ea_router_workspace_size

LOGIT_ABS = 1e-4     # the router logit tolerance used by the other GPU tests


def _inputs(seed, B=2, Hkv=8, N=4099, d=128, hidden=256, Hq=32):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn((B, Hkv, N, d), generator=g) + torch.randn((1, Hkv, 1, d), generator=g))
    w1 = torch.randn((hidden, Hkv * d), generator=g) * 0.05
    b1 = torch.randn((hidden,), generator=g) * 0.05
    w2 = torch.randn((Hq, hidden), generator=g) * 0.2
    b2 = torch.randn((Hq,), generator=g) * 0.1
    return k.to(torch.bfloat16), w1, b1, w2, b2


def test_noalloc_rejects_problems_beyond_its_scratch():
    build.build()
    lib = _lib.load()
    # B*Hkv*d*4 bytes > 1 MiB of scratch even with a single split per row
    B, Hkv, N, d = 300, 8, 64, 128
    assert lib.ea_router_workspace_size(B, Hkv, N, d) > _lib.EA_ROUTER_NOALLOC_MAX_BYTES
    rc = lib.ea_router_decide_noalloc(16, B, Hkv, N, d, 16, 16, 256, 16, 16, 32, 0.0, 16, None,
                                      None)
    assert rc == _lib.EA_ERR_SCRATCH_LIMIT
    assert "no-allocation" in _lib.status_string(rc)


@pytest.mark.gpu
def test_noalloc_router_matches_workspace_router_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    for seed in (1, 2):     # two calls in a row, different inputs
        k, w1, b1, w2, b2 = (t.to(dev) for t in _inputs(seed))
        B, Hkv, N, d = k.shape
        Hq = w2.shape[0]
        assert ea_router_workspace_size(B, Hkv, N, d) <= _lib.EA_ROUTER_NOALLOC_MAX_BYTES
        ref_mask, ref_z = ea_router_decide(k, w1, b1, w2, b2)
        mask = torch.full((B, Hq), 7, dtype=torch.uint8, device=dev)
        z = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
        rc = lib.ea_router_decide_noalloc(k.data_ptr(), B, Hkv, N, d, w1.data_ptr(),
                                          b1.data_ptr(), w1.shape[0], w2.data_ptr(),
                                          b2.data_ptr(), Hq, 0.0, mask.data_ptr(), z.data_ptr(),
                                          ctypes.c_void_p(int(stream.cuda_stream)))
        assert rc == _lib.EA_OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(mask.cpu().numpy(), ref_mask.cpu().numpy())
        np.testing.assert_allclose(z.cpu().numpy(), ref_z.cpu().numpy(), rtol=0, atol=LOGIT_ABS)
        assert 0 < int(mask.sum()) < mask.numel()
