"""The C-ABI library loads, exports every symbol include/ea.h declares, and
rejects bad arguments before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import make_params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ea.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(ea_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("ea_router_decide", "ea_hybrid_attn_prefill", "ea_status_string",
                 "ea_router_workspace_size", "ea_hybrid_attn_workspace_size",
                 "ea_get_device_status"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTED)
    for n in names:
        assert hasattr(lib, n), f"libea.so does not export {n}"


def test_library_is_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH_FLAGS)
    assert os.path.exists(_lib.LIB_PATH)


def test_status_strings(lib):
    for code in range(0, 7):
        s = _lib.status_string(code)
        assert isinstance(s, str) and s
    assert _lib.status_string(5) == "device wait timed out"
    assert _lib.status_string(99) == "unknown status"
    assert lib.ea_version() >> 16 == 1


def _attn(lib, p, q=16, k=16, v=16, mask=16, out=16, ws=256, wsbytes=256):
    return lib.ea_hybrid_attn_prefill(q, k, v, mask, ctypes.byref(p), out, ws, wsbytes, None)


def test_attention_argument_errors(lib):
    good = make_params(1, 4, 2, 512, 64, 16, 128)
    cases = [
        (make_params(0, 4, 2, 512, 64, 16, 128), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 3, 512, 64, 16, 128), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 2, 0, 64, 16, 128), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 2, 512, 64, -1, 128), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 2, 512, 64, 16, 0), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 2, 512, 64, 16, 128, select=3), {}, _lib.EA_ERR_INVALID_ARG),
        (make_params(1, 4, 2, 512, 96, 16, 128), {}, _lib.EA_ERR_UNSUPPORTED),
        (make_params(2, 4096, 4096, 512, 64, 16, 128), {}, _lib.EA_ERR_UNSUPPORTED),
        (make_params(1, 4, 2, 512, 64, 16, 128, softmax_scale=float("nan")), {},
         _lib.EA_ERR_INVALID_ARG),
        (good, {"q": 0}, _lib.EA_ERR_INVALID_ARG),
        (good, {"mask": 0}, _lib.EA_ERR_INVALID_ARG),
        (good, {"out": 0}, _lib.EA_ERR_INVALID_ARG),
        (good, {"k": 24}, _lib.EA_ERR_MISALIGNED),
        (good, {"out": 8}, _lib.EA_ERR_MISALIGNED),
        (good, {"ws": 0}, _lib.EA_ERR_WORKSPACE),
        (good, {"wsbytes": 4}, _lib.EA_ERR_WORKSPACE),
    ]
    for p, kw, want in cases:
        assert _attn(lib, p, **kw) == want, (p.B, p.Hq, p.Hkv, p.N, p.d, kw)
    assert lib.ea_hybrid_attn_prefill(16, 16, 16, 16, None, 16, 16, 256, None) == \
        _lib.EA_ERR_INVALID_ARG


def test_traced_prefill_argument_errors(lib):
    """The traced entry point's own checks (trace buffer, record count), then
    the untraced call's; every case returns before any CUDA call."""
    good = make_params(1, 4, 2, 512, 64, 16, 128)

    def traced(p, trace=256, records=8, q=16, ws=256, wsbytes=256):
        return lib.ea_hybrid_attn_prefill_traced(q, 16, 16, 16, ctypes.byref(p), 16, ws, wsbytes,
                                                 trace, records, None)
    assert traced(good, trace=None) == _lib.EA_ERR_INVALID_ARG
    assert traced(good, records=-1) == _lib.EA_ERR_INVALID_ARG
    assert traced(good, trace=260) == _lib.EA_ERR_MISALIGNED      # 4-byte aligned only
    assert traced(make_params(0, 4, 2, 512, 64, 16, 128)) == _lib.EA_ERR_INVALID_ARG
    assert traced(make_params(1, 4, 2, 512, 96, 16, 128)) == _lib.EA_ERR_UNSUPPORTED
    assert traced(good, q=0) == _lib.EA_ERR_INVALID_ARG
    assert traced(good, q=24) == _lib.EA_ERR_MISALIGNED
    assert traced(good, wsbytes=4) == _lib.EA_ERR_WORKSPACE


def test_workspace_sizes(lib):
    p = make_params(1, 32, 8, 32768, 128, 64, 1024)
    assert lib.ea_hybrid_attn_workspace_size(ctypes.byref(p)) >= 4
    bad = make_params(1, 32, 8, 32768, 100, 64, 1024)
    assert lib.ea_hybrid_attn_workspace_size(ctypes.byref(bad)) == 0
    n = lib.ea_router_workspace_size(1, 8, 32768, 128)
    assert n > 0 and n % (128 * 4) == 0
    assert lib.ea_router_workspace_size(1, 8, 32768, 96) == 0


def test_router_argument_errors(lib):
    def call(k=16, B=1, Hkv=8, N=64, d=128, w1=16, b1=16, hidden=256, w2=16, b2=16, Hq=32,
             thr=0.0, mask=16, ws=256, wsb=1 << 20):
        return lib.ea_router_decide(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, thr, mask, None,
                                    ws, wsb, None)
    assert call(k=0) == _lib.EA_ERR_INVALID_ARG
    assert call(mask=0) == _lib.EA_ERR_INVALID_ARG
    assert call(N=0) == _lib.EA_ERR_INVALID_ARG
    assert call(thr=float("nan")) == _lib.EA_ERR_INVALID_ARG
    assert call(d=96) == _lib.EA_ERR_UNSUPPORTED
    assert call(hidden=8192) == _lib.EA_ERR_UNSUPPORTED
    assert call(hidden=254) == _lib.EA_ERR_UNSUPPORTED
    assert call(w1=20) == _lib.EA_ERR_MISALIGNED
    assert call(ws=0) == _lib.EA_ERR_WORKSPACE
    assert call(wsb=8) == _lib.EA_ERR_WORKSPACE


def test_router_training_argument_errors(lib):
    ws_need = lib.ea_router_ste_backward_workspace_size(2, 8, 64, 128, 256, 32)
    assert ws_need > 0 and lib.ea_router_ste_backward_workspace_size(2, 8, 64, 96, 256, 32) == 0
    assert lib.ea_router_gumbel_workspace_size(2, 8, 64, 128, 256, 32) > 0

    def ste(k=16, B=2, Hkv=8, N=64, d=128, hidden=256, Hq=32, g0=16, tau=1.0, dout=16, dw1=16,
            ws=256, wsb=ws_need):
        return lib.ea_router_ste_backward(k, B, Hkv, N, d, 16, 16, hidden, 16, 16, Hq, g0, 16, tau,
                                          dout, 16, 16, None, None, dw1, 16, 16, 16, None, None,
                                          ws, wsb, None)
    assert ste(k=0) == _lib.EA_ERR_INVALID_ARG
    assert ste(g0=0) == _lib.EA_ERR_INVALID_ARG
    assert ste(dout=0) == _lib.EA_ERR_INVALID_ARG
    assert ste(dw1=0) == _lib.EA_ERR_INVALID_ARG
    assert ste(tau=0.0) == _lib.EA_ERR_INVALID_ARG
    assert ste(tau=float("nan")) == _lib.EA_ERR_INVALID_ARG
    assert ste(tau=float("inf")) == _lib.EA_ERR_INVALID_ARG
    assert ste(B=0) == _lib.EA_ERR_INVALID_ARG
    assert ste(d=96) == _lib.EA_ERR_UNSUPPORTED
    assert ste(hidden=254) == _lib.EA_ERR_UNSUPPORTED
    assert ste(B=1025) == _lib.EA_ERR_UNSUPPORTED
    assert ste(k=24) == _lib.EA_ERR_MISALIGNED
    assert ste(dout=24) == _lib.EA_ERR_MISALIGNED
    assert ste(ws=0) == _lib.EA_ERR_WORKSPACE
    assert ste(wsb=ws_need - 1) == _lib.EA_ERR_WORKSPACE

    def gumbel(mask=16, tau=1.0, wsb=1 << 20):
        return lib.ea_router_decide_gumbel(16, 2, 8, 64, 128, 16, 16, 256, 16, 16, 32, 16, 16, tau,
                                           mask, None, None, 256, wsb, None)
    assert gumbel(mask=0) == _lib.EA_ERR_INVALID_ARG
    assert gumbel(tau=-1.0) == _lib.EA_ERR_INVALID_ARG
    assert gumbel(wsb=8) == _lib.EA_ERR_WORKSPACE


def test_grid_size(lib):
    p = make_params(1, 4, 2, 512, 64, 16, 128)
    assert lib.ea_attn_grid_size(ctypes.byref(p), 148) == 8      # 4 heads x 2 units
    p = make_params(1, 32, 8, 32768, 128, 64, 1024)
    assert lib.ea_attn_grid_size(ctypes.byref(p), 148) == 148


def test_product_path_has_no_oracle_import():
    """The package never imports the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "sparse_attention_head_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def _host(lib, p, qh=16, kh=16, vh=16, mask=16, w1=None, hidden=0, out=16, chunk=0, ws=256,
          wsbytes=1 << 40):
    return lib.ea_hybrid_attn_prefill_host(qh, kh, vh, mask, w1, 16 if w1 else None, hidden,
                                           16 if w1 else None, 16 if w1 else None, 0.0,
                                           ctypes.byref(p), out, None, chunk, ws, wsbytes, None)


def test_host_entry_argument_errors(lib):
    """ea_hybrid_attn_prefill_host rejects bad arguments before anything is
    enqueued (so these calls need no GPU)."""
    good = make_params(1, 8, 4, 700, 128, 16, 200)
    assert _host(lib, make_params(0, 8, 4, 700, 128, 16, 200)) == _lib.EA_ERR_INVALID_ARG
    assert _host(lib, good, qh=0) == _lib.EA_ERR_INVALID_ARG
    assert _host(lib, good, out=0) == _lib.EA_ERR_INVALID_ARG
    assert _host(lib, good, chunk=-1) == _lib.EA_ERR_INVALID_ARG
    assert _host(lib, good, mask=0) == _lib.EA_ERR_INVALID_ARG          # no mask, no router
    assert _host(lib, make_params(1, 8, 4, 700, 128, 16, 200, select=1)) == \
        _lib.EA_ERR_INVALID_ARG
    assert _host(lib, good, ws=0) == _lib.EA_ERR_WORKSPACE
    assert _host(lib, good, w1=16, hidden=0) == _lib.EA_ERR_INVALID_ARG  # router, hidden 0
    assert _host(lib, good, w1=24, hidden=64) == _lib.EA_ERR_MISALIGNED
    assert _host(lib, good, wsbytes=1024) == _lib.EA_ERR_WORKSPACE
    assert _host(lib, good, ws=264) == _lib.EA_ERR_MISALIGNED


def test_host_workspace_and_chunks(lib):
    """Workspace: the 256-byte status block, the mask, the router's scratch
    (with a router) and device copies of q, k, v, out; about eight chunks by
    default, never straddling a batch element."""
    from sparse_attention_head_b200.api import (ea_hybrid_attn_host_chunks,
                                                ea_hybrid_attn_host_workspace_size)
    p = make_params(1, 32, 8, 32768, 128, 64, 1024)
    tensors = (2 * 32 + 2 * 8) * 32768 * 128 * 2
    n0 = ea_hybrid_attn_host_workspace_size(p, 0)
    n1 = ea_hybrid_attn_host_workspace_size(p, 256)
    assert tensors + 512 <= n0 < tensors + 4096
    assert n1 > n0
    assert ea_hybrid_attn_host_workspace_size(make_params(1, 8, 3, 64, 128, 0, 1), 0) == 0
    assert ea_hybrid_attn_host_chunks(p, 0) == 8
    assert ea_hybrid_attn_host_chunks(p, 3) == 3          # 3 + 3 + 2 kv heads
    assert ea_hybrid_attn_host_chunks(p, 100) == 1
    assert ea_hybrid_attn_host_chunks(make_params(2, 32, 8, 65536, 128, 64, 2048), 0) == 8
    assert ea_hybrid_attn_host_chunks(make_params(4, 32, 8, 16384, 128, 128, 512), 0) == 8
    assert ea_hybrid_attn_host_chunks(make_params(3, 4, 2, 512, 64, 16, 128), 0) == 6
    assert ea_hybrid_attn_host_chunks(p, -1) == 0


def test_shutdown_without_streams(lib):
    """With no host-buffer call made, ea_shutdown has nothing to release and
    makes no CUDA call (so it runs without a GPU)."""
    assert lib.ea_shutdown() == _lib.EA_OK


def test_host_prefill_needs_a_mask_without_router():
    """Without router weights the host-buffer wrapper needs the caller's mask
    (checked before any CUDA work)."""
    import torch
    from sparse_attention_head_b200.api import HostPrefill
    hp = HostPrefill.__new__(HostPrefill)
    hp.has_router = False
    with pytest.raises(ValueError):
        hp(torch.zeros(1), torch.zeros(1), torch.zeros(1), None)
