"""Host logic of the decode step (no GPU): the per-head KV-cache policy
against the oracle's rule, and argument checks that return before any
launch."""
import ctypes

import numpy as np
import pytest

import oracle
from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import ea_decode_kv_policy, make_decode_params


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


@pytest.mark.parametrize("B,Hq,Hkv,seed", [(1, 4, 4, 0), (2, 8, 2, 1), (3, 32, 8, 2),
                                           (4, 16, 1, 3), (2, 6, 3, 4)])
def test_kv_policy_matches_oracle(B, Hq, Hkv, seed):
    rng = np.random.default_rng(seed)
    # bias towards SA so that all-SA groups occur at G = 4 and 8
    mask = (rng.random((B, Hq)) < 0.8).astype(np.uint8)
    mask[0, : Hq // Hkv] = 1                       # group 0 of b = 0 all SA
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    want = oracle.kv_head_sparse(mask, Hq, Hkv)
    assert slots.shape == (B, Hkv)
    assert np.array_equal(slots < 0, want.astype(bool))
    assert n_sa == int(want.sum()) and n_full == B * Hkv - n_sa
    # each pool is numbered 0.. in (b, kv head) order, every index once
    full = slots[slots >= 0]
    compact = -slots[slots < 0] - 1
    assert np.array_equal(full, np.arange(n_full))
    assert np.array_equal(compact, np.arange(n_sa))


def test_kv_policy_invalid(lib):
    slots = np.zeros(4, np.int32)
    mask = np.ones(4, np.uint8)
    assert lib.ea_decode_kv_policy(mask.ctypes.data, 1, 4, 3, slots.ctypes.data, None, None) == -1
    assert lib.ea_decode_kv_policy(None, 1, 4, 2, slots.ctypes.data, None, None) == -1
    assert lib.ea_decode_kv_policy(mask.ctypes.data, 0, 4, 2, slots.ctypes.data, None, None) == -1


def test_decode_workspace_size(lib):
    p = make_decode_params(2, 32, 8, 128, 64, 1024, 4096, 10, 6)
    n = lib.ea_decode_workspace_size(ctypes.byref(p))
    # status block, two segment counters per kv group (256-byte blocks), and
    # one (o, max, sum) partial per (b, head, 512-key split)
    assert n == 256 + 256 + 2 * 32 * (4096 // 512) * (128 + 2) * 4
    # the compact cache alone can need more splits than max_len
    p = make_decode_params(1, 4, 4, 64, 600, 600, 100, 0, 4)
    assert lib.ea_decode_workspace_size(ctypes.byref(p)) == 256 + 256 + 4 * 3 * 66 * 4
    p = make_decode_params(20, 32, 8, 128, 4, 16, 64, 160, 0)       # 320 counters: 1280 B
    assert lib.ea_decode_workspace_size(ctypes.byref(p)) == 256 + 1280 + 20 * 32 * 1 * 130 * 4
    # more than 4096 kv groups per step is not supported
    p = make_decode_params(513, 32, 8, 128, 4, 16, 64, 513 * 8, 0)
    assert lib.ea_decode_workspace_size(ctypes.byref(p)) == 0
    for bad in (make_decode_params(1, 4, 4, 96, 4, 16, 64, 4, 0),      # d
                make_decode_params(1, 12, 4, 64, 4, 16, 64, 4, 0),     # G = 3
                make_decode_params(1, 4, 3, 64, 4, 16, 64, 4, 0),      # Hq % Hkv
                make_decode_params(1, 4, 4, 64, 4, 0, 64, 4, 0),       # window
                make_decode_params(1, 4, 4, 64, -1, 16, 64, 4, 0),     # sink
                make_decode_params(1, 4, 4, 64, 4, 16, 64, 0, 0),      # empty pools
                make_decode_params(1, 4, 4, 64, 4, 16, 64, 4, 0, float("nan"))):
        assert lib.ea_decode_workspace_size(ctypes.byref(bad)) == 0


def test_decode_argument_errors(lib):
    p = make_decode_params(1, 4, 2, 64, 4, 16, 64, 2, 0)
    good = dict(q=16, kn=16, vn=16, pos=16, mask=16, slot=16, kf=16, vf=16, ks=None, vs=None,
                out=16, ws=256, wsb=1 << 20)

    def call(params=p, **kw):
        a = dict(good, **kw)
        return lib.ea_hybrid_attn_decode(a["q"], a["kn"], a["vn"], a["pos"], a["mask"],
                                         a["slot"], a["kf"], a["vf"], a["ks"], a["vs"],
                                         ctypes.byref(params), a["out"], a["ws"], a["wsb"], None)
    assert call(q=0) == _lib.EA_ERR_INVALID_ARG
    assert call(pos=0) == _lib.EA_ERR_INVALID_ARG
    assert call(slot=0) == _lib.EA_ERR_INVALID_ARG
    assert call(kf=0) == _lib.EA_ERR_INVALID_ARG                     # n_full > 0
    with_sa = make_decode_params(1, 4, 2, 64, 4, 16, 64, 1, 1)
    assert call(params=with_sa) == _lib.EA_ERR_INVALID_ARG           # n_sa > 0, no k_sa
    assert call(q=24) == _lib.EA_ERR_MISALIGNED
    assert call(kf=40) == _lib.EA_ERR_MISALIGNED
    assert call(ws=0) == _lib.EA_ERR_WORKSPACE
    assert call(wsb=8) == _lib.EA_ERR_WORKSPACE
    assert call(params=make_decode_params(1, 4, 2, 96, 4, 16, 64, 2, 0)) == \
        _lib.EA_ERR_UNSUPPORTED
    assert lib.ea_hybrid_attn_decode(16, 16, 16, 16, 16, 16, 16, 16, None, None, None, 16, 256,
                                     1 << 20, None) == _lib.EA_ERR_INVALID_ARG
