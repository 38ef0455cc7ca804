"""GPU parity of the decode step (through the C ABI) against the oracle's
decode_step: the output at position t is prefill row t of the same head, the
caches follow the per-head policy (compact sink + window ring for all-SA kv
heads), sequences sit at different positions, and invalid slots or
positions are reported through the status word."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import compare, f64
from sparse_attention_head_b200 import _lib, build
from sparse_attention_head_b200.api import (decode_workspace, ea_decode_kv_policy,
                                            ea_get_device_status, ea_hybrid_attn_decode,
                                            make_decode_params)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def _history(B, Hq, Hkv, L, d, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, L, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _mask(B, Hq, Hkv, seed):
    """Every kind of kv group: all SA (compact cache), mixed, all FA."""
    rng = np.random.default_rng(seed)
    G = Hq // Hkv
    m = (rng.random((B, Hq)) < 0.5).astype(np.uint8)
    for b in range(B):
        for hk in range(Hkv):
            kind = (b + hk) % 3
            if kind == 0:
                m[b, hk * G:(hk + 1) * G] = 1
            elif kind == 1 and G > 1:
                m[b, hk * G] = 0
                m[b, hk * G + 1] = 1
            else:
                m[b, hk * G:(hk + 1) * G] = 0
    return m


def _caches(slots, n_full, n_sa, max_len, S, W, d):
    z = dict(dtype=torch.bfloat16, device=DEV)
    kf = torch.zeros((n_full, max_len, d), **z) if n_full else None
    vf = torch.zeros((n_full, max_len, d), **z) if n_full else None
    ks = torch.zeros((n_sa, S + W, d), **z) if n_sa else None
    vs = torch.zeros((n_sa, S + W, d), **z) if n_sa else None
    return kf, vf, ks, vs


def _prefill_caches(caches, slots, k, v, pos, S, W):
    """Write positions [0, pos[b]) of every (b, kv head) into its cache, as
    earlier decode steps would have left it (test setup on the host)."""
    kf, vf, ks, vs = caches
    B, Hkv = slots.shape
    for b in range(B):
        t = int(pos[b])
        for hk in range(Hkv):
            c = int(slots[b, hk])
            if c >= 0:
                kf[c, :t] = k[b, hk, :t].to(DEV)
                vf[c, :t] = v[b, hk, :t].to(DEV)
            else:
                # the sinks, then the last W positions (distinct ring slots)
                ps = list(range(min(S, t))) + list(range(max(S, t - W), t))
                rows = [oracle.compact_slot(p, S, W) for p in ps]
                assert len(set(rows)) == len(rows)
                ks[-c - 1, rows] = k[b, hk, ps].to(DEV)
                vs[-c - 1, rows] = v[b, hk, ps].to(DEV)


def _step(q_t, k_t, v_t, pos, mask, slots, caches, S, W, max_len, ws):
    kf, vf, ks, vs = caches
    return ea_hybrid_attn_decode(q_t.to(DEV).contiguous(), k_t.to(DEV).contiguous(),
                                 v_t.to(DEV).contiguous(),
                                 torch.as_tensor(pos, dtype=torch.int32, device=DEV),
                                 torch.as_tensor(mask, device=DEV),
                                 torch.as_tensor(slots, dtype=torch.int32, device=DEV),
                                 kf, vf, ks, vs, S, W, max_len, workspace=ws)


CASES = [
    # B, Hq, Hkv, d, S, W, max_len, positions
    (3, 32, 8, 128, 64, 1024, 4096, [4095, 37, 1500]),     # GQA 4, several splits
    (2, 16, 2, 64, 4, 100, 2000, [1999, 700]),             # GQA 8, ring wrapped many times
    (2, 4, 4, 128, 0, 1, 600, [599, 0]),                   # MHA, no sink, window 1
    (1, 8, 4, 64, 130, 257, 1300, [1299]),                 # GQA 2, sinks span two chunks
    (2, 8, 8, 128, 1, 512, 1541, [1540, 1024]),            # ragged split tail
    (1, 8, 1, 128, 2000, 300, 1800, [1799]),               # sinks beyond max_len (all sink)
    # the bench's layer shape at the positions it decodes (16K-32K): long
    # full caches split many ways, wrapped rings
    (3, 32, 8, 128, 64, 1024, 32768, [32767, 16384, 24001]),
]


@pytest.mark.parametrize("B,Hq,Hkv,d,S,W,max_len,pos", CASES)
def test_decode_step_matches_oracle(B, Hq, Hkv, d, S, W, max_len, pos):
    L = max(pos) + 1
    q, k, v = _history(B, Hq, Hkv, L, d, seed=B * 1000 + L)
    mask = _mask(B, Hq, Hkv, seed=L)
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    caches = _caches(slots, n_full, n_sa, max_len, S, W, d)
    _prefill_caches(caches, slots, k, v, pos, S, W)
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    idx = torch.as_tensor(pos, dtype=torch.long)
    bi = torch.arange(B)
    q_t, k_t, v_t = q[bi, :, idx], k[bi, :, idx], v[bi, :, idx]
    out = _step(q_t, k_t, v_t, pos, mask, slots, caches, S, W, max_len, ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0
    ref = oracle.decode_step(f64(q_t), f64(k), f64(v), pos, mask, S, W)
    compare(out, ref, f"decode B{B} Hq{Hq} Hkv{Hkv} d{d} S{S} W{W}", few_keys=W <= 2)
    # the step appended the new key and value where the policy puts them
    kf, vf, ks, vs = caches
    for b in range(B):
        for hk in range(Hkv):
            c = int(slots[b, hk])
            row = kf[c, pos[b]] if c >= 0 else ks[-c - 1, oracle.compact_slot(pos[b], S, W)]
            assert torch.equal(row.cpu(), k_t[b, hk])


@pytest.mark.parametrize("d,G", [(128, 4), (64, 2), (128, 8), (64, 1)])
def test_decode_steps_build_the_cache(d, G):
    """Token by token from an empty cache: every step appends, then attends;
    the compact ring wraps several times (S = 3, W = 16, 60 steps)."""
    B, Hkv, S, W, T = 2, 2, 3, 16, 60
    Hq = Hkv * G
    q, k, v = _history(B, Hq, Hkv, T, d, seed=77 + d + G)
    mask = _mask(B, Hq, Hkv, seed=G)
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    caches = _caches(slots, n_full, n_sa, T, S, W, d)
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, T, n_full, n_sa), DEV)
    kd, vd = f64(k), f64(v)
    for t in range(T):
        pos = [t] * B
        out = _step(q[:, :, t], k[:, :, t], v[:, :, t], pos, mask, slots, caches, S, W, T, ws)
        ref = oracle.decode_step(f64(q[:, :, t]), kd, vd, pos, mask, S, W)
        compare(out, ref, f"step {t}", few_keys=t < 4)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == 0


def test_fa_head_on_compact_cache_is_reported():
    """A compact cache behind a kv group with an FA query head: the status
    word says so and the group attends over sink + window keys."""
    B, Hq, Hkv, d, S, W, max_len = 1, 4, 2, 64, 2, 8, 64
    t = 40
    q, k, v = _history(B, Hq, Hkv, t + 1, d, seed=5)
    mask = np.array([[0, 1, 1, 1]], np.uint8)             # group 0 mixed
    slots = np.array([[-1, -2]], np.int32)                 # both compact
    caches = _caches(slots, 0, 2, max_len, S, W, d)
    _prefill_caches(caches, slots, k, v, [t], S, W)
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, 0, 2), DEV)
    out = _step(q[:, :, t], k[:, :, t], v[:, :, t], [t], mask, slots, caches, S, W, max_len, ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == _lib.EA_ERR_INVALID_ARG
    ref = oracle.decode_step(f64(q[:, :, t]), f64(k), f64(v), [t], np.ones_like(mask), S, W)
    compare(out, ref, "compact FA group")


@pytest.mark.parametrize("case", ["pos_past_full_cache", "negative_pos", "slot_out_of_pool"])
def test_invalid_positions_and_slots_are_reported(case):
    B, Hq, Hkv, d, S, W, max_len = 2, 4, 2, 128, 2, 8, 32
    q, k, v = _history(B, Hq, Hkv, 1, d, seed=9)
    mask = np.zeros((B, Hq), np.uint8)
    slots, n_full, n_sa = ea_decode_kv_policy(mask, Hkv)
    pos = [5, 5]
    if case == "pos_past_full_cache":
        pos = [5, max_len]
    elif case == "negative_pos":
        pos = [5, -1]
    else:
        slots = slots.copy()
        slots[1, 1] = n_full                               # one past the pool
    caches = _caches(slots, n_full, n_sa, max_len, S, W, d)
    before = caches[0].clone()
    ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa), DEV)
    out = _step(q[:, :, 0], k[:, :, 0], v[:, :, 0], pos, mask, slots, caches, S, W, max_len, ws)
    torch.cuda.synchronize()
    assert ea_get_device_status(ws) == _lib.EA_ERR_INVALID_ARG
    bad = (1, slice(2, 4)) if case == "slot_out_of_pool" else (1, slice(0, 4))
    assert torch.count_nonzero(out[bad]) == 0
    # only the valid (b, kv head) pairs appended, at position 5
    valid = [(0, 0), (0, 1)] + ([(1, 0)] if case == "slot_out_of_pool" else [])
    changed = (caches[0] != before).any(dim=-1).nonzero().tolist()
    assert sorted(changed) == sorted([int(slots[b, hk]), 5] for b, hk in valid)
