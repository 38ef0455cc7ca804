"""Pins for the CPU oracle: facts fixed by the pages or by mathematics, not by
the oracle itself.  Each test is chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign, an off-by-one window, a transposed
operand, a wrong GQA mapping, a wrong scale) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=np.float64):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape).astype(dtype)


def _bf16(x):
    """Round float64 values to bf16 exactly as the GPU inputs are rounded."""
    return torch.from_numpy(np.asarray(x)).to(torch.bfloat16).double().numpy()


def _qkv(B, Hq, Hkv, N, d, seed):
    q = _bf16(_rand((B, Hq, N, d), seed))
    k = _bf16(_rand((B, Hkv, N, d), seed + 1))
    v = _bf16(_rand((B, Hkv, N, d), seed + 2))
    return q, k, v


# --------------------------------------------------------------------------
# Router pins
# --------------------------------------------------------------------------

def test_router_size_matches_printed_value():
    """EA blog §2.2 prints 0.27M router parameters per layer (8B model)."""
    g = json.load(open(os.path.join(GOLDEN, "router_size.json")))
    n = oracle.router_param_count(*g["dims"])
    assert n == 270624
    assert abs(n - g["printed_params_per_layer"]) <= g["printed_precision"]
    # a router without biases or with a 2-way output per head would not round
    # to the printed value
    assert abs(1024 * 256 + 256 * 64 + 256 + 64 - 270000) > 5000


def test_router_pool_closed_forms():
    B, Hkv, N, d = 2, 3, 37, 5
    k = np.zeros((B, Hkv, N, d))
    for b in range(B):
        for h in range(Hkv):
            for n in range(N):
                for c in range(d):
                    k[b, h, n, c] = 1000.0 * h + c + 0.5 * n + 7.0 * b
    x = oracle.router_pool(k)
    assert x.shape == (B, Hkv * d)
    for b in range(B):
        for h in range(Hkv):
            for c in range(d):
                # mean of 0.5 n over n = 0..N-1 is 0.25 (N - 1)
                want = 1000.0 * h + c + 0.25 * (N - 1) + 7.0 * b
                assert x[b, h * d + c] == pytest.approx(want, abs=1e-9)


def test_router_mlp_hand_example():
    """A hand-worked two-layer MLP: ReLU kills the negative pre-activation,
    the biases enter once, a logit exactly at the threshold routes to FA."""
    x = np.array([[1.0, -2.0, 3.0]])
    w1 = np.eye(3)
    b1 = np.array([0.0, 0.0, -1.0])         # pre = [1, -2, 2] -> h = [1, 0, 2]
    w2 = np.array([[1.0, 1.0, 1.0], [0.0, -1.0, 0.0], [-1.0, 0.0, 0.0]])
    b2 = np.array([0.5, 0.0, 0.25])         # z = [3.5, 0, -0.75]
    z = oracle.router_mlp(x, w1, b1, w2, b2)
    np.testing.assert_allclose(z, [[3.5, 0.0, -0.75]], atol=0, rtol=0)
    k = np.broadcast_to(np.array([1.0, -2.0, 3.0]), (1, 1, 4, 3)).copy()
    mask, z2 = oracle.router_decide(k, w1, b1, w2, b2, threshold=0.0)
    np.testing.assert_array_equal(mask, [[1, 0, 0]])   # r=1 -> SA, tie -> FA
    mask_hi, _ = oracle.router_decide(k, w1, b1, w2, b2, threshold=3.5)
    np.testing.assert_array_equal(mask_hi, [[0, 0, 0]])


def test_router_matches_torch_linear():
    """Cross-check with torch's nn.functional.linear in float64."""
    B, Hkv, N, d, hid, Hq = 2, 2, 19, 8, 16, 4
    k = _rand((B, Hkv, N, d), 5)
    w1, b1 = _rand((hid, Hkv * d), 6), _rand((hid,), 7)
    w2, b2 = _rand((Hq, hid), 8), _rand((Hq,), 9)
    z = oracle.router_mlp(oracle.router_pool(k), w1, b1, w2, b2)
    kt = torch.from_numpy(k)
    x = kt.mean(dim=2).reshape(B, Hkv * d)
    h = torch.relu(torch.nn.functional.linear(x, torch.from_numpy(w1), torch.from_numpy(b1)))
    zt = torch.nn.functional.linear(h, torch.from_numpy(w2), torch.from_numpy(b2))
    np.testing.assert_allclose(z, zt.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Attention pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,d", [(1, 8), (63, 16), (300, 32)])
def test_all_fa_is_dense_causal_sdpa(N, d):
    """An all-zero mask is dense causal attention: torch SDPA in float64."""
    B, Hq, Hkv = 2, 4, 2
    q, k, v = _qkv(B, Hq, Hkv, N, d, 11)
    mask = np.zeros((B, Hq), np.uint8)
    out = oracle.attention(q, k, v, mask, sink=3, window=5, block=64)
    g = Hq // Hkv
    kt = torch.from_numpy(k).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(g, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), kt, vt, is_causal=True)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_sparse_equals_full_when_window_covers_sequence():
    B, Hq, Hkv, N, d = 1, 4, 4, 90, 16
    q, k, v = _qkv(B, Hq, Hkv, N, d, 12)
    full = oracle.attention(q, k, v, np.zeros((B, Hq), np.uint8), 10, 80, block=32)
    for S, W in [(10, 80), (0, 90), (90, 1), (45, 45), (5, 200)]:
        sa = oracle.attention(q, k, v, np.ones((B, Hq), np.uint8), S, W, block=32)
        np.testing.assert_array_equal(sa, full)
    # one key short of covering: a late row must differ
    sa = oracle.attention(q, k, v, np.ones((B, Hq), np.uint8), 10, 79, block=32)
    assert np.max(np.abs(sa[..., -1, :] - full[..., -1, :])) > 1e-6


def test_window_one_no_sink_returns_own_value():
    """S = 0, W = 1: each query sees only itself, out[i] = v[i] (GQA h // G)."""
    B, Hq, Hkv, N, d = 2, 6, 2, 40, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 13)
    out = oracle.attention(q, k, v, np.ones((B, Hq), np.uint8), 0, 1, block=16)
    for h in range(Hq):
        np.testing.assert_array_equal(out[:, h], v[:, h // 3])


def test_sink_one_window_one_two_key_closed_form():
    """S = 1, W = 1: query i > 0 sees keys {0, i}.  With a = (q.k0 - q.ki)/sqrt(d),
    out[i] = sigma(a) v0 + (1 - sigma(a)) vi, and out[0] = v0."""
    B, Hq, Hkv, N, d = 1, 2, 1, 30, 16
    q, k, v = _qkv(B, Hq, Hkv, N, d, 14)
    out = oracle.attention(q, k, v, np.ones((B, Hq), np.uint8), 1, 1, block=8)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h, 0], v[0, 0, 0], atol=1e-15)
        for i in range(1, N):
            a = (q[0, h, i] @ k[0, 0, 0] - q[0, h, i] @ k[0, 0, i]) / math.sqrt(d)
            sig = 1.0 / (1.0 + math.exp(-a))
            want = sig * v[0, 0, 0] + (1.0 - sig) * v[0, 0, i]
            np.testing.assert_allclose(out[0, h, i], want, rtol=0, atol=1e-13)


def test_explicit_scale_enters_scores():
    B, Hq, Hkv, N, d = 1, 1, 1, 12, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 15)
    m = np.ones((1, 1), np.uint8)
    out = oracle.attention(q, k, v, m, 1, 1, scale=0.25, block=4)
    i = 7
    a = 0.25 * (q[0, 0, i] @ k[0, 0, 0] - q[0, 0, i] @ k[0, 0, i])
    sig = 1.0 / (1.0 + math.exp(-a))
    np.testing.assert_allclose(out[0, 0, i], sig * v[0, 0, 0] + (1 - sig) * v[0, 0, i],
                               atol=1e-13)


def test_constant_values_give_constant_output():
    B, Hq, Hkv, N, d = 1, 4, 2, 77, 8
    q, k, _ = _qkv(B, Hq, Hkv, N, d, 16)
    v = np.broadcast_to(np.arange(d, dtype=np.float64) - 2.5, (B, Hkv, N, d)).copy()
    mask = np.array([[0, 1, 1, 0]], np.uint8)
    out = oracle.attention(q, k, v, mask, 4, 9, block=16)
    np.testing.assert_allclose(out, np.broadcast_to(v[:, :1], out.shape), atol=1e-13)


def test_weights_sum_to_one_and_vanish_off_pattern():
    B, Hq, Hkv, N, d = 1, 2, 1, 50, 8
    q, k, _ = _qkv(B, Hq, Hkv, N, d, 17)
    mask = np.array([[0, 1]], np.uint8)
    S, W = 3, 7
    for h in range(Hq):
        w = oracle.attention_weights(q, k, mask, 0, h, S, W)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-14)
        for i in range(N):
            for j in range(N):
                causal = j <= i
                seen = causal and (h == 0 or j < S or i - j < W)
                if not seen:
                    assert w[i, j] == 0.0
                else:
                    assert w[i, j] > 0.0
    # visible-key counts per row of the SA head
    counts = [(oracle.attention_weights(q, k, mask, 0, 1, S, W)[i] > 0).sum()
              for i in range(N)]
    for i, c in enumerate(counts):
        assert c == min(i + 1, W + min(S, max(0, i - W + 1)))


def test_head_permutation_equivariance():
    """Permuting kv groups and heads within a group, together with their mask
    bits, permutes the outputs the same way."""
    B, Hq, Hkv, N, d = 2, 6, 3, 45, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 18)
    rng = np.random.default_rng(3)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    out = oracle.attention(q, k, v, mask, 2, 6, block=16)
    gperm = np.array([2, 0, 1])
    inner = np.array([1, 0])
    hperm = np.array([gp * 2 + inner[i] for gp in gperm for i in range(2)])
    out2 = oracle.attention(q[:, hperm], k[:, gperm], v[:, gperm], mask[:, hperm], 2, 6,
                            block=16)
    np.testing.assert_allclose(out2, out[:, hperm], atol=1e-14, rtol=0)


def test_batch_rows_independent():
    B, Hq, Hkv, N, d = 3, 2, 1, 33, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 19)
    mask = np.array([[0, 1], [1, 1], [0, 0]], np.uint8)
    out = oracle.attention(q, k, v, mask, 2, 5, block=8)
    for b in range(B):
        one = oracle.attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], mask[b:b + 1], 2, 5,
                               block=8)
        np.testing.assert_array_equal(one[0], out[b])


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_agrees(seed):
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.integers(1, 3))
    g = int(rng.integers(1, 3))
    Hq = Hkv * g
    B = int(rng.integers(1, 3))
    N = int(rng.integers(1, 65))
    d = int(rng.choice([4, 8]))
    S = int(rng.integers(0, 9))
    W = int(rng.integers(1, 20))
    q, k, v = _qkv(B, Hq, Hkv, N, d, 200 + seed)
    mask = rng.integers(0, 2, size=(B, Hq)).astype(np.uint8)
    fast = oracle.attention(q, k, v, mask, S, W, block=int(rng.integers(1, 40)))
    slow = oracle.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), mask.tolist(),
                                        S, W)
    np.testing.assert_allclose(fast, slow, rtol=0, atol=1e-12)
    rows = sorted(set(int(r) for r in rng.integers(0, N, size=5)))
    for b in range(B):
        for h in range(Hq):
            part = oracle.attention_rows(q, k, v, mask, b, h, rows, S, W)
            np.testing.assert_allclose(part, slow[b, h, rows], rtol=0, atol=1e-12)


def test_visible_pair_counts_closed_forms():
    for N in [1, 2, 17, 300]:
        assert oracle.count_visible_pairs(N, False, 5, 7) == N * (N + 1) // 2
    # pure sliding window: row i sees min(i + 1, W) keys
    for N, W in [(50, 7), (10, 20), (129, 128)]:
        want = sum(min(i + 1, W) for i in range(N))
        assert oracle.count_visible_pairs(N, True, 0, W) == want
    # sink + window: a row past S + W - 1 sees exactly S + W keys
    S, W, N = 4, 6, 40
    assert len(oracle.visible_keys(N - 1, True, S, W)) == S + W
    assert len(oracle.visible_keys(S + W - 1, True, S, W)) == S + W
    assert len(oracle.visible_keys(S + W - 2, True, S, W)) == S + W - 1


# --------------------------------------------------------------------------
# Decode-step pins
# --------------------------------------------------------------------------

def test_decode_step_is_the_prefill_row():
    """A decode step at position t gives prefill row t of the same head."""
    B, Hq, Hkv, N, d = 2, 4, 2, 70, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 31)
    mask = np.array([[0, 1, 1, 1], [1, 0, 0, 1]], np.uint8)
    S, W = 3, 9
    pos = np.array([N - 1, 37])
    full = oracle.attention(q, k, v, mask, S, W, block=16)
    qt = np.stack([q[b, :, pos[b]] for b in range(B)])
    out = oracle.decode_step(qt, k, v, pos, mask, S, W)
    for b in range(B):
        np.testing.assert_allclose(out[b], full[b, :, pos[b]], rtol=0, atol=1e-13)


def test_decode_step_closed_forms():
    B, Hq, Hkv, N, d = 1, 2, 1, 30, 8
    q, k, v = _qkv(B, Hq, Hkv, N, d, 32)
    qt = q[:, :, 17]
    out = oracle.decode_step(qt, k, v, [17], np.ones((1, 2), np.uint8), 0, 1)
    np.testing.assert_array_equal(out[0, 0], v[0, 0, 17])   # W=1, S=0: its own value
    out = oracle.decode_step(qt, k, v, [17], np.ones((1, 2), np.uint8), 1, 1)
    a = (qt[0, 1] @ k[0, 0, 0] - qt[0, 1] @ k[0, 0, 17]) / math.sqrt(d)
    sig = 1.0 / (1.0 + math.exp(-a))
    np.testing.assert_allclose(out[0, 1], sig * v[0, 0, 0] + (1 - sig) * v[0, 0, 17], atol=1e-13)


def test_compact_cache_slots():
    S, W = 4, 6
    # sinks never move
    assert [oracle.compact_slot(p, S, W) for p in range(S)] == list(range(S))
    # the last W positions (>= S) of any query occupy distinct ring slots
    for t in range(S, 60):
        window = [p for p in range(max(S, t - W + 1), t + 1)]
        slots = [oracle.compact_slot(p, S, W) for p in window]
        assert len(set(slots)) == len(slots)
        assert all(S <= s < S + W for s in slots)
    # the ring wraps with period W
    assert oracle.compact_slot(S + 3, S, W) == oracle.compact_slot(S + 3 + W, S, W)
    # layout convention (part of the cache API): the first position after the
    # sinks fills the first ring slot, and the ring restarts there every W
    assert oracle.compact_slot(S, S, W) == S
    assert oracle.compact_slot(S + W, S, W) == S
    assert oracle.compact_slot(S + W - 1, S, W) == S + W - 1


def test_kv_head_sparse_requires_all_query_heads():
    mask = np.array([[1, 1, 0, 1, 1, 1], [0, 0, 1, 1, 1, 0]], np.uint8)
    np.testing.assert_array_equal(oracle.kv_head_sparse(mask, 6, 3), [[1, 0, 1], [0, 1, 0]])
    np.testing.assert_array_equal(oracle.kv_head_sparse(mask, 6, 6), mask)


# --------------------------------------------------------------------------
# Packed variable-length batches: every sequence is its own prefill
# --------------------------------------------------------------------------

def _packed(cu, Hq, Hkv, d, seed):
    T = cu[-1]
    q = _bf16(_rand((T, Hq, d), seed))
    k = _bf16(_rand((T, Hkv, d), seed + 1))
    v = _bf16(_rand((T, Hkv, d), seed + 2))
    return q, k, v


def test_varlen_matches_brute_force_per_sequence():
    cu = [0, 5, 5, 17, 40]                      # includes an empty sequence
    Hq, Hkv, d, S, W = 4, 2, 8, 2, 5
    q, k, v = _packed(cu, Hq, Hkv, d, 61)
    mask = np.array([[0, 1, 1, 0], [1, 1, 1, 1], [1, 0, 1, 0], [0, 0, 1, 1]], np.uint8)
    out = oracle.attention_varlen(q, k, v, cu, mask, S, W)
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        if t1 == t0:
            continue
        # brute force on the sequence laid out as its own batch of one
        qs = q[t0:t1].transpose(1, 0, 2)[None]
        ks = k[t0:t1].transpose(1, 0, 2)[None]
        vs = v[t0:t1].transpose(1, 0, 2)[None]
        ref = oracle.brute_force_attention(qs, ks, vs, mask[b:b + 1], S, W)
        np.testing.assert_allclose(out[t0:t1], ref[0].transpose(1, 0, 2), rtol=0, atol=1e-12)


def test_varlen_positions_restart_per_sequence():
    """The first token of every sequence sees only itself: out = its own v."""
    cu = [0, 7, 19, 20, 33]
    Hq, Hkv, d = 4, 2, 8
    q, k, v = _packed(cu, Hq, Hkv, d, 62)
    mask = np.array([[0, 1, 0, 1]] * 4, np.uint8)
    out = oracle.attention_varlen(q, k, v, cu, mask, 3, 4)
    for b in range(4):
        for h in range(Hq):
            np.testing.assert_array_equal(out[cu[b], h], v[cu[b], h // 2])


def test_varlen_sequences_are_independent():
    cu = [0, 9, 30, 44]
    Hq, Hkv, d = 2, 1, 8
    q, k, v = _packed(cu, Hq, Hkv, d, 63)
    mask = np.array([[0, 1], [1, 0], [0, 0]], np.uint8)
    out = oracle.attention_varlen(q, k, v, cu, mask, 2, 6)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[9:30] += 1.0
    k2[9:30] -= 0.5
    v2[9:30] *= 3.0
    out2 = oracle.attention_varlen(q2, k2, v2, cu, mask, 2, 6)
    np.testing.assert_array_equal(out2[:9], out[:9])
    np.testing.assert_array_equal(out2[30:], out[30:])
    assert not np.allclose(out2[9:30], out[9:30])


def test_varlen_router_pool_closed_forms():
    cu = [0, 4, 4, 11]
    Hkv, d = 2, 3
    T = cu[-1]
    # key rows k[t, kh, c] = t + 100 kh + 1000 c: the mean over [t0, t1) is
    # (t0 + t1 - 1) / 2 + 100 kh + 1000 c
    k = np.array([[[t + 100 * kh + 1000 * c for c in range(d)] for kh in range(Hkv)]
                  for t in range(T)], np.float64)
    x = oracle.router_pool_varlen(k, cu)
    assert x.shape == (3, Hkv * d)
    for b, (t0, t1) in enumerate(zip(cu[:-1], cu[1:])):
        want = np.zeros(Hkv * d) if t1 == t0 else np.array(
            [(t0 + t1 - 1) / 2 + 100 * kh + 1000 * c for kh in range(Hkv) for c in range(d)])
        np.testing.assert_allclose(x[b], want, rtol=0, atol=1e-9)


# --------------------------------------------------------------------------
# Backward pass and the straight-through router gradients
# --------------------------------------------------------------------------

def _fd_grad(f, x, eps=1e-6):
    """Central finite differences of scalar f over every element of x."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def test_attention_backward_matches_finite_differences():
    """Gradients of L = sum(dout * out) against central differences of the
    per-element brute-force forward (independent of the backward formulas);
    GQA with FA and SA heads sharing kv heads."""
    rng = np.random.default_rng(71)
    B, Hq, Hkv, N, d, S, W = 1, 4, 2, 9, 3, 1, 3
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    dout = rng.standard_normal((B, Hq, N, d))
    mask = np.array([[0, 1, 1, 0]], np.uint8)

    def loss():
        return float(np.sum(dout * oracle.brute_force_attention(q, k, v, mask, S, W)))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, mask, S, W)
    np.testing.assert_allclose(dq, _fd_grad(loss, q), rtol=0, atol=1e-6)
    np.testing.assert_allclose(dk, _fd_grad(loss, k), rtol=0, atol=1e-6)
    np.testing.assert_allclose(dv, _fd_grad(loss, v), rtol=0, atol=1e-6)


def test_sampled_backward_matches_finite_differences():
    """The sampled gradients of one kv group at every row and key against
    central differences of the brute-force forward (independent of both
    backward functions); a block smaller than N so the row blocks meet."""
    rng = np.random.default_rng(73)
    B, Hq, Hkv, N, d, S, W = 2, 4, 2, 8, 2, 2, 3
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    dout = rng.standard_normal((B, Hq, N, d))
    mask = np.array([[0, 1, 1, 1], [1, 0, 0, 1]], np.uint8)

    def loss():
        return float(np.sum(dout * oracle.brute_force_attention(q, k, v, mask, S, W)))
    fq, fk, fv = _fd_grad(loss, q), _fd_grad(loss, k), _fd_grad(loss, v)
    for b in range(B):
        for hk in range(Hkv):
            dq, dk, dv = oracle.attention_backward_sampled(
                q, k, v, dout, mask, b, hk, np.arange(N), np.arange(N), S, W, block=3)
            np.testing.assert_allclose(dq, fq[b, 2 * hk:2 * hk + 2], rtol=0, atol=1e-6)
            np.testing.assert_allclose(dk, fk[b, hk], rtol=0, atol=1e-6)
            np.testing.assert_allclose(dv, fv[b, hk], rtol=0, atol=1e-6)


@pytest.mark.parametrize("S,W,block", [(4, 16, 32), (0, 1, 8), (3, 200, 64), (70, 5, 16)])
def test_sampled_backward_equals_dense_backward(S, W, block):
    """Sampled rows and keys (the first and last, block edges, sinks, window
    edges) equal the dense backward's, for mixed FA/SA groups."""
    rng = np.random.default_rng(74 + W)
    B, Hq, Hkv, N, d = 1, 8, 2, 150, 8
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    dout = rng.standard_normal((B, Hq, N, d))
    mask = np.array([[1, 0, 1, 1, 1, 1, 0, 0]], np.uint8)
    rq, rk, rv = oracle.attention_backward(q, k, v, dout, mask, S, W)
    rows = sorted({0, 1, max(S - 1, 0), S, W - 1, W, block - 1, block, 2 * block, N - 2, N - 1}
                  & set(range(N)))
    for hk in range(Hkv):
        dq, dk, dv = oracle.attention_backward_sampled(q, k, v, dout, mask, 0, hk, rows, rows,
                                                       S, W, block=block)
        np.testing.assert_allclose(dq, rq[0, 4 * hk:4 * hk + 4][:, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, rk[0, hk, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, rv[0, hk, rows], rtol=0, atol=1e-12)


def test_attention_lse_matches_the_definition():
    rng = np.random.default_rng(72)
    B, Hq, Hkv, N, d, S, W = 1, 2, 1, 11, 4, 2, 3
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    mask = np.array([[0, 1]], np.uint8)
    lse = oracle.attention_lse(q, k, mask, S, W)
    for h in range(Hq):
        for i in range(N):
            tot = 0.0
            for j in range(N):
                if oracle.visible(i, j, bool(mask[0, h]), S, W):
                    tot += math.exp(float(q[0, h, i] @ k[0, 0, j]) / math.sqrt(d))
            assert abs(lse[0, h, i] - math.log(tot)) < 1e-12


def test_router_ste_backward_matches_the_soft_surrogate():
    """The straight-through gradients equal the exact gradients of the soft
    surrogate sum(dout * (r_soft O_SA + (1 - r_soft) O_FA)) with both
    attention outputs held fixed (central differences)."""
    rng = np.random.default_rng(73)
    B, Hq, Hkv, N, d, hidden, tau = 2, 3, 2, 5, 2, 6, 0.7
    k = rng.standard_normal((B, Hkv, N, d))
    w1 = rng.standard_normal((hidden, Hkv * d)) * 0.7
    b1 = rng.standard_normal(hidden) * 0.3
    w2 = rng.standard_normal((Hq, hidden)) * 0.7
    b2 = rng.standard_normal(Hq) * 0.3
    g0 = rng.gumbel(size=(B, Hq))
    g1 = rng.gumbel(size=(B, Hq))
    dout = rng.standard_normal((B, Hq, 4, 3))
    o_fa = rng.standard_normal((B, Hq, 4, 3))
    o_sa = rng.standard_normal((B, Hq, 4, 3))

    def loss():
        x = k.mean(axis=2).reshape(B, Hkv * d)
        pre = x @ w1.T + b1
        z = np.maximum(pre, 0.0) @ w2.T + b2
        r = 1.0 / (1.0 + np.exp(-(z + g1 - g0) / tau))
        out = r[:, :, None, None] * o_sa + (1.0 - r[:, :, None, None]) * o_fa
        return float(np.sum(dout * out))
    dr, dz, dw1, db1, dw2, db2, dk = oracle.router_ste_backward(k, w1, b1, w2, b2, g0, g1, tau,
                                                                dout, o_fa, o_sa)
    np.testing.assert_allclose(dr, np.sum(dout * (o_sa - o_fa), axis=(2, 3)), atol=1e-12)
    for got, x in ((dw1, w1), (db1, b1), (dw2, w2), (db2, b2), (dk, k)):
        np.testing.assert_allclose(got, _fd_grad(loss, x), rtol=0, atol=1e-6)


def test_gumbel_hard_decision_is_the_soft_argmax():
    rng = np.random.default_rng(74)
    B, Hkv, N, d, Hq, hidden = 3, 2, 6, 4, 5, 8
    k = rng.standard_normal((B, Hkv, N, d))
    w1, b1 = rng.standard_normal((hidden, Hkv * d)), rng.standard_normal(hidden)
    w2, b2 = rng.standard_normal((Hq, hidden)), rng.standard_normal(Hq)
    g0, g1 = rng.gumbel(size=(B, Hq)), rng.gumbel(size=(B, Hq))
    r_hard, r_soft, z = oracle.router_gumbel_forward(k, w1, b1, w2, b2, g0, g1, 0.5)
    np.testing.assert_array_equal(r_hard, (r_soft > 0.5).astype(np.uint8))
    # no noise: the hard decision is the inference threshold z > 0
    r0, _, z0 = oracle.router_gumbel_forward(k, w1, b1, w2, b2, np.zeros_like(g0),
                                             np.zeros_like(g1), 0.5)
    np.testing.assert_array_equal(r0, oracle.router_decide(k, w1, b1, w2, b2)[0])
    # a small temperature makes the soft decision hard
    _, r_cold, _ = oracle.router_gumbel_forward(k, w1, b1, w2, b2, g0, g1, 1e-6)
    np.testing.assert_allclose(r_cold, r_hard, atol=1e-6)


# ---------------------------------------------------------------- FP8 (e4m3)
# The format is fixed by its definition (1 sign, 4 exponent bits with bias 7,
# 3 mantissa bits, no infinities, 0x7f / 0xff NaN, largest finite 448), not by
# the pages; the pins below are closed forms of that definition, ties to even
# at every midpoint, and an independent library conversion.

def test_e4m3_codes_closed_forms():
    x = np.array([1.0, 0.5, 2.0 ** -6, 2.0 ** -9, 7 * 2.0 ** -9, 448.0, 240.0, 1.125, -3.5,
                  -0.0, 0.0], np.float32)
    want = [0x38, 0x30, 0x08, 0x01, 0x07, 0x7E, 0x77, 0x39, 0xC6, 0x80, 0x00]
    assert oracle.e4m3_encode(x).tolist() == want
    np.testing.assert_array_equal(oracle.e4m3_decode(np.array(want)), x.astype(np.float64))
    # saturation: everything above 448 in magnitude stays finite
    assert oracle.e4m3_encode(np.array([449.0, 464.0, 1e9, -1e30], np.float32)).tolist() == \
        [0x7E, 0x7E, 0x7E, 0xFE]
    assert np.isnan(oracle.e4m3_decode(np.array([0x7F, 0xFF]))).all()


def test_e4m3_round_trip_and_ties_to_even():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals.astype(np.float32)), codes)
    pos = np.arange(0, 0x7E, dtype=np.int64)            # c and c + 1 both finite, positive
    lo, hi = oracle.e4m3_decode(pos), oracle.e4m3_decode(pos + 1)
    mid = ((lo + hi) / 2).astype(np.float32)             # exact in fp32
    even = np.where(pos % 2 == 0, pos, pos + 1)
    np.testing.assert_array_equal(oracle.e4m3_encode(mid), even)
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    np.testing.assert_array_equal(oracle.e4m3_encode(up), pos + 1)
    np.testing.assert_array_equal(oracle.e4m3_encode(down), pos)


def test_e4m3_encode_matches_library_conversion():
    rng = np.random.default_rng(80)
    x = np.concatenate([rng.standard_normal(4000) * 30, rng.standard_normal(2000) * 0.01,
                        rng.uniform(-448, 448, 2000)]).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), lib)


def test_quantize_per_head_properties():
    rng = np.random.default_rng(81)
    x = (rng.standard_normal((2, 3, 50, 16)) * np.array([1.0, 0.01, 20.0])[None, :, None, None])
    x = x.astype(np.float32)
    x[1, 2] = 0.0                                          # an all-zero head
    codes, scale = oracle.quantize_e4m3_per_head(x)
    for b in range(2):
        for h in range(3):
            amax = np.abs(x[b, h]).max()
            if amax == 0:
                assert scale[b, h] == 1.0 and not codes[b, h].any()
                continue
            assert scale[b, h] == np.float32(amax) / np.float32(448)
            # the largest magnitude maps to the largest code
            i = np.unravel_index(np.argmax(np.abs(x[b, h])), x[b, h].shape)
            assert codes[b, h][i] & 0x7F == 0x7E
    deq = oracle.dequantize_e4m3(codes, scale)
    err = np.abs(deq - x)
    # relative 2^-4 in the normal range, half a subnormal step below it
    s = scale.astype(np.float64)[:, :, None, None]
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s) * (1 + 1e-6)
    assert np.all(err <= bound)


@pytest.mark.parametrize("S,W", [(4, 16), (0, 3)])
def test_fp8_bound_holds_for_a_simulated_kernel(S, W):
    """A numpy model of the kernel's arithmetic (probabilities in a unit c >=
    1, rounded to e4m3, unrounded row sum) stays within the bound, and the
    bound is far from vacuous."""
    rng = np.random.default_rng(82 + S)
    B, Hq, Hkv, N, d = 1, 2, 1, 96, 8
    q = rng.standard_normal((B, Hq, N, d)) * 2.5
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    mask = np.array([[0, 1]], np.uint8)
    ref = oracle.attention(q, k, v, mask, S, W)
    bound = oracle.fp8_p_rounding_bound(q, k, v, mask, S, W)
    scale = 1.0 / math.sqrt(d)
    for h in range(Hq):
        for i in range(N):
            keys = oracle.visible_keys(i, bool(mask[0, h]), S, W)
            s = (k[0, 0, keys] @ q[0, h, i]) * scale
            p = np.exp(s - s.max())
            c = 2.0 ** rng.uniform(0, 8)                  # the kernel's unit
            pq = oracle.e4m3_decode(oracle.e4m3_encode((p * c).astype(np.float32))) / c
            out = (pq @ v[0, 0, keys]) / p.sum()
            assert np.all(np.abs(out - ref[0, h, i]) <= bound[0, h, i] + 1e-12), (h, i)
    assert bound.mean() < 0.1 * np.abs(v).mean()


def test_fp8_bound_covers_flushed_probabilities():
    """One dominant key and 90 keys at p = 2^-11, which e4m3 flushes to zero
    in the unit c = 1: the error is the whole mass of those keys, which only
    the absolute (subnormal) term of the bound covers."""
    N = 91
    q = np.ones((1, 1, N, 1))
    k = np.full((1, 1, N, 1), math.log(2.0 ** -11))
    k[0, 0, 0, 0] = 0.0
    v = np.full((1, 1, N, 1), 10.0)
    v[0, 0, 0, 0] = 0.0
    mask = np.zeros((1, 1), np.uint8)
    ref = oracle.attention(q, k, v, mask, 0, 1, scale=1.0)
    bound = oracle.fp8_p_rounding_bound(q, k, v, mask, 0, 1, scale=1.0)
    s = k[0, 0, :, 0]
    p = np.exp(s - s.max())
    pq = oracle.e4m3_decode(oracle.e4m3_encode(p.astype(np.float32)))
    out = (pq @ v[0, 0, :, 0]) / p.sum()
    err = abs(out - ref[0, 0, N - 1, 0])
    assert err > 0.4                                   # the flushed mass
    assert err <= bound[0, 0, N - 1, 0]


def test_attention_fp8_dequantizes_before_attending():
    rng = np.random.default_rng(83)
    x = rng.standard_normal((3, 1, 2, 40, 8)).astype(np.float32)
    (qc, qs), (kc, ks), (vc, vs) = (oracle.quantize_e4m3_per_head(t) for t in x)
    mask = np.array([[0, 1]], np.uint8)
    # SA heads with S = 0, W = 1: every row attends to itself only, so out is
    # the dequantized v
    out = oracle.attention_fp8(qc, qs, kc, ks, vc, vs, np.ones_like(mask), 0, 1)
    np.testing.assert_allclose(out, oracle.dequantize_e4m3(vc, vs), rtol=0, atol=1e-12)
    full = oracle.attention_fp8(qc, qs, kc, ks, vc, vs, mask, 2, 5)
    ref = oracle.attention(oracle.dequantize_e4m3(qc, qs), oracle.dequantize_e4m3(kc, ks),
                           oracle.dequantize_e4m3(vc, vs), mask, 2, 5)
    np.testing.assert_allclose(full, ref, rtol=0, atol=0)


def test_fp8_bound_rows_equals_the_dense_bound():
    rng = np.random.default_rng(84)
    q = rng.standard_normal((1, 4, 70, 8))
    k = rng.standard_normal((1, 2, 70, 8))
    v = rng.standard_normal((1, 2, 70, 8))
    mask = np.array([[0, 1, 0, 1]], np.uint8)
    dense = oracle.fp8_p_rounding_bound(q, k, v, mask, 3, 9)
    rows = [0, 1, 5, 9, 12, 69]
    for h in range(4):
        np.testing.assert_allclose(
            oracle.fp8_p_rounding_bound_rows(q, k, v, mask, 0, h, rows, 3, 9), dense[0, h, rows],
            rtol=1e-12, atol=1e-15)
