"""Plain, slow CPU oracle for Elastic Attention's prefill hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path.

What it computes, and where the pages define it
-----------------------------------------------
Sources are two pages about one method:

* the blog post "Elastic Attention：将 MoE 路由引入 Attention，让大模型长文本推理
  '该省省，该花花'" (bxzpzcl.cn), cited here as *EA blog*, and its copy with the
  results section on tiemojia.cn, cited as *EA blog (results copy)*;
* the explainer page "Elastic Attention: Test-time Adaptive Sparsity Ratios for
  Efficient Transformers" (gist.science), cited as *EA explainer*.

1. Attention Router (EA blog §2.1 "核心架构：Attention Router"): the router reads the
   layer's Key hidden states and a simple MLP emits one routing signal r per
   head; r = 0 sends the head to Full Attention (FA), r = 1 to Sparse
   Attention (SA).  The pages fix neither pooling, activation nor widths.
   Readings taken here (the plainest ones the text supports):
     - pooled input x[b] = mean over all N positions of K[b, :, n, :], flattened
       in (kv_head, channel) order;
     - h = ReLU(W1 x + b1), z = W2 h + b2 (nn.Linear convention, W is out x in);
     - hard decision r = 1 iff z > threshold (threshold 0), a tie goes to FA.
       Training uses Gumbel-Softmax with a straight-through estimator (EA blog
       §2.1, "训练Trick"); at inference no noise is drawn.
   The router size 0.27M parameters per layer for an 8B model (EA blog §2.2)
   matches 1024 -> 256 -> 32 with biases (270,624 parameters).

2. Full attention (EA blog §1 and §2.1): causal softmax attention over every
   earlier token, softmax(q k^T * scale + causal mask) v, scale = 1/sqrt(d).

3. Sparse attention (EA blog §1: heads that "only look locally or at a
   sliding window"): fixed here as streaming attention, S sink tokens plus a
   causal local window of W tokens.  Key j is visible from query i iff
   j <= i and (j < S or i - j < W).  The window counts the diagonal.

4. Result concat (EA blog §2.1 "结果融合"): every head writes its own slot of
   out[B, Hq, N, d]; there is no separate concat step.

GQA (not on the pages; the named backbones use it): query head h reads kv
head h // (Hq // Hkv).

Precision: everything in float64 from inputs the caller has already rounded
to bf16 (the tests convert the same bf16 tensors the GPU receives).

5. FP8 variant (not on the pages; a throughput variant of the same
   attention): Q, K, V are stored as e4m3 bytes with one fp32 scale per
   (batch, head).  What it computes is the attention of section 2/3 over the
   dequantized values code * scale.  The e4m3 format here is the 8-bit
   floating-point layout with 1 sign, 4 exponent (bias 7) and 3 mantissa bits,
   no infinities, the all-ones pattern as NaN, largest finite 448, smallest
   normal 2^-6 and subnormals m * 2^-9; conversion rounds to nearest, ties to
   even, and saturates to +-448.  A head is quantized with s = amax / 448 and
   codes e4m3(x * (448 / amax)), all in fp32.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "router_param_count",
    "router_pool",
    "router_mlp",
    "router_decide",
    "visible",
    "visible_spans",
    "visible_keys",
    "attention_rows",
    "attention",
    "attention_weights",
    "brute_force_attention",
    "count_visible_pairs",
    "kv_head_sparse",
    "compact_slot",
    "decode_step",
    "router_pool_varlen",
    "router_decide_varlen",
    "attention_varlen",
    "attention_lse",
    "attention_backward",
    "attention_backward_sampled",
    "router_gumbel_forward",
    "router_ste_backward",
    "e4m3_decode",
    "e4m3_encode",
    "quantize_e4m3_per_head",
    "dequantize_e4m3",
    "attention_fp8",
    "fp8_p_rounding_bound",
    "fp8_p_rounding_bound_rows",
]


# --------------------------------------------------------------------------
# Attention Router (EA blog §2.1; size from EA blog §2.2)
# --------------------------------------------------------------------------

def router_param_count(in_dim: int, hidden: int, out_dim: int) -> int:
    """Parameters of a two-layer MLP with biases (EA blog §2.2: 0.27M/layer)."""
    return in_dim * hidden + hidden + hidden * out_dim + out_dim


def router_pool(k: np.ndarray) -> np.ndarray:
    """Mean of the key states over the sequence.

    k: [B, Hkv, N, d] (float64 values of the bf16 keys).
    Returns x: [B, Hkv * d], flattened in (kv_head, channel) order.
    Written as an explicit sum over positions divided by N.
    """
    k = np.asarray(k, dtype=np.float64)
    B, Hkv, N, d = k.shape
    total = np.zeros((B, Hkv, d), dtype=np.float64)
    for n in range(N):
        total += k[:, :, n, :]
    return (total / N).reshape(B, Hkv * d)


def router_mlp(x: np.ndarray, w1: np.ndarray, b1: np.ndarray,
               w2: np.ndarray, b2: np.ndarray) -> np.ndarray:
    """z = W2 ReLU(W1 x + b1) + b2, per batch row.  W is [out, in]."""
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    b1 = np.asarray(b1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    b2 = np.asarray(b2, dtype=np.float64)
    pre = x @ w1.T + b1
    h = np.where(pre > 0.0, pre, 0.0)
    return h @ w2.T + b2


def router_decide(k, w1, b1, w2, b2, threshold: float = 0.0):
    """Route mask [B, Hq] (uint8, 1 = SA, 0 = FA) and the logits z [B, Hq].

    r = 1 (sparse) iff z > threshold; z == threshold routes to FA.
    """
    z = router_mlp(router_pool(k), w1, b1, w2, b2)
    mask = (z > threshold).astype(np.uint8)
    return mask, z


# --------------------------------------------------------------------------
# Visibility: FA = causal; SA = sink S + causal local window W (EA blog §1)
# --------------------------------------------------------------------------

def visible(i: int, j: int, sparse: bool, sink: int, window: int) -> bool:
    """Is key j visible from query i?  Square causal prefill, no offset."""
    if j > i:
        return False
    if not sparse:
        return True
    return j < sink or (i - j) < window


def visible_spans(i: int, sparse: bool, sink: int, window: int) -> list:
    """The keys query i sees as sorted, disjoint half-open spans [a, b)."""
    if not sparse:
        return [(0, i + 1)]
    lo = max(0, i - window + 1)
    spans = []
    sink_end = min(sink, lo)                       # sink keys left of the window
    if sink_end > 0:
        spans.append((0, sink_end))
    spans.append((lo, i + 1))
    return spans


def visible_keys(i: int, sparse: bool, sink: int, window: int) -> np.ndarray:
    """Sorted indices of the keys query i sees (each key once)."""
    return np.concatenate([np.arange(a, b) for a, b in
                           visible_spans(i, sparse, sink, window)])


def count_visible_pairs(n: int, sparse: bool, sink: int, window: int) -> int:
    """Number of visible (i, j) pairs of one head, by enumeration of rows."""
    return int(sum(len(visible_keys(i, sparse, sink, window)) for i in range(n)))


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _softmax_row_weighted(scores: np.ndarray, vals: np.ndarray) -> np.ndarray:
    """softmax(scores) @ vals for a block of rows; scores may hold -inf."""
    m = np.max(scores, axis=-1, keepdims=True)
    e = np.exp(scores - m)
    return (e @ vals) / np.sum(e, axis=-1, keepdims=True)


def attention_rows(q, k, v, mask, b: int, h: int, rows, sink: int, window: int,
                   scale: float | None = None) -> np.ndarray:
    """Output rows out[b, h, rows, :] in float64.

    Each row is an exact function of that row alone, so any subset of rows can
    be checked.  Scores use only the keys the row sees (EA blog §1, §2.1).
    """
    Hq = q.shape[1]
    Hkv = k.shape[1]
    d = q.shape[3]
    g = Hq // Hkv
    hk = h // g
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    sparse = bool(mask[b, h])
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), d), dtype=np.float64)
    qh = np.asarray(q[b, h], dtype=np.float64)
    kh = np.asarray(k[b, hk], dtype=np.float64)
    vh = np.asarray(v[b, hk], dtype=np.float64)
    for r, i in enumerate(rows):
        spans = visible_spans(int(i), sparse, sink, window)
        if len(spans) == 1:
            kk, vv = kh[spans[0][0]:spans[0][1]], vh[spans[0][0]:spans[0][1]]
        else:
            kk = np.concatenate([kh[j0:j1] for j0, j1 in spans])
            vv = np.concatenate([vh[j0:j1] for j0, j1 in spans])
        s = (kk @ qh[i]) * scale
        out[r] = _softmax_row_weighted(s[None, :], vv)[0]
    return out


def attention(q, k, v, mask, sink: int, window: int, scale: float | None = None,
              block: int = 256) -> np.ndarray:
    """Full output out[B, Hq, N, d] in float64.

    Rows are processed in blocks; each block forms scores against the union of
    the keys its rows may see and then applies the exact element mask, so the
    result equals the row-by-row definition.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, Hq, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            sparse = bool(mask[b, h])
            for i0 in range(0, N, block):
                i1 = min(N, i0 + block)
                if sparse:
                    lo = max(0, i0 - window + 1)
                    keys = np.concatenate([np.arange(min(sink, lo)),
                                           np.arange(lo, i1)])
                else:
                    keys = np.arange(i1)
                s = (q[b, h, i0:i1] @ k[b, hk, keys].T) * scale
                ii = np.arange(i0, i1)[:, None]
                jj = keys[None, :]
                vis = jj <= ii
                if sparse:
                    vis &= (jj < sink) | ((ii - jj) < window)
                s = np.where(vis, s, -np.inf)
                out[b, h, i0:i1] = _softmax_row_weighted(s, v[b, hk, keys])
    return out


def attention_weights(q, k, mask, b: int, h: int, sink: int, window: int,
                      scale: float | None = None) -> np.ndarray:
    """Dense N x N attention weights of one head (small N only)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    Hq, N, d = q.shape[1], q.shape[2], q.shape[3]
    g = Hq // k.shape[1]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    sparse = bool(mask[b, h])
    s = (q[b, h] @ k[b, h // g].T) * scale
    vis = np.array([[visible(i, j, sparse, sink, window) for j in range(N)]
                    for i in range(N)])
    s = np.where(vis, s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def brute_force_attention(q, k, v, mask, sink: int, window: int,
                          scale: float | None = None) -> np.ndarray:
    """Per-element loops, for N <= 64: independent of the blocked version."""
    B, Hq, N, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0])
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hq, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            sparse = bool(mask[b][h])
            for i in range(N):
                scores = []
                keys = []
                for j in range(N):
                    if visible(i, j, sparse, sink, window):
                        dot = 0.0
                        for c in range(d):
                            dot += float(q[b][h][i][c]) * float(k[b][hk][j][c])
                        scores.append(dot * scale)
                        keys.append(j)
                mx = max(scores)
                w = [math.exp(s - mx) for s in scores]
                tot = sum(w)
                for c in range(d):
                    acc = 0.0
                    for wj, j in zip(w, keys):
                        acc += wj * float(v[b][hk][j][c])
                    out[b, h, i, c] = acc / tot
    return out


# --------------------------------------------------------------------------
# Decode step with a per-head KV-cache policy (EA blog §3: the fused kernel
# lowers memory use; a head routed to SA only ever needs its S sink tokens
# and its last W tokens).  Readings: query position t of sequence b sees the
# same keys as prefill row t (FA: 0..t; SA: sink + window); a kv head keeps a
# compact sink + window cache iff every query head that reads it is SA.
# --------------------------------------------------------------------------

def kv_head_sparse(mask, hq: int, hkv: int) -> np.ndarray:
    """[B, Hkv] uint8: 1 iff all query heads of the kv group route to SA."""
    m = np.asarray(mask, dtype=np.uint8).reshape(-1, hq)
    g = hq // hkv
    return np.all(m.reshape(m.shape[0], hkv, g) != 0, axis=2).astype(np.uint8)


def compact_slot(p: int, sink: int, window: int) -> int:
    """Cache slot of position p in a sink + window cache: sinks stay put, the
    rest cycle through a ring of W slots after them."""
    if p < sink:
        return p
    return sink + (p - sink) % window


def decode_step(q, k_hist, v_hist, pos, mask, sink: int, window: int,
                scale: float | None = None) -> np.ndarray:
    """out[b, h, :] for one new token per sequence.

    q      : [B, Hq, d]      the new token's queries
    k_hist : [B, Hkv, L, d]  every key up to and including position pos[b]
    v_hist : [B, Hkv, L, d]
    pos    : [B]             the new token's position t_b (its key is at t_b)
    Each output is the prefill row t_b of the same head (EA blog §2.1: r
    decides FA or SA per head)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = k_hist.shape[1]
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, Hq, d), dtype=np.float64)
    for b in range(B):
        t = int(pos[b])
        for h in range(Hq):
            hk = h // g
            keys = visible_keys(t, bool(mask[b][h]), sink, window)
            kk = np.asarray(k_hist[b, hk], dtype=np.float64)[keys]
            vv = np.asarray(v_hist[b, hk], dtype=np.float64)[keys]
            s = (kk @ q[b, h]) * scale
            out[b, h] = _softmax_row_weighted(s[None, :], vv)[0]
    return out


# --------------------------------------------------------------------------
# Packed variable-length batches.  A serving prefill batch is ragged: sequence
# b holds tokens [cu[b], cu[b+1]) of packed tensors q [T, Hq, d] and k, v
# [T, Hkv, d] (token-major, heads, channels).  The method routes per input
# (EA blog §2.1), so each sequence is its own square causal prefill: its
# router input is the mean of its own keys, and its attention sees only its
# own tokens, positions counted from the sequence's first token.  Reading
# taken for an empty sequence: its pooled keys are zero (no tokens), so its
# routing comes from the biases alone, and it has no output rows.
# --------------------------------------------------------------------------

def router_pool_varlen(k_packed, cu_seqlens) -> np.ndarray:
    """x [B, Hkv * d]: per sequence, the explicit sum of its key rows divided
    by its length (zeros for an empty sequence)."""
    k = np.asarray(k_packed, dtype=np.float64)
    cu = [int(c) for c in cu_seqlens]
    B = len(cu) - 1
    T, Hkv, d = k.shape
    x = np.zeros((B, Hkv * d), dtype=np.float64)
    for b in range(B):
        n = cu[b + 1] - cu[b]
        if n <= 0:
            continue
        total = np.zeros((Hkv, d), dtype=np.float64)
        for t in range(cu[b], cu[b + 1]):
            total += k[t]
        x[b] = (total / n).reshape(Hkv * d)
    return x


def router_decide_varlen(k_packed, cu_seqlens, w1, b1, w2, b2, threshold: float = 0.0):
    """Route mask [B, Hq] and logits z [B, Hq] of a packed batch."""
    z = router_mlp(router_pool_varlen(k_packed, cu_seqlens), w1, b1, w2, b2)
    return (z > threshold).astype(np.uint8), z


def attention_varlen(q, k, v, cu_seqlens, mask, sink: int, window: int,
                     scale: float | None = None, block: int = 256) -> np.ndarray:
    """out [T, Hq, d] in float64: every sequence's tokens attend within the
    sequence, each head in its own mode (mask [B, Hq])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cu = [int(c) for c in cu_seqlens]
    T, Hq, d = q.shape
    out = np.zeros((T, Hq, d), dtype=np.float64)
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        if t1 <= t0:
            continue
        # [n, H, d] -> [1, H, n, d]: the sequence as a batch of one
        qs = q[t0:t1].transpose(1, 0, 2)[None]
        ks = k[t0:t1].transpose(1, 0, 2)[None]
        vs = v[t0:t1].transpose(1, 0, 2)[None]
        o = attention(qs, ks, vs, np.asarray(mask)[b:b + 1], sink, window, scale, block)
        out[t0:t1] = o[0].transpose(1, 0, 2)
    return out


# --------------------------------------------------------------------------
# Backward pass (training).  EA blog §2.1, training trick: the discrete
# routing decision is made differentiable with Gumbel-Softmax and a
# straight-through estimator.  Readings taken here (the pages give no
# formula): one logit z per head is the two-class pair (0, z); with Gumbel
# noise g0, g1 (drawn by the caller and passed in) and temperature tau,
#   r_soft = sigmoid((z + g1 - g0) / tau),   r_hard = [z + g1 - g0 > 0];
# the forward uses r_hard (out = r_hard O_SA + (1 - r_hard) O_FA per head)
# and the backward differentiates r_soft, so that
#   dL/dr = sum over the head's rows and channels of dO * (O_SA - O_FA),
#   dL/dz = dL/dr * r_soft (1 - r_soft) / tau,
# and the gradient reaches the attention of the selected mode only.
# --------------------------------------------------------------------------

def _head_probs(q, k, mask, b, h, sink, window, scale):
    """Dense softmax probabilities [N, N] of one head (zeros off the pattern)."""
    Hq, N = q.shape[1], q.shape[2]
    g = Hq // k.shape[1]
    s = (q[b, h] @ k[b, h // g].T) * scale
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = j <= i
    if mask[b, h]:
        vis &= (j < sink) | ((i - j) < window)
    s = np.where(vis, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=1, keepdims=True), s


def attention_lse(q, k, mask, sink: int, window: int, scale: float | None = None) -> np.ndarray:
    """[B, Hq, N]: natural log of sum_j exp(scale q_i . k_j) over visible j."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, Hq, N, d = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, Hq, N), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            _, s = _head_probs(q, k, mask, b, h, sink, window, scale)
            m = np.max(s, axis=1)
            out[b, h] = m + np.log(np.sum(np.exp(s - m[:, None]), axis=1))
    return out


def attention_backward(q, k, v, dout, mask, sink: int, window: int,
                       scale: float | None = None):
    """(dq [B,Hq,N,d], dk [B,Hkv,N,d], dv [B,Hkv,N,d]) of L = sum(dout * out),
    out = attention(q, k, v, mask, ...); per head in its own mode, a kv
    head's gradients summed over its query heads.  Dense per head (small N):
      P = softmax(scale q k^T | visible), dV = P^T dO, dP = dO V^T,
      D_i = sum_c dO_ic O_ic, dS = P * (dP - D), dQ = scale dS K,
      dK = scale dS^T Q."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            p, _ = _head_probs(q, k, mask, b, h, sink, window, scale)
            o = p @ v[b, hk]
            dv[b, hk] += p.T @ dout[b, h]
            dp = dout[b, h] @ v[b, hk].T
            dd = np.sum(dout[b, h] * o, axis=1, keepdims=True)
            ds = p * (dp - dd)
            dq[b, h] = scale * (ds @ k[b, hk])
            dk[b, hk] += scale * (ds.T @ q[b, h])
    return dq, dk, dv


def _visible_grid(rows, cols, sparse: bool, sink: int, window: int) -> np.ndarray:
    """bool [len(rows), len(cols)]: visible(i, j) for every pair, elementwise."""
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.asarray(cols, dtype=np.int64)[None, :]
    vis = j <= i
    if sparse:
        vis &= (j < sink) | ((i - j) < window)
    return vis


def attention_backward_sampled(q, k, v, dout, mask, b: int, hk: int, q_rows, key_rows,
                               sink: int, window: int, scale: float | None = None,
                               block: int = 512):
    """Sampled gradients of L = sum(dout * out) for one kv group (batch b, kv
    head hk) at any N, from the same definitions as attention_backward:
    (dq [G, len(q_rows), d] for the group's query heads at rows q_rows,
     dk [len(key_rows), d], dv [len(key_rows), d] of kv head hk at key_rows).

    Per query head h of the group and per row i, over the keys i sees:
      P_ij = exp(scale q_i.k_j - lse_i),  O_i = sum_j P_ij v_j,
      D_i = dO_i . O_i,  dS_ij = P_ij (dO_i . v_j - D_i);
    then dq_i = scale sum_j dS_ij k_j, and for a key j the sums run over the
    rows i that see j and over the group's query heads:
      dv_j = sum_h sum_i P_ij dO_i,  dk_j = scale sum_h sum_i dS_ij q_i.
    lse_i and D_i come first, for every row: rows are taken in blocks, each
    block's scores formed against the key range its rows may see with the
    exact element mask applied, so every row's values are those of the
    row-by-row definition."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    kh, vh = k[b, hk], v[b, hk]
    q_rows = np.asarray(q_rows, dtype=np.int64)
    key_rows = np.asarray(key_rows, dtype=np.int64)
    dq = np.zeros((g, len(q_rows), d))
    dk = np.zeros((len(key_rows), d))
    dv = np.zeros((len(key_rows), d))
    for hh in range(g):
        h = hk * g + hh
        sparse = bool(mask[b, h])
        qh, doh = q[b, h], dout[b, h]
        lse = np.empty(N)
        dd = np.empty(N)
        for i0 in range(0, N, block):
            i1 = min(N, i0 + block)
            rows = np.arange(i0, i1)
            # keys any row of the block may see: [0, i1) for FA; the sinks and
            # [i0 - window + 1, i1) for SA
            if sparse:
                lo = max(0, i0 - window + 1)
                cols = np.unique(np.concatenate([np.arange(0, min(sink, i1)),
                                                 np.arange(lo, i1)]))
            else:
                cols = np.arange(0, i1)
            sc = (qh[rows] @ kh[cols].T) * scale
            sc = np.where(_visible_grid(rows, cols, sparse, sink, window), sc, -np.inf)
            m = np.max(sc, axis=1, keepdims=True)
            e = np.exp(sc - m)
            tot = np.sum(e, axis=1, keepdims=True)
            lse[i0:i1] = (m + np.log(tot))[:, 0]
            o = (e / tot) @ vh[cols]
            dd[i0:i1] = np.sum(doh[rows] * o, axis=1)
        for r, i in enumerate(q_rows):
            cols = visible_keys(int(i), sparse, sink, window)
            p = np.exp((kh[cols] @ qh[i]) * scale - lse[i])
            ds = p * (vh[cols] @ doh[i] - dd[i])
            dq[hh, r] = scale * (ds @ kh[cols])
        for r, j in enumerate(key_rows):
            j = int(j)
            rows = np.arange(j, N)
            rows = rows[_visible_grid(rows, [j], sparse, sink, window)[:, 0]]
            if len(rows) == 0:
                continue
            p = np.exp((qh[rows] @ kh[j]) * scale - lse[rows])
            dv[r] += p @ doh[rows]
            ds = p * (doh[rows] @ vh[j] - dd[rows])
            dk[r] += scale * (ds @ qh[rows])
    return dq, dk, dv


def router_gumbel_forward(k, w1, b1, w2, b2, g0, g1, tau: float):
    """Training-time routing: (r_hard [B,Hq] uint8, r_soft [B,Hq], z [B,Hq])."""
    z = router_mlp(router_pool(k), w1, b1, w2, b2)
    u = (z + np.asarray(g1, dtype=np.float64) - np.asarray(g0, dtype=np.float64)) / tau
    # exp(-u) overflows to inf for u < -709, where the sigmoid is 0 anyway
    with np.errstate(over="ignore"):
        r_soft = 1.0 / (1.0 + np.exp(-u))
    r_hard = (u > 0.0).astype(np.uint8)
    return r_hard, r_soft, z


def router_ste_backward(k, w1, b1, w2, b2, g0, g1, tau: float, dout, o_fa, o_sa):
    """Router gradients through the straight-through estimator.

    dout, o_fa, o_sa: [B, Hq, N, d] (the layer's output gradient and both
    modes' outputs).  Returns (dr [B,Hq], dz [B,Hq], dw1, db1, dw2, db2,
    dk_router [B,Hkv,N,d]) where dk_router is the keys' gradient through the
    pooling (each position gets dx / N)."""
    k = np.asarray(k, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    b1 = np.asarray(b1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    B, Hkv, N, d = k.shape
    dout = np.asarray(dout, dtype=np.float64)
    diff = np.asarray(o_sa, dtype=np.float64) - np.asarray(o_fa, dtype=np.float64)
    dr = np.sum(dout * diff, axis=(2, 3))
    _, r_soft, _ = router_gumbel_forward(k, w1, b1, w2, b2, g0, g1, tau)
    dz = dr * r_soft * (1.0 - r_soft) / tau
    x = router_pool(k)
    pre = x @ w1.T + b1
    h = np.where(pre > 0.0, pre, 0.0)
    dw2 = dz.T @ h
    db2 = np.sum(dz, axis=0)
    dh = dz @ w2
    dpre = np.where(pre > 0.0, dh, 0.0)
    dw1 = dpre.T @ x
    db1 = np.sum(dpre, axis=0)
    dx = dpre @ w1
    dk_router = np.broadcast_to((dx / N).reshape(B, Hkv, 1, d), (B, Hkv, N, d)).copy()
    return dr, dz, dw1, db1, dw2, db2, dk_router


# --------------------------------------------------------------------------
# FP8 (e4m3) variant: codec, per-head quantization, reference and the error
# bound of an e4m3 probability matrix
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of each e4m3 byte (NaN for 0x7f / 0xff)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & ((c & 7) == 7), np.nan, val)
    return sign * val


def e4m3_encode(x) -> np.ndarray:
    """uint8 e4m3 codes of fp32 values: round to nearest, ties to even, magnitudes
    above 448 saturate to 448; the sign of a zero result is kept."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # binade of a (at least the subnormal one, 2^-6 with quantum 2^-9)
    _, ex = np.frexp(a)                      # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)
    quantum = np.exp2(e - 3.0)
    v = np.rint(a / quantum) * quantum       # rint: ties to even (448 stays 448)
    # code: subnormals (and 2^-6 itself) are v / 2^-9; normals (E << 3) | M
    _, ev = np.frexp(v)
    en = ev - 1
    normal = v >= 2.0 ** -6
    m_norm = np.where(normal, v / np.exp2(en) * 8.0 - 8.0, 0.0)
    code = np.where(normal, ((en + 7) << 3) + m_norm.astype(np.int64),
                    (v / 2.0 ** -9).astype(np.int64))
    code = np.where(np.isnan(x), 0x7F, code)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def quantize_e4m3_per_head(x):
    """x: [B, H, N, d] (values already exact in fp32).  Per (b, h): amax =
    max |x|, inv = 448 / amax and scale = amax / 448 in fp32 (1 and 1 when
    amax = 0), codes = e4m3(fp32(x * inv)).  Returns (codes uint8, scale
    float32 [B, H])."""
    x = np.asarray(x, dtype=np.float32)
    B, H = x.shape[:2]
    codes = np.empty(x.shape, dtype=np.uint8)
    scale = np.empty((B, H), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            amax = np.float32(np.max(np.abs(x[b, h]))) if x[b, h].size else np.float32(0)
            if amax > 0:
                inv = np.float32(E4M3_MAX) / amax
                scale[b, h] = amax / np.float32(E4M3_MAX)
            else:
                inv = np.float32(1.0)
                scale[b, h] = np.float32(1.0)
            codes[b, h] = e4m3_encode((x[b, h] * inv).astype(np.float32))
    return codes, scale


def dequantize_e4m3(codes, scale) -> np.ndarray:
    """float64 code * scale, scale per (b, h) of [B, H, N, d] codes."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, :, None, None]


def attention_fp8(q_codes, q_scale, k_codes, k_scale, v_codes, v_scale, mask, sink: int,
                  window: int, scale: float | None = None) -> np.ndarray:
    """The FP8 variant's result: the attention of the dequantized Q, K, V."""
    return attention(dequantize_e4m3(q_codes, q_scale), dequantize_e4m3(k_codes, k_scale),
                     dequantize_e4m3(v_codes, v_scale), mask, sink, window, scale)


def fp8_p_rounding_bound(q, k, v, mask, sink: int, window: int,
                         scale: float | None = None) -> np.ndarray:
    """Elementwise bound [B, Hq, N, d] on how far a kernel that rounds the
    probabilities to e4m3 before the P.V product can be from the exact result.

    Exact weights: w_j = p_j / l with p_j = exp(s_j - m) over the row's
    visible keys, m the row max and l = sum p_j (>= 1, the max term is 1).
    The kernel works in a unit c >= 1 (its running reference max is at or
    below the row max) and forms sum_j e4m3(c p_j) v_j / (c l): the
    probabilities are rounded, the row sum is not.  e4m3 rounding moves a
    normal value by at most 2^-4 of itself and a subnormal one by at most
    2^-10 (half its spacing), so |e4m3(c p_j) - c p_j| <= max(2^-4 c p_j,
    2^-10) and
        |out - out*| <= sum_j max(2^-4 w_j, 2^-10 / (c l)) |v_j|
                     <= sum_j max(2^-4 w_j, 2^-10 / l) |v_j|.
    Returns that last sum per element."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, N, d = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    g = Hq // k.shape[1]
    out = np.empty((B, Hq, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            p, s = _head_probs(q, k, mask, b, h, sink, window, scale)
            vis = np.isfinite(s)
            m = np.max(s, axis=1, keepdims=True)
            ell = np.sum(np.where(vis, np.exp(s - m), 0.0), axis=1, keepdims=True)
            per = np.maximum(2.0 ** -4 * p, 2.0 ** -10 / ell)
            per = np.where(vis, per, 0.0)
            out[b, h] = per @ np.abs(v[b, h // g])
    return out


def fp8_p_rounding_bound_rows(q, k, v, mask, b: int, h: int, rows, sink: int, window: int,
                              scale: float | None = None) -> np.ndarray:
    """fp8_p_rounding_bound for the listed query rows of head (b, h) only
    ([len(rows), d]), computed row by row from the visible keys."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, N, d = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    g = Hq // np.asarray(k).shape[1]
    kh = np.asarray(k[b, h // g], dtype=np.float64)
    vh = np.asarray(v[b, h // g], dtype=np.float64)
    out = np.empty((len(rows), d), dtype=np.float64)
    for r, i in enumerate(rows):
        keys = visible_keys(int(i), bool(mask[b, h]), sink, window)
        s = (kh[keys] @ q[b, h, i]) * scale
        e = np.exp(s - np.max(s))
        ell = np.sum(e)
        per = np.maximum(2.0 ** -4 * e / ell, 2.0 ** -10 / ell)
        out[r] = per @ np.abs(vh[keys])
    return out
