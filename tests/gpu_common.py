"""Helpers shared by the GPU parity tests: tolerances, comparison, sampled
rows, and router-margin control (the margin check calls only the oracle)."""
import numpy as np
import torch

import oracle

# Output tolerance for bf16 output with fp32 accumulation (bf16 P.V operands):
# max |gpu - oracle| <= 1e-2 and mean |gpu - oracle| <= 1e-3.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
# Router logits: fp32 pooling and GEMVs against float64.
LOGIT_ABS = 1e-4
# Bit-exact masks need every oracle logit at least this far from the threshold.
MARGIN = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def few_key_rows_packed(cu, mask, Hq, sink, window, limit=4):
    """bool [T, Hq, 1]: output rows of a packed batch that see at most `limit`
    keys (each sequence's first rows), from the visibility definition."""
    T = cu[-1]
    few = np.zeros((T, Hq, 1), dtype=bool)
    for b in range(len(cu) - 1):
        for h in range(Hq):
            for i in range(min(limit, cu[b + 1] - cu[b])):
                n = len(oracle.visible_keys(i, bool(mask[b][h]), sink, window))
                few[cu[b] + i, h, 0] = n <= limit
    return few


def compare(out_gpu: torch.Tensor, ref: np.ndarray, label="", few_keys=False, few_rows=None):
    """Strict bound: max |err| <= 1e-2 and mean |err| <= 1e-3.

    few_keys: rows that see only a handful of keys (window <= 2) output values
    of the size of V itself, and rounding the output to bf16 alone moves a
    value by up to 2^-8 |out| (bf16 unit roundoff; 2^-9 on average), more
    than 1e-2 once |out| >= 2.6.  For such
    cases the bound adds that rounding: |err| <= 1e-2 + 2^-8 |ref| element-
    wise and mean |err| <= 1e-3 + mean(2^-9 |ref|).  few_rows marks such rows
    individually (the first rows of every sequence of a packed batch); the
    rest keep the strict bound."""
    got = f64(out_gpu)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{label}: non-finite output"
    err = np.abs(got - ref)
    mx, mean = float(err.max()), float(err.mean())
    if few_rows is not None:
        # rows seeing at most a handful of keys (few_rows, broadcastable) get
        # the few-key bound below; every other element the strict one
        few = np.broadcast_to(few_rows, err.shape)
        bound = np.where(few, MAX_ABS + 2.0 ** -8 * np.abs(ref), MAX_ABS)
        mean_bound = MEAN_ABS + float(np.mean(np.where(few, 2.0 ** -9 * np.abs(ref), 0.0)))
        assert np.all(err <= bound) and mean <= mean_bound, \
            f"{label}: max {mx:.3e} mean {mean:.3e} (strict rows max " \
            f"{float(np.where(few, 0.0, err).max()):.3e})"
        return mx, mean
    if few_keys:
        bound = MAX_ABS + 2.0 ** -8 * np.abs(ref)
        mean_bound = MEAN_ABS + float(np.mean(2.0 ** -9 * np.abs(ref)))
        assert np.all(err <= bound) and mean <= mean_bound, \
            f"{label}: max {mx:.3e} mean {mean:.3e} (few-key bound)"
    else:
        assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{label}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def sample_rows(N, S, W, n_random, seed):
    special = {0, 1, S - 1, S, W - 1, W, W + S - 1, W + S, 127, 128, 255, 256, N - 1}
    rng = np.random.default_rng(seed)
    rows = set(r for r in special if 0 <= r < N)
    rows.update(int(r) for r in rng.integers(0, N, size=n_random))
    return sorted(rows)


def margin_controlled_b2(k_f64, w1, b1, w2, b2, threshold=0.0, margin=MARGIN, shift=1e-2,
                         cu=None):
    """Return b2 shifted (per head, away from the threshold on its current side)
    until every oracle logit clears the margin; the routing is unchanged in
    sign.  Uses only the oracle.  With cu, k_f64 is a packed [T, Hkv, d]
    batch with sequence offsets cu."""
    b2 = np.array(b2, dtype=np.float64)
    for _ in range(8):
        if cu is None:
            _, z = oracle.router_decide(k_f64, w1, b1, w2, b2, threshold)
        else:
            _, z = oracle.router_decide_varlen(k_f64, cu, w1, b1, w2, b2, threshold)
        close = np.abs(z - threshold) < margin
        if not close.any():
            return b2
        heads = np.where(close.any(axis=0))[0]
        for h in heads:
            side = np.sign(np.mean(z[:, h] - threshold)) or 1.0
            b2[h] += side * shift
    raise AssertionError("could not establish the router margin")
