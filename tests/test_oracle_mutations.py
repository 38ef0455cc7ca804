"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins in test_oracle_pins.py catch every one of them."""
import importlib.util
import inspect
import os
import types

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "ea_oracle.py")

MUTATIONS = {
    "window_off_by_one_visible": ("return j < sink or (i - j) < window",
                                  "return j < sink or (i - j) <= window"),
    "window_off_by_one_blocked": ("vis &= (jj < sink) | ((ii - jj) < window)",
                                  "vis &= (jj < sink) | ((ii - jj) <= window)"),
    "window_off_by_one_rows": ("lo = max(0, i - window + 1)",
                               "lo = max(0, i - window)"),
    "causal_strict": ("if j > i:", "if j >= i:"),
    "gqa_modulo_mapping": ("    hk = h // g\n", "    hk = h % Hkv\n"),
    "gqa_modulo_mapping_blocked": ("            hk = h // g\n", "            hk = h % Hkv\n"),
    "scale_one_over_d": ("        scale = 1.0 / math.sqrt(d)\n    sparse = bool(mask[b, h])\n    rows",
                         "        scale = 1.0 / d\n    sparse = bool(mask[b, h])\n    rows"),
    "scale_one_over_d_blocked": ("        scale = 1.0 / math.sqrt(d)\n    out = np.empty((B, Hq, N, d)",
                                 "        scale = 1.0 / d\n    out = np.empty((B, Hq, N, d)"),
    "relu_dropped": ("h = np.where(pre > 0.0, pre, 0.0)", "h = pre"),
    "bias2_dropped": ("return h @ w2.T + b2", "return h @ w2.T"),
    "bias1_dropped": ("pre = x @ w1.T + b1", "pre = x @ w1.T"),
    "w1_transposed": ("pre = x @ w1.T + b1", "pre = x @ w1 + b1"),
    "tie_to_sparse": ("mask = (z > threshold)", "mask = (z >= threshold)"),
    "pool_divisor": ("return (total / N)", "return (total / (N - 1))"),
    "pool_flatten_order": ("return (total / N).reshape(B, Hkv * d)",
                           "return (total / N).transpose(0, 2, 1).reshape(B, Hkv * d)"),
    "sink_double_count": ("sink_end = min(sink, lo)", "sink_end = min(sink, i + 1)"),
    "softmax_unnormalised": ("return (e @ vals) / np.sum(e, axis=-1, keepdims=True)",
                             "return (e @ vals)"),
    "sink_ignored_blocked": ("vis &= (jj < sink) | ((ii - jj) < window)",
                             "vis &= ((ii - jj) < window)"),
    "ring_slot_unshifted": ("return sink + (p - sink) % window", "return sink + p % window"),
    "kv_policy_any": ("np.all(m.reshape(m.shape[0], hkv, g) != 0, axis=2)",
                      "np.any(m.reshape(m.shape[0], hkv, g) != 0, axis=2)"),
    "decode_gqa_modulo": ("            hk = h // g\n            keys = visible_keys",
                          "            hk = h % Hkv\n            keys = visible_keys"),
    "varlen_pool_total_divisor": ("x[b] = (total / n).reshape(Hkv * d)",
                                  "x[b] = (total / T).reshape(Hkv * d)"),
    "varlen_pool_drops_last_token": ("for t in range(cu[b], cu[b + 1]):",
                                     "for t in range(cu[b], cu[b + 1] - 1):"),
    "varlen_first_mask_row": ("np.asarray(mask)[b:b + 1]", "np.asarray(mask)[0:1]"),
    "varlen_heads_as_positions": ("qs = q[t0:t1].transpose(1, 0, 2)[None]",
                                  "qs = q[t0:t1].reshape(Hq, t1 - t0, d)[None]"),
    "bwd_missing_rowsum": ("ds = p * (dp - dd)", "ds = p * dp"),
    "bwd_dk_unscaled": ("dk[b, hk] += scale * (ds.T @ q[b, h])", "dk[b, hk] += ds.T @ q[b, h]"),
    "bwd_dv_untransposed": ("dv[b, hk] += p.T @ dout[b, h]", "dv[b, hk] += p @ dout[b, h]"),
    "bwd_gqa_overwrite": ("dv[b, hk] += p.T @ dout[b, h]", "dv[b, hk] = p.T @ dout[b, h]"),
    "bwd_sampled_missing_rowsum": ("ds = p * (vh[cols] @ doh[i] - dd[i])",
                                   "ds = p * (vh[cols] @ doh[i])"),
    "bwd_sampled_keys_strict": ("rows = np.arange(j, N)\n", "rows = np.arange(j + 1, N)\n"),
    "bwd_sampled_block_window": ("lo = max(0, i0 - window + 1)", "lo = max(0, i0 - window + 2)"),
    "bwd_sampled_dk_unscaled": ("dk[r] += scale * (ds @ qh[rows])", "dk[r] += ds @ qh[rows]"),
    "bwd_sampled_lse_unshifted": ("lse[i0:i1] = (m + np.log(tot))[:, 0]",
                                  "lse[i0:i1] = np.log(tot)[:, 0]"),
    "lse_without_max": ("out[b, h] = m + np.log(", "out[b, h] = np.log("),
    "ste_missing_tau": ("dz = dr * r_soft * (1.0 - r_soft) / tau",
                        "dz = dr * r_soft * (1.0 - r_soft)"),
    "ste_relu_mask_dropped": ("dpre = np.where(pre > 0.0, dh, 0.0)", "dpre = dh"),
    "ste_pool_not_divided": ("(dx / N).reshape(B, Hkv, 1, d)", "dx.reshape(B, Hkv, 1, d)"),
    "e4m3_ties_away": ("v = np.rint(a / quantum) * quantum", "v = np.floor(a / quantum + 0.5) * quantum"),
    "e4m3_no_saturation": ("a = np.minimum(np.abs(x), E4M3_MAX)", "a = np.abs(x)"),
    "e4m3_subnormal_quantum": ("e = np.maximum(ex - 1, -6)", "e = np.maximum(ex - 1, -7)"),
    "e4m3_bias_8": ("(1.0 + m / 8.0) * np.exp2(e - 7.0)", "(1.0 + m / 8.0) * np.exp2(e - 8.0)"),
    "quant_scale_inverted": ("scale[b, h] = amax / np.float32(E4M3_MAX)",
                             "scale[b, h] = np.float32(E4M3_MAX) / amax"),
    "quant_amax_signed": ("amax = np.float32(np.max(np.abs(x[b, h])))", "amax = np.float32(np.max(x[b, h]))"),
    "fp8_bound_relative_only": ("per = np.maximum(2.0 ** -4 * p, 2.0 ** -10 / ell)", "per = 2.0 ** -4 * p"),
    "fp8_attention_v_scale_of_k": ("dequantize_e4m3(v_codes, v_scale), mask, sink, window, scale)",
                                   "dequantize_e4m3(v_codes, k_scale), mask, sink, window, scale)"),
    "ste_diff_sign": ("diff = np.asarray(o_sa, dtype=np.float64) - np.asarray(o_fa",
                      "diff = np.asarray(o_fa, dtype=np.float64) - np.asarray(o_sa"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation {name} does not apply"
    src = src.replace(old, new, 1)
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


def _pin_calls():
    """Every pin with a fixed argument set (parametrised pins expanded)."""
    calls = []
    for fname, fn in inspect.getmembers(pins, inspect.isfunction):
        if not fname.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            calls.append((fname, fn, {}))
            continue
        argnames, values = params[0].args[0], params[0].args[1]
        names = [a.strip() for a in argnames.split(",")]
        for val in values:
            vals = val if isinstance(val, tuple) else (val,)
            calls.append((fname, fn, dict(zip(names, vals))))
    return calls


# a planted mistake may produce NaN or out-of-range values on the way to a
# failing pin; numpy's warnings about them are expected here
@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mutant = _mutant(name)
    monkeypatch.setattr(pins, "oracle", mutant)
    caught = []
    for fname, fn, kwargs in _pin_calls():
        try:
            fn(**kwargs)
        except Exception:       # an assertion, or a shape error from the slip
            caught.append(fname)
    assert caught, f"no pin catches mutation {name}"


def test_unmutated_oracle_passes_every_pin():
    assert pins.oracle is oracle
    for fname, fn, kwargs in _pin_calls():
        fn(**kwargs)
