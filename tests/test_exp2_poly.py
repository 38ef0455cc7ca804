"""The exp2 the attention kernel evaluates on the FMA pipe (range reduction
plus a degree-3 polynomial, csrc/ea_math.cuh), replayed step by step in
float32 with the header's own constants, against exp2 in float64."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_attention_head_b200", "csrc", "ea_math.cuh")


def constants():
    src = open(HDR).read()
    c = {}
    for name in ("c0", "c1", "c2", "c3", "kShift"):
        m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, src)
        assert m, name
        c[name] = np.float32(float(m.group(1)))
    return c


def emulate(x):
    c = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + c["kShift"]).astype(np.float32)
    r = (t - c["kShift"]).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = (c["c3"] * f + c["c2"]).astype(np.float32)
    p = (p * f + c["c1"]).astype(np.float32)
    p = (p * f + c["c0"]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_over_kernel_range():
    # the kernel feeds x = score * scale * log2(e) - reference max <= 8
    x = np.linspace(-125.0, 8.0, 1_000_001).astype(np.float32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 2.0 ** -13, rel.max()


def test_integers_and_masked_inputs():
    x = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_allclose(emulate(x), np.exp2(x.astype(np.float64)), rtol=1e-4)
    tiny = emulate(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)


def test_polynomial_is_a_fit_of_two_to_the_f():
    c = constants()
    f = np.linspace(-0.5, 0.5, 10001)
    p = ((float(c["c3"]) * f + float(c["c2"])) * f + float(c["c1"])) * f + float(c["c0"])
    rel = np.abs(p - np.exp2(f)) / np.exp2(f)
    assert rel.max() < 8e-5
