"""Host checks of numeric constants compiled into the CUDA kernels (no GPU needed).

The bf16 window attention computes one pair in four of its exponentials on the FMA pipe:
x is range-reduced by Cody-Waite rounding (n = x rounded to the nearest integer, f = x - n in
[-1/2, 1/2]), 2^f comes from a cubic, and n is added to the exponent bits. The cubic's
coefficients are read from the kernel source here, and the reduction is replayed in float32.
The error must stay well below bf16's rounding of P (2^-9 relative).
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "linear_video_world_b200", "csrc", "attn_tc2.cu")


def _coefficients():
    with open(SRC) as f:
        src = f.read()
    c = {}
    for name in ("EXP2_C0", "EXP2_C1", "EXP2_C2", "EXP2_C3"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", src)
        assert m, name + " not found in attn_tc2.cu"
        c[name] = float(m.group(1))
    return c["EXP2_C0"], c["EXP2_C1"], c["EXP2_C2"], c["EXP2_C3"]


def test_cubic_relative_error_on_the_reduced_interval():
    c0, c1, c2, c3 = _coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    p = c0 + f * (c1 + f * (c2 + f * c3))
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= 7.6e-5
    # a plausible slip (a coefficient from another base, a dropped term) fails the bound
    assert np.abs((c0 + f * (c1 + f * c2)) / np.exp2(f) - 1.0).max() > 1e-3


def test_reduction_replayed_in_float32():
    c0, c1, c2, c3 = (np.float32(c) for c in _coefficients())
    sh = np.float32(12582912.0)                       # 1.5 * 2^23
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), [-np.inf, -300.0, 0.0, -0.5, 0.5]])
    x = x.astype(np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    t = (xc + sh).astype(np.float32)
    n = (t - sh).astype(np.float32)
    fr = (xc - n).astype(np.float32)
    assert np.all(np.abs(fr) <= 0.5)
    q = (c3 * fr + c2).astype(np.float32)
    q = (q * fr + c1).astype(np.float32)
    q = (q * fr + c0).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(xc.astype(np.float64))
    assert np.all(np.abs(y / ref - 1.0) <= 1e-4)
    # masked keys (-inf) and anything below the floor give about 2^-125, a normal float
    assert abs(y[-5] / 2.0 ** -125 - 1.0) <= 1e-4 and y[-4] == y[-5]
