"""The attention kernel computes a share of its softmax exponentials on the FMA pipe with a
cubic polynomial (exp2_fma in attn_tc.cu). This re-evaluates that exact float32 formula, with
the coefficients read from the kernel source, against numpy's exp2 (CPU only)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    with open(os.path.join(ROOT, "linear_video_world_b200", "csrc", "attn_tc.cu")) as fh:
        src = fh.read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("\n}\n")]
    m = re.search(r"fmaf\(fmaf\(fmaf\(([0-9.e+-]+)f, f, ([0-9.e+-]+)f\), f, ([0-9.e+-]+)f\), f, 1\.f\)", body)
    assert m, "polynomial not found"
    c3, c2, c1 = (np.float32(float(v)) for v in m.groups())
    return c1, c2, c3


C1, C2, C3 = _coeffs()


def exp2_fma(x):
    c1, c2, c3 = C1, C2, C3
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    # fmaf chains: evaluated in float64 then rounded once per step, as a fused multiply-add
    p = np.float32(np.float64(c3) * f + np.float64(c2))
    p = np.float32(np.float64(p) * f + np.float64(c1))
    p = np.float32(np.float64(p) * f + 1.0)
    e = (t.view(np.int32).astype(np.int64) << 23) & 0xFFFFFFFF
    return ((p.view(np.int32).astype(np.int64) + e) & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_fma_relative_error():
    x = np.linspace(-60.0, 8.0, 1_000_001).astype(np.float32)
    rel = np.abs(exp2_fma(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2e-4          # bf16 rounding of P is 2^-9 ~ 2e-3


def test_exp2_fma_integers_and_clamp():
    for n in range(-120, 9):
        assert abs(float(exp2_fma(np.array([n], np.float32))[0]) / 2.0 ** n - 1.0) < 2e-4
    tiny = exp2_fma(np.array([-1000.0, -200.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-36)
