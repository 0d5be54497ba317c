"""Pins of the oracle's FP8 (E4M3) quantisation to facts other than its own code.

The codec is checked against the format's definition worked by hand and against PyTorch's
float8_e4m3fn conversion (a library routine: round to nearest even); the quantisers against
the reconstruction bound of round-to-nearest, the block geometry (blocks never span frames)
and exactly representable cases in which quantisation loses nothing.
"""
import math

import numpy as np
import pytest
import torch


def _torch_codes(y):
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_for_every_code(orc):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.e4m3_values()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))   # 0x80 is -0


def test_e4m3_landmarks_from_the_format_definition(orc):
    # bias 7: 0.0111.000 = 2^(7-7) = 1; 0.1111.110 = 2^8 * 1.75 = 448 (0.1111.111 is NaN);
    # smallest normal 0.0001.000 = 2^-6; smallest subnormal 0.0000.001 = 1/8 * 2^-6 = 2^-9
    cases = {0x38: 1.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x07: 7 / 8 * 2.0 ** -6,
             0x30: 0.5, 0xC0: -2.0, 0x3C: 1.5, 0x77: 240.0, 0x00: 0.0}
    for c, v in cases.items():
        assert orc.e4m3_decode(c) == v, hex(c)
        assert orc.e4m3_encode(v) == c, hex(c)
    assert math.isnan(orc.e4m3_decode(0x7F)) and math.isnan(orc.e4m3_decode(0xFF))


def test_e4m3_encode_matches_torch_rounding_on_a_sweep(orc):
    vals = orc.e4m3_values()
    pos = np.sort(vals[:0x7F])
    mids = (pos[1:] + pos[:-1]) / 2                      # exact ties (representable in f32)
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(0))
    rng = np.random.default_rng(0)
    rand = (rng.standard_normal(3000) * rng.choice([1e-3, 0.05, 1, 30, 200], 3000)).astype(np.float32)
    rand = rand[np.abs(rand) <= 448]
    y = np.concatenate([mids32, up, dn, -mids32, -up, rand, pos.astype(np.float32)])
    got = np.array([orc.e4m3_encode(v) for v in y], dtype=np.uint8)
    assert np.array_equal(got, _torch_codes(y))


def test_e4m3_encode_saturates_and_keeps_sign(orc):
    for y in (449.0, 463.9, 464.0, 1000.0, 3.4e38, math.inf):
        assert orc.e4m3_encode(y) == 0x7E
        assert orc.e4m3_encode(-y) == 0xFE
    assert orc.e4m3_encode(math.nan) == 0x7F
    assert orc.e4m3_encode(-1e-5) == 0x80               # rounds to zero, keeps the sign
    assert orc.e4m3_encode(2.0 ** -10) == 0x00          # tie between 0 and 2^-9: even code
    assert orc.e4m3_encode(3 * 2.0 ** -10) == 0x02      # tie between 2^-9 and 2^-8: even code


def _blocks(L, frame, block):
    out = []
    for f0 in range(0, L, frame):
        f1 = min(f0 + frame, L)
        for r0 in range(f0, f1, block):
            out.append((f0 // frame, (r0 - f0) // block, r0, min(r0 + block, f1)))
    return out


@pytest.mark.parametrize("L,frame,block", [(300, 100, 64), (257, 257, 128), (64, 64, 64), (70, 7, 64)])
def test_quantize_rows_reconstruction_bound_and_block_geometry(orc, L, frame, block):
    rng = np.random.default_rng(L)
    x = (rng.standard_normal((2, L, 16)) * rng.choice([0.01, 1.0, 50.0], (2, L, 1))).astype(np.float32)
    c, s = orc.fp8_quantize_rows(x, frame, block)
    vals = orc.e4m3_values()
    for bh in range(2):
        for f, j, r0, r1 in _blocks(L, frame, block):
            xb = x[bh, r0:r1]
            amax = np.abs(xb).max()
            assert s[bh, f, j] == np.float32(amax) / np.float32(448)
            dq = vals[c[bh, r0:r1]]
            assert np.abs(dq).max() == 448.0                        # the block's largest maps to 448
            # round to nearest: half a step of the E4M3 grid (2^-4 relative, 2^-10 absolute
            # in code units below 2^-6), plus the f32 roundings of 448/amax and the product
            err = np.abs(dq * np.float64(s[bh, f, j]) - xb)
            assert np.all(err <= 2.0 ** -4 * np.abs(xb) * (1 + 2e-6) + 2.0 ** -10 * s[bh, f, j] * 1.001 + 1e-30)
    # the encoder inside the quantiser agrees with the library's rounding of x * (448/amax)
    true_amax = np.zeros((2, L), np.float32)
    for f, j, r0, r1 in _blocks(L, frame, block):
        true_amax[:, r0:r1] = np.abs(x[:, r0:r1]).max(axis=(1, 2))[:, None]
    inv = (np.float32(448) / true_amax).astype(np.float32)
    assert np.array_equal(c, _torch_codes((x * inv[..., None]).astype(np.float32)))


def test_quantize_rows_locality(orc):
    """Raising one element changes the scale of its block only and the codes of that block only."""
    L, frame, block = 300, 100, 64
    x = np.random.default_rng(3).standard_normal((1, L, 8)).astype(np.float32)
    c0, s0 = orc.fp8_quantize_rows(x, frame, block)
    x2 = x.copy()
    x2[0, 170, 3] = 40.0                    # frame 1, rows 164..199 form its block j = 1
    c1, s1 = orc.fp8_quantize_rows(x2, frame, block)
    diff_s = np.argwhere(s0 != s1)
    assert diff_s.tolist() == [[0, 1, 1]]
    rows = np.unique(np.argwhere(c0 != c1)[:, 1])
    assert rows.min() >= 164 and rows.max() <= 199 and rows.size > 10


def test_quantize_rows_shift_is_subtracted_first(orc):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 130, 32)).astype(np.float32) + 3.0
    sh = rng.standard_normal((2, 32)).astype(np.float32) + 3.0
    ca, sa = orc.fp8_quantize_rows(x, 130, 64, shift=sh)
    cb, sb = orc.fp8_quantize_rows((x - sh[:, None, :]).astype(np.float32), 130, 64)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)


def test_quantize_channels_bound_and_locality(orc):
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((3, 200, 12)) * rng.choice([0.1, 2.0, 30.0], (3, 1, 12))).astype(np.float32)
    c, s = orc.fp8_quantize_channels(x)
    vals = orc.e4m3_values()
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    dq = vals[c]
    assert np.all(np.abs(dq).max(axis=1) == 448.0)
    err = np.abs(dq * s[:, None, :].astype(np.float64) - x)
    assert np.all(err <= 2.0 ** -4 * np.abs(x) * (1 + 2e-6) + 2.0 ** -10 * s[:, None, :] * 1.001 + 1e-30)
    x2 = x.copy()
    x2[1, 50, 4] = 1e3
    c2, s2 = orc.fp8_quantize_channels(x2)
    assert np.argwhere(s != s2).tolist() == [[1, 4]]
    ch = np.unique(np.argwhere(c != c2)[:, [0, 2]], axis=0)
    assert ch.tolist() == [[1, 4]]


def test_zero_block_has_zero_scale_and_codes(orc):
    x = np.zeros((1, 128, 8), np.float32)
    x[0, 64:] = np.random.default_rng(1).standard_normal((64, 8))
    c, s = orc.fp8_quantize_rows(x, 128, 64)
    assert s[0, 0, 0] == 0 and np.all(c[0, :64] == 0)
    c, s = orc.fp8_quantize_channels(np.zeros((1, 10, 4), np.float32))
    assert np.all(s == 0) and np.all(c == 0)


def test_window_fp8_equals_window_attention_when_quantisation_is_exact(orc):
    """Inputs that are E4M3 values times a power of two per block (the block's largest being
    448 times that power) quantise without loss, so the FP8 attention must equal the plain
    attention of the same inputs: this pins the block-to-scale mapping of the dequantisation."""
    T, N, d = 3, 80, 16
    L = T * N
    rng = np.random.default_rng(11)
    vals = orc.e4m3_values()
    finite = vals[:0x7F]

    def exact(frame, block, per_channel=False):
        c = rng.choice(np.arange(0x7F), size=(1, L, d))
        sign = rng.choice([1.0, -1.0], size=(1, L, d))
        x = sign * finite[c]
        if per_channel:
            e = rng.integers(-8, -4, size=d)
            x[0, 0, :] = 448.0
            return (x * 2.0 ** e[None, None, :]).astype(np.float32)
        for f, j, r0, r1 in _blocks(L, frame, block):
            x[0, r0, 0] = 448.0
            x[0, r0:r1] *= 2.0 ** int(rng.integers(-9, -5))
        return x.astype(np.float32)

    q, k, v = exact(L, 128), exact(N, 64), exact(0, 0, per_channel=True)
    q8, qs = orc.fp8_quantize_rows(q, L, 128)
    k8, ks = orc.fp8_quantize_rows(k, N, 64)
    v8, vs = orc.fp8_quantize_channels(v)
    assert np.array_equal(orc.fp8_dequantize_rows(q8, qs, L, 128), q)
    assert np.array_equal(orc.fp8_dequantize_rows(k8, ks, N, 64), k)
    assert np.array_equal(orc.fp8_dequantize_channels(v8, vs), v)
    for w, r in ((2, 1), (2, 2)):
        got = orc.window_fp8(q8, qs, k8, ks, v8, vs, T, N, w, r)
        ref = orc.swa(q, k, v, T, N, w) if r == 1 else orc.dswa(q, k, v, T, N, w, r)
        assert np.array_equal(got, ref)
