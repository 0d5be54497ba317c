"""Pins of the oracle's rotary position embedding (CPU only).

The rotation is pinned by what RoPE is for and by an independent formulation, not by
retyping the loop: the complex-exponential form (each pair as one complex number times
e^{i p theta}), the relative-position property (the dot product of a rotated query and key
depends only on the difference of their positions, so their Gram matrix over positions is
Toeplitz), norm preservation, the identity at position 0, the inverse, composition of two
rotations, the two-dimensional case (a plain rotation by p radians) and the per-frame reset
of the within-frame position.
"""
import numpy as np
import pytest

import oracle as orc


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def test_complex_exponential_form():
    x = _rand((2, 3, 40, 16), 1)
    N, base = 7, 500.0
    y = orc.rope(x, N, base=base, pos_mode=0)
    d = x.shape[-1]
    theta = base ** (-np.arange(d // 2) * 2.0 / d)
    p = (np.arange(x.shape[-2]) % N).astype(np.float64)
    z = x[..., 0::2].astype(np.float64) + 1j * x[..., 1::2].astype(np.float64)
    zr = z * np.exp(1j * p[:, None] * theta[None, :])
    assert np.allclose(y[..., 0::2], zr.real, atol=1e-12)
    assert np.allclose(y[..., 1::2], zr.imag, atol=1e-12)


def test_relative_position_gram_is_toeplitz():
    # the same query and the same key at every position (global positions): <R_m q, R_n k>
    # must depend on m - n only
    L, d = 24, 32
    q, k = _rand((d,), 2), _rand((d,), 3)
    Q = orc.rope(np.tile(q, (1, L, 1)), 1, pos_mode=1)[0]
    K = orc.rope(np.tile(k, (1, L, 1)), 1, pos_mode=1)[0]
    G = Q @ K.T
    for s in range(-L + 1, L):
        diag = np.diagonal(G, offset=s)
        assert np.allclose(diag, diag[0], atol=1e-10)
    # and at equal positions it is the unrotated product
    assert np.allclose(np.diagonal(G), float(q.astype(np.float64) @ k.astype(np.float64)), atol=1e-10)


def test_norms_identity_inverse_composition():
    x = _rand((1, 2, 50, 8), 4)
    y = orc.rope(x, 10, pos_mode=0)
    pairs = lambda a: np.hypot(a[..., 0::2], a[..., 1::2])
    assert np.allclose(pairs(y), pairs(x.astype(np.float64)), atol=1e-12)
    assert np.array_equal(y[..., ::10, :], x[..., ::10, :].astype(np.float64))   # position 0
    back = orc.rope(y.astype(np.float32), 10, pos_mode=0, sign=-1)
    assert np.allclose(back, x, atol=1e-6)                                        # f32 round of y
    # rotating twice at position l equals rotating once at position 2l (global positions):
    # place token l's vector at row 2l of a longer sequence and rotate that once
    x1 = _rand((1, 1, 12, 8), 5)
    twice = orc.rope(orc.rope(x1, 1, pos_mode=1).astype(np.float32), 1, pos_mode=1)
    spread = np.zeros((1, 1, 24, 8), dtype=np.float32)
    spread[..., ::2, :] = x1
    once = orc.rope(spread, 1, pos_mode=1)[..., ::2, :]
    assert np.allclose(twice, once, atol=1e-5)


def test_two_dimensional_case_is_a_rotation_by_p_radians():
    # d = 2: one pair with theta = base^0 = 1, so position p rotates by p radians
    x = np.tile(np.array([1.0, 0.0], dtype=np.float32), (1, 6, 1))
    y = orc.rope(x, 1, base=123.0, pos_mode=1)[0]
    p = np.arange(6)
    assert np.allclose(y[:, 0], np.cos(p), atol=1e-15)
    assert np.allclose(y[:, 1], np.sin(p), atol=1e-15)
    # d = 4, base 100: the second pair turns with theta = 100^(-1/2) = 0.1 per position
    x4 = np.tile(np.array([0.0, 0.0, 1.0, 0.0], dtype=np.float32), (1, 11, 1))
    y4 = orc.rope(x4, 1, base=100.0, pos_mode=1)[0]
    assert np.allclose(y4[10, 2:], [np.cos(1.0), np.sin(1.0)], atol=1e-15)


def test_within_frame_position_resets_each_frame():
    x = _rand((1, 1, 30, 8), 6)
    N = 10
    y = orc.rope(x, N, pos_mode=0)
    # token l + N sits at the same in-frame position as token l: same rotation
    same = orc.rope(np.concatenate([x[..., 10:20, :], x[..., 10:20, :]], axis=2), N, pos_mode=0)
    assert np.allclose(y[..., 10:20, :], same[..., 0:10, :], atol=1e-15)
    g = orc.rope(x, N, pos_mode=1)
    assert np.allclose(y[..., :N, :], g[..., :N, :])                 # first frame: both agree
    assert not np.allclose(y[..., N:, :], g[..., N:, :])


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        orc.rope(_rand((1, 4, 3), 7), 2)                              # odd d
    with pytest.raises(ValueError):
        orc.rope(_rand((1, 4, 4), 7), 2, base=1.0)
