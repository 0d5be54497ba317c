"""Pins of the oracle's attention backward to facts other than its own formulas: central finite
differences of a dense fp64 forward written here (full score matrix, -inf outside the window),
and two invariants of softmax attention (shifting every key by one vector leaves every output
unchanged, so the key gradients sum to zero; shifting every value by c shifts every output by
c, so the value gradients sum to the sum of the upstream gradients)."""
import math

import numpy as np
import pytest


def _allowed(T, N, w, r):
    fr = np.arange(T * N) // N
    dist = fr[:, None] - fr[None, :]
    return (dist >= 0) & (dist <= r * (w - 1)) & (dist % r == 0)


def _dense_loss(q, k, v, g, allowed, scale):
    s = (q @ k.T) * scale
    s = np.where(allowed, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return float(np.sum((p @ v) * g))


@pytest.mark.parametrize("T,N,d,w,r", [(3, 4, 6, 2, 1), (5, 3, 5, 3, 2), (4, 2, 4, 4, 1)])
def test_window_bwd_matches_finite_differences(orc, T, N, d, w, r):
    rng = np.random.default_rng(T * 10 + r)
    # float32-representable inputs (the oracle reads float32); the dense forward runs in fp64
    q, k, v, g = (rng.standard_normal((T * N, d)).astype(np.float32) for _ in range(4))
    scale = 1 / math.sqrt(d)
    dq, dk, dv = orc.window_bwd(q, k, v, g, T, N, w, r)
    allowed = _allowed(T, N, w, r)
    base = [x.astype(np.float64) for x in (q, k, v)]
    eps = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            xs_p = [b.copy() for b in base]
            xs_m = [b.copy() for b in base]
            xs_p[which][idx] += eps
            xs_m[which][idx] -= eps
            fd[idx] = (_dense_loss(*xs_p, g, allowed, scale) - _dense_loss(*xs_m, g, allowed, scale)) / (2 * eps)
        assert np.abs(fd - grad).max() <= 1e-6 * max(1.0, np.abs(grad).max()), which


def test_window_bwd_invariants(orc):
    rng = np.random.default_rng(9)
    T, N, d, w, r = 6, 7, 8, 3, 2
    q, k, v, g = (rng.standard_normal((2, T * N, d)).astype(np.float32) for _ in range(4))
    dq, dk, dv = orc.window_bwd(q, k, v, g, T, N, w, r)
    assert np.abs(dk.sum(axis=1)).max() < 1e-12
    assert np.abs(dv.sum(axis=1) - g.astype(np.float64).sum(axis=1)).max() < 1e-12


@pytest.mark.parametrize("T,N,d,w,r", [(3, 4, 6, 2, 1), (7, 3, 5, 3, 2)])
def test_window_lse_matches_dense_logsumexp(orc, T, N, d, w, r):
    rng = np.random.default_rng(3 + r)
    q, k = (rng.standard_normal((2, T * N, d)).astype(np.float32) for _ in range(2))
    got = orc.window_lse(q, k, T, N, w, r)
    allowed = _allowed(T, N, w, r)
    for b in range(2):
        s = (q[b].astype(np.float64) @ k[b].astype(np.float64).T) / math.sqrt(d)
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1)
        ref = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
        assert np.abs(got[b] - ref).max() < 1e-12
