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


def _gdn_loss(q, k, v, a, b, S0, g, gS):
    """Dense fp64 forward of the gated delta rule written here, loss = <dO, o> + <gS, S_L>."""
    S = S0.copy()
    loss = 0.0
    for t in range(q.shape[0]):
        S = a[t] * (S - b[t] * np.outer(S @ k[t], k[t])) + b[t] * np.outer(v[t], k[t])
        loss += float(g[t] @ (S @ q[t]))
    return loss + float(np.sum(gS * S))


def test_gdn_bwd_matches_finite_differences(orc):
    rng = np.random.default_rng(21)
    L, d = 7, 5
    q, k, v, g = (rng.standard_normal((L, d)).astype(np.float32) for _ in range(4))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    a = rng.uniform(0.3, 1.0, L).astype(np.float32)
    b = rng.uniform(0.1, 0.9, L).astype(np.float32)
    S0 = rng.standard_normal((d, d))
    gS = rng.standard_normal((d, d))
    dq, dk, dv, da, db, dS0 = orc.gdn_bwd(q, k, v, a, b, g, S0=S0, dS_final=gS)
    base = [x.astype(np.float64) for x in (q, k, v, a, b)] + [S0]
    grads = [dq, dk, dv, da, db, dS0]
    eps = 1e-6
    for which, grad in enumerate(grads):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            xp = [x.copy() for x in base]
            xm = [x.copy() for x in base]
            xp[which][idx] += eps
            xm[which][idx] -= eps
            fd[idx] = (_gdn_loss(*xp, g, gS) - _gdn_loss(*xm, g, gS)) / (2 * eps)
        assert np.abs(fd - grad).max() <= 1e-6 * max(1.0, np.abs(grad).max()), which


def test_gdn_bwd_zero_gates_cut_the_history(orc):
    """With a_3 = 0 the state before token 3 is forgotten: outputs from t = 3 on do not depend on
    S0 or on tokens 0..2, so their upstream gradients change neither dS0 nor the gradients of
    tokens 0..2."""
    rng = np.random.default_rng(4)
    L, d = 6, 4
    q, k, v, g = (rng.standard_normal((1, L, d)).astype(np.float32) for _ in range(4))
    a = np.full((1, L), 0.8, np.float32)
    b = np.full((1, L), 0.5, np.float32)
    a[0, 3] = 0.0
    S0 = rng.standard_normal((1, d, d))
    g2 = g.copy()
    g2[0, 3:] = 0
    full = orc.gdn_bwd(q, k, v, a, b, g, S0=S0)
    cut = orc.gdn_bwd(q, k, v, a, b, g2, S0=S0)
    assert np.abs(full[5] - cut[5]).max() < 1e-12                   # dS0
    for xf, xc in zip(full[:5], cut[:5]):                           # dq dk dv da db, tokens < 3
        assert np.abs(xf[0, :3] - xc[0, :3]).max() < 1e-12
    assert np.abs(cut[5]).max() > 0
