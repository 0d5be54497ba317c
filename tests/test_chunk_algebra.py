"""The chunkwise (UT-transform) form of the gated delta rule, checked against the oracle.

The long-context explainer (llm-atlas, section 06: RetNet's parallel, recurrent and
chunkwise forms are equivalent; section 09: "parallel within a block, recurrent across
blocks") is the idea; the algebra below is derived from the token recurrence
S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T. Within a chunk with start state S0,
with g_t the running sum of log a and u_t = b_t (v_t - a_t S_{t-1} k_t):

    S_t = e^{g_t} S0 + sum_{i<=t} e^{g_t - g_i} u_i k_i^T
    (I + A) U = diag(b) V - diag(b e^g) K S0^T,   A_ti = b_t e^{g_t-g_i} k_t.k_i  (i < t)
    U = U' - W S0^T,  U' = T diag(b) V,  W = T diag(b e^g) K,  T = (I + A)^{-1}
    O = diag(e^g) Q S0^T + P U,  P_ti = e^{g_t - g_i} q_t.k_i  (i <= t)
    S_C = e^{g_C} S0 + U^T diag(e^{g_C - g}) K

This numpy restatement is test code only (the CUDA kernels implement the same algebra on
their own); it shows, on the CPU, that the chunk form reaches the recurrence's result for
any chunk length and a ragged last chunk, before any kernel relies on it.
"""
import numpy as np
import pytest


def chunk_form(q, k, v, a, b, S0, C):
    L, d = q.shape
    S = S0.copy()
    o = np.zeros((L, d))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        Q, K, V = q[sl], k[sl], v[sl]
        g = np.cumsum(np.log(a[sl]))
        n = g.size
        diff = g[:, None] - g[None, :]
        low = np.tril(np.ones((n, n)), -1)
        A = low * b[sl][:, None] * np.exp(np.where(low > 0, diff, 0)) * (K @ K.T)
        Tm = np.linalg.solve(np.eye(n) + A, np.eye(n))
        W = Tm @ (b[sl][:, None] * np.exp(g)[:, None] * K)
        Up = Tm @ (b[sl][:, None] * V)
        U = Up - W @ S.T
        inc = np.tril(np.ones((n, n)))
        P = inc * np.exp(np.where(inc > 0, diff, 0)) * (Q @ K.T)
        o[sl] = np.exp(g)[:, None] * (Q @ S.T) + P @ U
        S = np.exp(g[-1]) * S + U.T @ (np.exp(g[-1] - g)[:, None] * K)
    return o, S


@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_chunk_form_equals_recurrence(orc, C):
    rng = np.random.default_rng(20 + C)
    L, d = 150, 16
    q = rng.standard_normal((L, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, d))
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L))))
    b = 1 / (1 + np.exp(-rng.standard_normal(L)))
    q, k, v, a, b = (x.astype(np.float32) for x in (q, k, v, a, b))
    S0 = rng.standard_normal((d, d))
    o_ref, S_ref = orc.gdn(q[None], k[None], v[None], a[None], b[None], S0[None])
    o, S = chunk_form(*(x.astype(np.float64) for x in (q, k, v, a, b)), S0, C)
    np.testing.assert_allclose(o, o_ref[0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(S, S_ref[0], rtol=1e-9, atol=1e-10)


def test_chunk_form_strong_decay_no_overflow(orc):
    """Gates as strong as the 480P workload's over a 64-token chunk (e^{g} down to ~1e-22):
    only ratios e^{g_t - g_i} with t >= i are formed, so nothing overflows."""
    rng = np.random.default_rng(5)
    L, d = 128, 8
    q = rng.standard_normal((L, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, d))
    a = np.full(L, np.exp(-0.8))
    b = np.full(L, 0.5)
    q, k, v, a, b = (x.astype(np.float32) for x in (q, k, v, a, b))
    o_ref, S_ref = orc.gdn(q[None], k[None], v[None], a[None], b[None])
    o, S = chunk_form(*(x.astype(np.float64) for x in (q, k, v, a, b)), np.zeros((d, d)), 64)
    assert np.all(np.isfinite(o))
    np.testing.assert_allclose(o, o_ref[0], rtol=1e-9, atol=1e-12)
