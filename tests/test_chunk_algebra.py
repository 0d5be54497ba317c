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


def test_segment_maps_compose_to_the_recurrence(orc):
    """The two-level scan the GPU pass over the chunks uses: the map of a run of tokens is
    affine in the start state (rows of S evolve independently), S_end = S_start A + B, with
    A = the run from the identity with v = 0 (every write U is linear in v, so Up = 0) and
    B = the run from zero with v. Composing the maps of consecutive segments serially gives
    each segment's true start state, and replaying a segment from it gives the recurrence's
    outputs (llm-atlas long-context explainer, section 09: state passing as composed
    transitions). Ragged segment lengths, slow decay so the maps stay far from zero."""
    rng = np.random.default_rng(11)
    L, d = 230, 12
    q = rng.standard_normal((L, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, d))
    a = np.exp(-0.05 * np.log1p(np.exp(rng.standard_normal(L))))
    b = 1 / (1 + np.exp(-rng.standard_normal(L)))
    q, k, v, a, b = (x.astype(np.float32) for x in (q, k, v, a, b))
    S0 = rng.standard_normal((d, d))
    o_all, S_all = orc.gdn(q[None], k[None], v[None], a[None], b[None], S0[None])
    cuts = [0, 64, 100, 192, L]
    S = S0.copy()
    zero_v = np.zeros_like(v)
    for s0, s1 in zip(cuts[:-1], cuts[1:]):
        sl = slice(s0, s1)
        # replay from the composed start state: the recurrence's outputs on this segment
        o_seg, _ = orc.gdn(q[None, sl], k[None, sl], v[None, sl], a[None, sl], b[None, sl], S[None])
        np.testing.assert_allclose(o_seg[0], o_all[0, sl], rtol=1e-9, atol=1e-10)
        _, Am = orc.gdn(q[None, sl], k[None, sl], zero_v[None, sl], a[None, sl], b[None, sl],
                        np.eye(d)[None])
        _, Bm = orc.gdn(q[None, sl], k[None, sl], v[None, sl], a[None, sl], b[None, sl],
                        np.zeros((1, d, d)))
        S = S @ Am[0] + Bm[0]
    np.testing.assert_allclose(S, S_all[0], rtol=1e-9, atol=1e-10)


# --------------------------------------------------------------------------------------
# Backward pass in chunk form
# --------------------------------------------------------------------------------------
# Reverse-mode derivative of the chunk form above, term by term (derived here from it; the
# kernels implement the same algebra). Per chunk, with R = diag(b)(V - diag(e^g) K S0^T)
# (so U = T R), Qt = diag(e^g) Q - P W, Kt = diag(e^{g_C - g}) K and dS_C the gradient of the
# chunk's end state:
#   across chunks (serial, last to first): dS0 = dS_C (gamma I - Kt^T W) + dO^T Qt
#   within a chunk (parallel):
#     dU = P^T dO + Kt dS_C^T,  dR = T^T dU,  dA = -(dR U^T) on s < t,  dP = dO U^T on s <= t
#     dQ = diag(e^g) dO S0 + (dP o Gam) K
#     dK = (dP o Gam)^T Q + diag(e^{g_C - g}) U dS_C + M K + M^T K - diag(b e^g) dR S0,
#          M = dA o (b_t e^{g_t - g_s})
#     dV = diag(b) dR
#     db = rowsum(dA o Gam o K K^T) + rowsum(dR o (V - diag(e^g) K S0^T))
#     dg = rowsum - colsum of (dP o P) and of (dA o A) + e^g o rowsum(dO o Q S0^T)
#          - b e^g o rowsum(dR o K S0^T) - e^{g_C - g} o rowsum(U o K dS_C^T)
#          + [last token] (gamma <dS_C, S0> + sum_s e^{g_C - g_s} u_s^T dS_C k_s)
#     d(log a) = reverse running sum of dg inside the chunk;  da = d(log a) / a

def chunk_backward(q, k, v, a, b, S0, dO, dSL, C):
    L, d = q.shape
    S = S0.copy()
    chunks = []
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        Q, K, V, G = q[sl], k[sl], v[sl], dO[sl]
        bb = b[sl]
        g = np.cumsum(np.log(a[sl]))
        n = g.size
        diff = g[:, None] - g[None, :]
        low = np.tril(np.ones((n, n)), -1)
        inc = np.tril(np.ones((n, n)))
        E_low = low * np.exp(np.where(low > 0, diff, 0))
        Gam = inc * np.exp(np.where(inc > 0, diff, 0))
        A = bb[:, None] * E_low * (K @ K.T)
        Tm = np.linalg.solve(np.eye(n) + A, np.eye(n))
        W = Tm @ ((bb * np.exp(g))[:, None] * K)
        Up = Tm @ (bb[:, None] * V)
        P = Gam * (Q @ K.T)
        Qt = np.exp(g)[:, None] * Q - P @ W
        Kt = np.exp(g[-1] - g)[:, None] * K
        chunks.append(dict(sl=sl, Q=Q, K=K, V=V, G=G, b=bb, a=a[sl], g=g, E_low=E_low, Gam=Gam,
                           A=A, T=Tm, W=W, Up=Up, P=P, Qt=Qt, Kt=Kt, S0=S.copy()))
        U = Up - W @ S.T
        S = np.exp(g[-1]) * S + U.T @ Kt
    dS = np.zeros((d, d)) if dSL is None else dSL.copy()
    for ch in reversed(chunks):
        ch["dSC"] = dS.copy()
        dS = dS @ (np.exp(ch["g"][-1]) * np.eye(d) - ch["Kt"].T @ ch["W"]) + ch["G"].T @ ch["Qt"]
    dS0 = dS
    dq, dk, dv = (np.zeros((L, d)) for _ in range(3))
    da, db = np.zeros(L), np.zeros(L)
    for ch in chunks:
        Q, K, V, G, bb, g, S0c, dSC = (ch[x] for x in ("Q", "K", "V", "G", "b", "g", "S0", "dSC"))
        U = ch["Up"] - ch["W"] @ S0c.T
        dU = ch["P"].T @ G + ch["Kt"] @ dSC.T
        dR = ch["T"].T @ dU
        inc = ch["Gam"] > 0
        low = ch["E_low"] > 0
        dP = np.where(inc, G @ U.T, 0.0)
        dA = np.where(low, -(dR @ U.T), 0.0)
        eg = np.exp(g)
        dQc = eg[:, None] * (G @ S0c) + (dP * ch["Gam"]) @ K
        M = dA * bb[:, None] * ch["E_low"]
        KS = K @ S0c.T
        dKc = (dP * ch["Gam"]).T @ Q + np.exp(g[-1] - g)[:, None] * (U @ dSC) + M @ K + M.T @ K \
            - (bb * eg)[:, None] * (dR @ S0c)
        dVc = bb[:, None] * dR
        dbc = (dA * ch["E_low"] * (K @ K.T)).sum(1) + (dR * (V - eg[:, None] * KS)).sum(1)
        PP, AA = dP * ch["P"], dA * ch["A"]
        dg = PP.sum(1) - PP.sum(0) + AA.sum(1) - AA.sum(0) + eg * (G * (Q @ S0c.T)).sum(1) \
            - bb * eg * (dR * KS).sum(1) - np.exp(g[-1] - g) * (U * (K @ dSC.T)).sum(1)
        dg[-1] += np.exp(g[-1]) * np.sum(dSC * S0c) + np.sum(np.exp(g[-1] - g) * (U * (K @ dSC.T)).sum(1))
        dlog = np.cumsum(dg[::-1])[::-1]
        sl = ch["sl"]
        dq[sl], dk[sl], dv[sl], db[sl], da[sl] = dQc, dKc, dVc, dbc, dlog / ch["a"]
    return dq, dk, dv, da, db, dS0


@pytest.mark.parametrize("C", [1, 5, 16, 64])
def test_chunk_backward_equals_recurrence_backward(orc, C):
    rng = np.random.default_rng(40 + C)
    L, d = 150, 16
    q = rng.standard_normal((L, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((L, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, d))
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L))))
    b = 1 / (1 + np.exp(-rng.standard_normal(L)))
    dO = rng.standard_normal((L, d))
    q, k, v, a, b, dO = (x.astype(np.float32) for x in (q, k, v, a, b, dO))
    S0 = rng.standard_normal((d, d))
    dSL = rng.standard_normal((d, d))
    ref = orc.gdn_bwd(q[None], k[None], v[None], a[None], b[None], dO[None], S0=S0[None],
                      dS_final=dSL[None])
    got = chunk_backward(*(x.astype(np.float64) for x in (q, k, v, a, b)), S0,
                         dO.astype(np.float64), dSL, C)
    for x, r in zip(got, ref):
        np.testing.assert_allclose(x, r[0], rtol=1e-8, atol=1e-9)


def _blocked_unit_lower_inverse(A):
    """(I + A)^-1 for strictly lower-triangular 64 x 64 A the way the chunk preparation forms
    it: the two diagonal 32 x 32 blocks by forward substitution, then T10 = -T11 A10 T00."""
    n = A.shape[0]
    h = n // 2
    T = np.zeros_like(A)
    for base in (0, h):
        for j in range(h):
            col = np.zeros(h)
            for t in range(h):
                if t < j:
                    continue
                col[t] = 1.0 if t == j else -A[base + t, base:base + t] @ col[:t]
            T[base:base + h, base + j] = col
    T[h:, :h] = -T[h:, h:] @ (A[h:, :h] @ T[:h, :h])
    return T


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_blocked_inverse_equals_inverse(seed):
    rng = np.random.default_rng(seed)
    n = 64
    k = rng.standard_normal((n, 128))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    b = rng.uniform(0.0, 1.0, n)
    g = np.cumsum(np.log(rng.uniform(0.5, 1.0, n)))
    low = np.tril(np.ones((n, n)), -1)
    A = low * b[:, None] * np.exp(np.where(low > 0, g[:, None] - g[None, :], 0)) * (k @ k.T)
    T = _blocked_unit_lower_inverse(A)
    assert np.allclose(T, np.linalg.inv(np.eye(n) + A), atol=1e-10)
    assert np.allclose(np.triu(T, 1), 0.0) and np.allclose(np.diag(T), 1.0)
