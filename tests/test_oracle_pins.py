"""Pins of the CPU oracle to facts other than its own formulas.

Each test fixes the oracle against something independent: a brute-force dense computation
on tiny inputs, a closed form worked by hand, or an invariant the pages state or imply.
Chosen so that a plausible slip in the oracle (an off-by-one window, a clamped instead of a
dropped tap, a transposed state, a wrong sign in the erase term, a misplaced decay) fails
at least one of them.
"""
import math

import numpy as np
import pytest


def _rng(seed):
    return np.random.default_rng(seed)


def _dense_masked_attention(q, k, v, allowed, scale):
    """Brute force: full score matrix, -inf where not allowed, softmax, times V."""
    s = (q.astype(np.float64) @ k.astype(np.float64).T) * scale
    s = np.where(allowed, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v.astype(np.float64)


# --------------------------------------------------------------------------------------
# Sliding-window attention
# --------------------------------------------------------------------------------------

def test_swa_window_covering_clip_is_block_causal_full_attention(orc):
    """w >= T: every earlier frame is in the window, so SWA is block-causal full attention."""
    T, N, d = 5, 6, 8
    r = _rng(1)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) for _ in range(3))
    fr = np.arange(T * N) // N
    allowed = fr[None, :] <= fr[:, None]
    ref = _dense_masked_attention(q, k, v, allowed, 1 / math.sqrt(d))
    for w in (T, T + 3):
        o = orc.swa(q[None], k[None], v[None], T, N, w)[0]
        np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_swa_window_one_is_per_frame_attention(orc):
    """w = 1: each frame attends only to itself, bidirectionally within the frame."""
    T, N, d = 4, 7, 5
    r = _rng(2)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) for _ in range(3))
    o = orc.swa(q[None], k[None], v[None], T, N, 1)[0]
    for f in range(T):
        s = slice(f * N, (f + 1) * N)
        ref = _dense_masked_attention(q[s], k[s], v[s], np.ones((N, N), bool), 1 / math.sqrt(d))
        np.testing.assert_allclose(o[s], ref, rtol=1e-12, atol=1e-12)


def test_swa_hand_closed_form():
    """d = 1, N = 1, q = 1, k = (0, ln 3, ln 2), v = (4, 8, 16), w = 2, scale 1.

    Weights are e^{q k_j}: frame 0 sees {1}, frame 1 sees {1, 3}, frame 2 sees {3, 2}, so
    o = (4, (4 + 3*8)/4, (3*8 + 2*16)/5) = (4, 7, 11.2). The float32 rounding of ln 3 and
    ln 2 is carried into the closed form."""
    import oracle
    k = np.array([0.0, math.log(3), math.log(2)], dtype=np.float32)
    q = np.ones(3, dtype=np.float32)
    v = np.array([4.0, 8.0, 16.0], dtype=np.float32)
    o = oracle.swa(q[None, :, None], k[None, :, None], v[None, :, None], 3, 1, 2, scale=1.0)
    w1, w2 = math.exp(float(k[1])), math.exp(float(k[2]))
    expect = [4.0, (4.0 + w1 * 8.0) / (1.0 + w1), (w1 * 8.0 + w2 * 16.0) / (w1 + w2)]
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-15)
    np.testing.assert_allclose(o[0, :, 0], [4.0, 7.0, 11.2], rtol=1e-6)


def test_swa_rows_are_convex_combinations(orc):
    """Every output coordinate lies within [min, max] of v over the query's window."""
    T, N, d, w = 6, 5, 4, 3
    r = _rng(3)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) * 3 for _ in range(3))
    o = orc.swa(q[None], k[None], v[None], T, N, w)[0]
    for l in range(T * N):
        f = l // N
        win = v[max(0, f - w + 1) * N:(f + 1) * N].astype(np.float64)
        assert np.all(o[l] <= win.max(0) + 1e-12) and np.all(o[l] >= win.min(0) - 1e-12)


def test_swa_invariant_to_permuting_a_key_frame(orc):
    """Softmax over a set: permuting (k, v) pairs within one frame changes no output row."""
    T, N, d, w = 5, 6, 4, 2
    r = _rng(4)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) for _ in range(3))
    perm = np.arange(T * N)
    f = 2
    perm[f * N:(f + 1) * N] = f * N + r.permutation(N)
    o1 = orc.swa(q[None], k[None], v[None], T, N, w)[0]
    o2 = orc.swa(q[None], k[perm][None], v[perm][None], T, N, w)[0]
    # queries of frame f are not permuted (only its keys/values), so all rows must agree
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)


def test_swa_row_subset_matches_full(orc):
    T, N, d, w = 4, 5, 3, 2
    r = _rng(5)
    q, k, v = (r.standard_normal((2, T * N, d)).astype(np.float32) for _ in range(3))
    full = orc.swa(q, k, v, T, N, w).reshape(-1, d)
    rows = np.array([0, 7, 19, 20, 39])
    part = orc.swa(q, k, v, T, N, w, rows=rows)
    np.testing.assert_array_equal(part, full[rows])


# --------------------------------------------------------------------------------------
# Dilated sliding-window attention
# --------------------------------------------------------------------------------------

def test_dswa_dilation_one_is_swa(orc):
    T, N, d = 7, 4, 6
    r = _rng(6)
    q, k, v = (r.standard_normal((2, T * N, d)).astype(np.float32) for _ in range(3))
    for w in (1, 2, 3, 9):
        np.testing.assert_array_equal(orc.dswa(q, k, v, T, N, w, 1), orc.swa(q, k, v, T, N, w))


def test_dswa_window_one_is_own_frame(orc):
    T, N, d = 5, 3, 4
    r = _rng(7)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) for _ in range(3))
    for rr in (2, 3, 10):
        np.testing.assert_array_equal(orc.dswa(q[None], k[None], v[None], T, N, 1, rr),
                                      orc.swa(q[None], k[None], v[None], T, N, 1))


def test_dswa_hand_closed_form_drops_missing_taps():
    """T = 5, N = 1, d = 1, w = 2, r = 2, scale 1, q = 1, k = ln(c_j): frame f sees frames
    {f-2, f} with weights c; frame 0 and 1 see only themselves (tap f-2 < 0 is dropped,
    not clamped to frame 0), frame 4 sees {2, 4}."""
    import oracle
    c = np.array([1.0, 2.0, 3.0, 4.0, 5.0])
    k = np.log(c).astype(np.float32)
    cw = np.exp(k.astype(np.float64))
    v = np.array([1.0, 10.0, 100.0, 1000.0, 10000.0], dtype=np.float32)
    q = np.ones(5, dtype=np.float32)
    o = oracle.dswa(q[None, :, None], k[None, :, None], v[None, :, None], 5, 1, 2, 2, scale=1.0)
    expect = [v[0], v[1],
              (cw[0] * v[0] + cw[2] * v[2]) / (cw[0] + cw[2]),
              (cw[1] * v[1] + cw[3] * v[3]) / (cw[1] + cw[3]),
              (cw[2] * v[2] + cw[4] * v[4]) / (cw[2] + cw[4])]
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-14)
    # the same numbers written out: frame 4 = (3*100 + 5*10000)/8
    np.testing.assert_allclose(o[0, 4, 0], (300 + 50000) / 8, rtol=1e-6)


def test_dswa_brute_force_tap_mask(orc):
    """Brute force on a tiny clip, mask from the frame distance: 0 <= f_q - f_k <= r(w-1)
    and divisible by r."""
    T, N, d, w, rr = 9, 3, 4, 3, 3
    r = _rng(8)
    q, k, v = (r.standard_normal((T * N, d)).astype(np.float32) for _ in range(3))
    fr = np.arange(T * N) // N
    dist = fr[:, None] - fr[None, :]
    allowed = (dist >= 0) & (dist <= rr * (w - 1)) & (dist % rr == 0)
    ref = _dense_masked_attention(q, k, v, allowed, 1 / math.sqrt(d))
    np.testing.assert_allclose(orc.dswa(q[None], k[None], v[None], T, N, w, rr)[0], ref,
                               rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------------------
# Gated delta rule
# --------------------------------------------------------------------------------------

def _unit_rows(x):
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


def test_gdn_zero_write_from_zero_state_stays_zero(orc):
    L, d = 50, 8
    r = _rng(10)
    q, k = _unit_rows(r.standard_normal((L, d))), _unit_rows(r.standard_normal((L, d)))
    v = r.standard_normal((L, d)).astype(np.float32)
    a = r.uniform(0.1, 1, L).astype(np.float32)
    o, S = orc.gdn(q[None], k[None], v[None], a[None], np.zeros((1, L), np.float32))
    assert np.all(o == 0.0) and np.all(S == 0.0)


def test_gdn_zero_write_is_pure_decay(orc):
    """b = 0: S_t = (prod_{s<=t} a_s) S_0, so o_t = (prod a) S_0 q_t."""
    L, d = 40, 6
    r = _rng(11)
    q, k = _unit_rows(r.standard_normal((L, d))), _unit_rows(r.standard_normal((L, d)))
    v = r.standard_normal((L, d)).astype(np.float32)
    a = r.uniform(0.5, 1, L).astype(np.float32)
    S0 = r.standard_normal((d, d))
    o, S = orc.gdn(q[None], k[None], v[None], a[None], np.zeros((1, L), np.float32), S0[None])
    decay = np.cumprod(a.astype(np.float64))
    expect = decay[:, None] * (q.astype(np.float64) @ S0.T)
    np.testing.assert_allclose(o[0], expect, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[0], decay[-1] * S0, rtol=1e-12)


def test_gdn_orthonormal_keys_retrieve_exactly(orc):
    """a = b = 1, orthonormal keys, zero start: the delta rule stores every pair without
    interference, S k_i = v_i; a query equal to k_i reads back v_i."""
    d, n = 16, 12
    r = _rng(12)
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    keys = Qm[:, :n].T.astype(np.float32)                      # n orthonormal rows (to f32)
    v = r.standard_normal((n, d)).astype(np.float32)
    q = keys.copy()
    ones = np.ones((1, n), np.float32)
    o, S = orc.gdn(q[None], keys[None], v[None], ones, ones)
    kd = keys.astype(np.float64)
    # float32 keys are orthonormal only to ~1e-7; the retrieval holds to that level
    np.testing.assert_allclose(S[0] @ kd.T, v.T.astype(np.float64), atol=2e-6)
    np.testing.assert_allclose(o[0], v.astype(np.float64), atol=2e-6)
    # orientation: o = S q, not S^T q
    assert np.abs(S[0].T @ kd.T - v.T).max() > 1e-2


def test_gdn_repeated_key_overwrites(orc):
    """a = b = 1 with one key repeated: each write erases the previous value, S k = v_last
    and S = v_last k^T (without the erase term S k would be the sum of the values)."""
    L, d = 7, 5
    r = _rng(13)
    key = _unit_rows(r.standard_normal((1, d)))[0]
    k = np.tile(key, (L, 1))
    v = r.standard_normal((L, d)).astype(np.float32)
    q = np.tile(key, (L, 1))
    ones = np.ones((1, L), np.float32)
    o, S = orc.gdn(q[None], k[None], v[None], ones, ones)
    kd = key.astype(np.float64)
    nk = float(kd @ kd)
    # exact unit norm up to the float32 rounding of the key
    np.testing.assert_allclose(S[0], np.outer(v[-1], kd), atol=5e-7)
    np.testing.assert_allclose(o[0], v.astype(np.float64) * nk, atol=5e-7)


def test_gdn_erase_then_write_single_step():
    """One step from S_0 = v0 k^T with the same unit key: S_1 k = (1-b) a v0 + b v1 ...
    worked out: S_1 = a S_0 (I - b k k^T) + b v1 k^T = a (1-b) v0 k^T + b v1 k^T."""
    import oracle
    d = 4
    key = np.array([0.0, 0.6, 0.8, 0.0], np.float32)           # exactly unit in float32? 0.36+0.64
    v0 = np.array([1.0, -2.0, 3.0, 0.5])
    v1 = np.array([4.0, 1.0, -1.0, 2.0], np.float32)
    S0 = np.outer(v0, key.astype(np.float64))
    for a_, b_ in ((1.0, 1.0), (1.0, 0.5), (0.5, 0.25)):
        o, S = oracle.gdn(key[None, None], key[None, None], v1[None, None],
                          np.float32([[a_]]), np.float32([[b_]]), S0[None])
        kk = float(key.astype(np.float64) @ key.astype(np.float64))
        expect = a_ * (np.outer(v0, key) - b_ * kk * np.outer(v0, key)) + b_ * np.outer(v1, key)
        np.testing.assert_allclose(S[0], expect, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[0] @ key, (a_ * (1 - b_ * kk) * v0 + b_ * v1) * kk,
                                   rtol=1e-6)


def test_gdn_orthogonal_write_does_not_disturb(orc):
    """a = 1: writing along k2 orthogonal to k1 leaves S k1 unchanged (the erase acts along
    the written key only)."""
    d = 6
    k1 = np.zeros(d, np.float32); k1[1] = 1
    k2 = np.zeros(d, np.float32); k2[4] = 1
    r = _rng(14)
    v = r.standard_normal((2, d)).astype(np.float32)
    k = np.stack([k1, k2])
    o, S = orc.gdn(k[None], k[None], v[None], np.ones((1, 2), np.float32),
                   np.float32([[1.0, 0.7]]))
    np.testing.assert_allclose(S[0] @ k1, v[0], atol=1e-12)
    np.testing.assert_allclose(S[0] @ k2, 0.7 * v[1], atol=1e-7)


def test_gdn_linear_in_values_from_zero_state(orc):
    L, d = 30, 7
    r = _rng(15)
    q, k = _unit_rows(r.standard_normal((L, d))), _unit_rows(r.standard_normal((L, d)))
    # dyadic values, so 2*v1 - 3*v2 is exact in float32
    v1 = (np.round(r.standard_normal((L, d)) * 64) / 64).astype(np.float32)
    v2 = (np.round(r.standard_normal((L, d)) * 64) / 64).astype(np.float32)
    a = r.uniform(0.3, 1, L).astype(np.float32)[None]
    b = r.uniform(0, 1, L).astype(np.float32)[None]
    o1, _ = orc.gdn(q[None], k[None], v1[None], a, b)
    o2, _ = orc.gdn(q[None], k[None], v2[None], a, b)
    o3, _ = orc.gdn(q[None], k[None], (2 * v1 - 3 * v2)[None], a, b)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=1e-10, atol=1e-12)


def test_gdn_contraction_bound_every_step(orc):
    """Contraction of the gated delta memory (researchpapers.dev Theorem 2 / zhichai.net
    section 4, gamma < 1): with unit keys and b in [0,1], two runs from different initial
    states differ at step t by at most prod_{s<=t} a_s times the initial gap, in Frobenius
    norm; the outputs differ by at most that times the spectral gap."""
    L, d = 80, 8
    r = _rng(16)
    q, k = _unit_rows(r.standard_normal((L, d))), _unit_rows(r.standard_normal((L, d)))
    v = r.standard_normal((L, d)).astype(np.float32)
    a = np.exp(-np.log1p(np.exp(r.standard_normal(L)))).astype(np.float32)
    b = (1 / (1 + np.exp(-r.standard_normal(L)))).astype(np.float32)
    S0a, S0b = r.standard_normal((d, d)), r.standard_normal((d, d))
    _, _, Ha = orc.gdn(q[None], k[None], v[None], a[None], b[None], S0a[None], history=True)
    _, _, Hb = orc.gdn(q[None], k[None], v[None], a[None], b[None], S0b[None], history=True)
    gap = np.linalg.norm(S0a - S0b)
    decay = np.cumprod(a.astype(np.float64))
    diffs = np.linalg.norm(Ha[0] - Hb[0], axis=(1, 2))
    # keys are unit only to float32 rounding: allow that relative slack per step
    assert np.all(diffs <= decay * gap * (1 + 1e-5) + 1e-12)
    # and the bound is not vacuous: with b = 0 it holds with equality
    _, _, Ha0 = orc.gdn(q[None], k[None], v[None], a[None], np.zeros((1, L), np.float32),
                        S0a[None], history=True)
    _, _, Hb0 = orc.gdn(q[None], k[None], v[None], a[None], np.zeros((1, L), np.float32),
                        S0b[None], history=True)
    np.testing.assert_allclose(np.linalg.norm(Ha0[0] - Hb0[0], axis=(1, 2)), decay * gap,
                               rtol=1e-10)


def test_gdn_wrong_sign_erase_would_break_contraction(orc):
    """Guard that the contraction pin has teeth: the same check on a planted variant of the
    update with a flipped erase sign (written here, on the CPU) fails."""
    L, d = 40, 6
    r = _rng(17)
    k = _unit_rows(r.standard_normal((L, d))).astype(np.float64)
    a = np.full(L, 0.99)
    b = np.full(L, 0.9)
    D = r.standard_normal((d, d))
    D0 = np.linalg.norm(D)
    bad = D.copy()
    for t in range(L):
        bad = a[t] * (bad + b[t] * np.outer(bad @ k[t], k[t]))
    assert np.linalg.norm(bad) > np.prod(a) * D0 * 1.01


def test_hybrid_head_groups_in_order(orc):
    """Heads are split SWA | DSWA | GDN and concatenated back in that order."""
    import hlta_inputs as hi
    wl = hi.WORKLOADS["tiny_fp32"]
    x = hi.make_inputs(wl, seed=3)
    q, k, v = (x[n].numpy() for n in ("q", "k", "v"))
    o, S = orc.hybrid(q, k, v, x["a"], x["b"], 1, 1, 1, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    np.testing.assert_array_equal(o[:, 0], orc.swa(q[:, 0], k[:, 0], v[:, 0], wl.T, wl.N, wl.w_swa))
    np.testing.assert_array_equal(o[:, 1], orc.dswa(q[:, 1], k[:, 1], v[:, 1], wl.T, wl.N,
                                                    wl.w_dswa, wl.r))
    og, Sg = orc.gdn(q[:, 2:], k[:, 2:], v[:, 2:], x["a"], x["b"])
    np.testing.assert_array_equal(o[:, 2:], og)
    np.testing.assert_array_equal(S, Sg)


# --------------------------------------------------------------------------------------
# GDN prologue (raw inputs): unit-norm q, k; a = exp(-c softplus(x)), b = sigmoid(y)
# --------------------------------------------------------------------------------------

def test_gdn_raw_is_scale_invariant_in_q_and_k(orc):
    """Only the direction of q and k matters: per-token positive scales (powers of two, exact
    in float32) leave every output and the final state unchanged."""
    r = _rng(21)
    L, d = 40, 16
    q, k, v = (r.standard_normal((2, L, d)).astype(np.float32) for _ in range(3))
    x, y = (r.standard_normal((2, L)).astype(np.float32) for _ in range(2))
    sq = np.exp2(r.integers(-6, 7, size=(2, L, 1))).astype(np.float32)
    sk = np.exp2(r.integers(-6, 7, size=(2, L, 1))).astype(np.float32)
    o1, S1 = orc.gdn_raw(q, k, v, x, y, 0.7)
    o2, S2 = orc.gdn_raw(q * sq, k * sk, v, x, y, 0.7)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-12)
    # and q, k are not used as given: doubling only k changes nothing, doubling v does
    o3, _ = orc.gdn_raw(q, k, 2 * v, x, y, 0.7)
    np.testing.assert_allclose(o3, 2 * o1, rtol=1e-12, atol=1e-12)


def test_gdn_raw_equals_gdn_through_inverse_gates(orc):
    """Gates given through the inverses of the activations (x = log(e^s - 1) so that
    softplus(x) = s = -log(a)/c; y = log(b / (1 - b))) and unit q, k: the raw path must
    reproduce the pinned recurrence."""
    r = _rng(22)
    L, d, c = 30, 12, 0.6
    q, k, v = (r.standard_normal((1, L, d)) for _ in range(3))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a = r.uniform(0.5, 0.99, size=(1, L))
    b = r.uniform(0.05, 0.95, size=(1, L))
    s = -np.log(a) / c
    x = np.log(np.expm1(s))
    y = np.log(b / (1 - b))
    o_raw, S_raw = orc.gdn_raw(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32),
                               x.astype(np.float32), y.astype(np.float32), c)
    # the reference gets the same float32-rounded values, gates recomputed from the rounded x, y
    xr, yr = x.astype(np.float32).astype(np.float64), y.astype(np.float32).astype(np.float64)
    a_r = np.exp(-c * np.log1p(np.exp(xr)))
    b_r = 1 / (1 + np.exp(-yr))
    o_ref, S_ref = orc.gdn(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32),
                           a_r.astype(np.float32), b_r.astype(np.float32))
    np.testing.assert_allclose(o_raw, o_ref, rtol=0, atol=2e-6)
    np.testing.assert_allclose(S_raw, S_ref, rtol=0, atol=2e-6)


def test_gdn_raw_neutral_gate_inputs_closed_form(orc):
    """x = 0 gives softplus(0) = ln 2, so a = 2^-c; y = -200 gives b = 0 to double precision:
    no writes, pure decay, o_t = 2^(-c (t+1)) S0 q_t / |q_t|."""
    r = _rng(23)
    L, d, c = 9, 6, 1.5
    q, k, v = (r.standard_normal((1, L, d)).astype(np.float32) for _ in range(3))
    S0 = r.standard_normal((1, d, d))
    x = np.zeros((1, L), np.float32)
    y = np.full((1, L), -200.0, np.float32)
    o, S = orc.gdn_raw(q, k, v, x, y, c, S0=S0)
    qn = q[0].astype(np.float64) / np.linalg.norm(q[0].astype(np.float64), axis=-1, keepdims=True)
    for t in range(L):
        np.testing.assert_allclose(o[0, t], 2.0 ** (-c * (t + 1)) * S0[0] @ qn[t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0], 2.0 ** (-c * L) * S0[0], rtol=1e-12, atol=1e-13)


def test_gdn_raw_zero_token_stays_zero(orc):
    """A token whose q and k are zero reads nothing and erases/writes along no direction:
    its output is zero and the state only decays."""
    r = _rng(24)
    L, d = 5, 8
    q, k, v = (r.standard_normal((1, L, d)).astype(np.float32) for _ in range(3))
    q[0, 2] = 0
    k[0, 2] = 0
    x, y = (r.standard_normal((1, L)).astype(np.float32) for _ in range(2))
    o, _ = orc.gdn_raw(q, k, v, x, y, 1.0)
    assert np.all(o[0, 2] == 0)
    assert np.all(np.isfinite(o))


def test_hybrid_raw_routes_gdn_heads_through_the_prologue(orc):
    import hlta_inputs as hi
    wl = hi.WORKLOADS["tiny_fp32"]
    x = hi.make_raw_inputs(wl, seed=4)
    q, k, v = (x[n].numpy() for n in ("q", "k", "v"))
    o, S = orc.hybrid(q, k, v, x["x"], x["y"], 1, 1, 1, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r,
                      raw=wl.decay)
    og, Sg = orc.gdn_raw(q[:, 2:], k[:, 2:], v[:, 2:], x["x"], x["y"], wl.decay)
    np.testing.assert_array_equal(o[:, 2:], og)
    np.testing.assert_array_equal(S, Sg)
    np.testing.assert_array_equal(o[:, 0], orc.swa(q[:, 0], k[:, 0], v[:, 0], wl.T, wl.N, wl.w_swa))
