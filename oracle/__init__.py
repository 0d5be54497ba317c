"""CPU oracle of the Hybrid Linear Temporal Attention operator (fp64, plain definitions).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference leg may import this package; the product package never does.
The arithmetic lives in ``hlta_oracle.c`` (explicit masked softmax, token-by-token gated
delta recurrence); this file only marshals numpy arrays and composes the branches.

Branch composition (Kairos abstract, chatpaper.ai page, item (2); researchpapers.dev summary,
"How hybrid linear temporal attention suppresses drift"): the heads are split into three
groups, SWA | DSWA | GDN, each group runs its own branch, and the outputs are concatenated
back on the head axis in the same order.

Streaming (zhichai.net blog, section 2.3, the "streaming token" design: generate
incrementally without waiting for the whole sequence): the oracle does not keep caches; the
output of a step that appends frame f is, by definition, the last frame of the hybrid output
over frames 0..f.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hlta_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, no fast-math) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32 = ctypes.POINTER(ctypes.c_float)
        f64 = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.POINTER(ctypes.c_long)
        L_, I_, D_ = ctypes.c_long, ctypes.c_int, ctypes.c_double
        lib.oracle_swa.argtypes = [f32, f32, f32, f64, L_, I_, I_, I_, I_, D_, i64, L_]
        lib.oracle_dswa.argtypes = [f32, f32, f32, f64, L_, I_, I_, I_, I_, I_, D_, i64, L_]
        lib.oracle_gdn.argtypes = [f32, f32, f32, f32, f32, f64, f64, f64, f64, L_, L_, I_]
        lib.oracle_gdn_raw.argtypes = [f32, f32, f32, f32, f32, D_, f64, f64, f64, L_, L_, I_]
        for fn in (lib.oracle_swa, lib.oracle_dswa, lib.oracle_gdn, lib.oracle_gdn_raw):
            fn.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        u8 = ctypes.POINTER(ctypes.c_ubyte)
        lib.oracle_e4m3_decode.argtypes = [I_]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_fp8_quantize_rows.argtypes = [f32, f32, L_, L_, I_, L_, I_, u8, f32]
        lib.oracle_fp8_quantize_channels.argtypes = [f32, L_, L_, I_, u8, f32]
        for fn in (lib.oracle_fp8_quantize_rows, lib.oracle_fp8_quantize_channels):
            fn.restype = ctypes.c_int
        lib.oracle_window_bwd.argtypes = [f32, f32, f32, f32, f64, f64, f64, L_, I_, I_, I_, I_,
                                          I_, D_]
        lib.oracle_window_bwd.restype = ctypes.c_int
        lib.oracle_window_lse.argtypes = [f32, f32, f64, L_, I_, I_, I_, I_, I_, D_]
        lib.oracle_window_lse.restype = ctypes.c_int
        lib.oracle_gdn_bwd.argtypes = [f32, f32, f32, f32, f32, f64, f32, f64, f64, f64, f64, f64,
                                       f64, f64, L_, L_, I_]
        lib.oracle_gdn_bwd.restype = ctypes.c_int
        lib.oracle_rope.argtypes = [f32, f64, L_, L_, I_, I_, D_, I_, I_]
        lib.oracle_rope.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    """Host float32 contiguous copy of a numpy array or torch tensor (bf16 is exact in f32)."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(arr, ctype):
    if arr is None:
        return None
    return arr.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _window(q, k, v, T, N, w, r, dilated, scale, rows):
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    d = qf.shape[-1]
    L = T * N
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    assert qf.shape[-2] == L, "q must hold T*N rows"
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    lib = _load()
    if rows is None:
        o = np.empty(qf.shape, dtype=np.float64)
        rp, nr = None, 0
    else:
        rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        o = np.empty((rr.size, d), dtype=np.float64)
        rp, nr = _ptr(rr, ctypes.c_long), rr.size
    if dilated:
        rc = lib.oracle_dswa(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                             _ptr(vf, ctypes.c_float), _ptr(o, ctypes.c_double),
                             BH, T, N, d, w, r, float(scale), rp, nr)
    else:
        rc = lib.oracle_swa(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                            _ptr(vf, ctypes.c_float), _ptr(o, ctypes.c_double),
                            BH, T, N, d, w, float(scale), rp, nr)
    if rc != 0:
        raise RuntimeError(f"oracle window attention failed ({rc})")
    return o


def swa(q, k, v, T: int, N: int, w: int, scale=None, rows=None) -> np.ndarray:
    """Block-causal sliding-window attention over frames max(0,f-w+1)..f.

    q, k, v: [..., L, d]. ``rows``: optional flat indices (head-major, bh*L + l) to compute
    only those query rows; the result is then [len(rows), d]."""
    return _window(q, k, v, T, N, w, 1, False, scale, rows)


def dswa(q, k, v, T: int, N: int, w: int, r: int, scale=None, rows=None) -> np.ndarray:
    """Dilated sliding-window attention over frames f, f-r, ..., f-r(w-1) (>= 0)."""
    return _window(q, k, v, T, N, w, r, True, scale, rows)


def gdn(q, k, v, a, b, S0=None, history: bool = False):
    """Gated delta rule, token by token. q,k,v: [..., L, d]; a,b: [..., L].

    Returns (o, S_final) and, with ``history``, also every S_t as [..., L, d, d]."""
    qf, kf, vf, af, bf = _f32(q), _f32(k), _f32(v), _f32(a), _f32(b)
    d = qf.shape[-1]
    L = qf.shape[-2]
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    S0d = None
    if S0 is not None:
        if hasattr(S0, "detach"):
            S0 = S0.detach().cpu().double().numpy()
        S0d = np.ascontiguousarray(np.asarray(S0, dtype=np.float64)).reshape(BH, d, d)
    o = np.empty(qf.shape, dtype=np.float64)
    S_out = np.empty(lead + (d, d), dtype=np.float64)
    hist = np.empty(lead + (L, d, d), dtype=np.float64) if history else None
    rc = _load().oracle_gdn(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                            _ptr(vf, ctypes.c_float), _ptr(af, ctypes.c_float),
                            _ptr(bf, ctypes.c_float), _ptr(S0d, ctypes.c_double),
                            _ptr(o, ctypes.c_double), _ptr(S_out, ctypes.c_double),
                            _ptr(hist, ctypes.c_double), BH, L, d)
    if rc != 0:
        raise RuntimeError(f"oracle gdn failed ({rc})")
    return (o, S_out, hist) if history else (o, S_out)


def gdn_bwd(q, k, v, a, b, dO, S0=None, dS_final=None):
    """Gradients of the gated delta rule for the upstream gradients dO (of every output) and
    dS_final (of the final state, or None for zero). Returns (dq, dk, dv, da, db, dS0), float64:
    dq, dk, dv [..., L, d]; da, db [..., L]; dS0 [..., d, d]."""
    qf, kf, vf, af, bf, gf = _f32(q), _f32(k), _f32(v), _f32(a), _f32(b), _f32(dO)
    d = qf.shape[-1]
    L = qf.shape[-2]
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1

    def dmat(x):
        if x is None:
            return None
        if hasattr(x, "detach"):
            x = x.detach().cpu().double().numpy()
        return np.ascontiguousarray(np.asarray(x, dtype=np.float64)).reshape(BH, d, d)

    S0d, dSd = dmat(S0), dmat(dS_final)
    dq, dk, dv = (np.empty(qf.shape, dtype=np.float64) for _ in range(3))
    da, db = (np.empty(qf.shape[:-1], dtype=np.float64) for _ in range(2))
    dS0 = np.empty(lead + (d, d), dtype=np.float64)
    rc = _load().oracle_gdn_bwd(*(_ptr(x, ctypes.c_float) for x in (qf, kf, vf, af, bf)),
                                _ptr(S0d, ctypes.c_double), _ptr(gf, ctypes.c_float),
                                _ptr(dSd, ctypes.c_double),
                                *(_ptr(x, ctypes.c_double) for x in (dq, dk, dv, da, db, dS0)),
                                BH, L, d)
    if rc != 0:
        raise RuntimeError(f"oracle gdn_bwd failed ({rc})")
    return dq, dk, dv, da, db, dS0


def gdn_raw(q, k, v, x, y, c: float, S0=None):
    """GDN heads from raw inputs: q, k scaled to unit L2 norm per token, gates
    a = exp(-c softplus(x)), b = sigmoid(y), then the recurrence (all fp64).
    q,k,v: [..., L, d]; x,y: [..., L]. Returns (o, S_final)."""
    qf, kf, vf, xf, yf = _f32(q), _f32(k), _f32(v), _f32(x), _f32(y)
    d = qf.shape[-1]
    L = qf.shape[-2]
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    S0d = None
    if S0 is not None:
        if hasattr(S0, "detach"):
            S0 = S0.detach().cpu().double().numpy()
        S0d = np.ascontiguousarray(np.asarray(S0, dtype=np.float64)).reshape(BH, d, d)
    o = np.empty(qf.shape, dtype=np.float64)
    S_out = np.empty(lead + (d, d), dtype=np.float64)
    rc = _load().oracle_gdn_raw(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                                _ptr(vf, ctypes.c_float), _ptr(xf, ctypes.c_float),
                                _ptr(yf, ctypes.c_float), float(c), _ptr(S0d, ctypes.c_double),
                                _ptr(o, ctypes.c_double), _ptr(S_out, ctypes.c_double), BH, L, d)
    if rc != 0:
        raise RuntimeError(f"oracle gdn_raw failed ({rc})")
    return o, S_out


def hybrid(q, k, v, a, b, Hs: int, Hd: int, Hg: int, T: int, N: int,
           w_swa: int, w_dswa: int, r: int, S0=None, scale=None, raw=None):
    """All three branches on their head groups of [B, H, L, d]; concat on the head axis.

    With ``raw`` = c the GDN heads take raw inputs: ``a``, ``b`` are then x, y and the GDN
    branch is ``gdn_raw(..., c=raw)``. Returns (o [B,H,L,d] float64, S_final [B,Hg,d,d])."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    B, H, L, d = qf.shape
    assert H == Hs + Hd + Hg
    o = np.empty(qf.shape, dtype=np.float64)
    if Hs:
        o[:, :Hs] = swa(qf[:, :Hs], kf[:, :Hs], vf[:, :Hs], T, N, w_swa, scale)
    if Hd:
        s = slice(Hs, Hs + Hd)
        o[:, s] = dswa(qf[:, s], kf[:, s], vf[:, s], T, N, w_dswa, r, scale)
    S_fin = np.zeros((B, Hg, d, d))
    if Hg:
        s = slice(Hs + Hd, H)
        if raw is None:
            og, S_fin = gdn(qf[:, s], kf[:, s], vf[:, s], a, b, S0)
        else:
            og, S_fin = gdn_raw(qf[:, s], kf[:, s], vf[:, s], a, b, raw, S0)
        o[:, s] = og
    return o, S_fin


def window_bwd(q, k, v, dO, T: int, N: int, w: int, r: int = 1, scale=None):
    """Gradients (dq, dk, dv) of the windowed attention (SWA for r == 1, DSWA otherwise) for
    the upstream gradient dO, float64 [..., L, d] each."""
    qf, kf, vf, gf = _f32(q), _f32(k), _f32(v), _f32(dO)
    d = qf.shape[-1]
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    assert qf.shape[-2] == T * N, "q must hold T*N rows"
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = [np.empty(qf.shape, dtype=np.float64) for _ in range(3)]
    rc = _load().oracle_window_bwd(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                                   _ptr(vf, ctypes.c_float), _ptr(gf, ctypes.c_float),
                                   *(_ptr(o, ctypes.c_double) for o in out), BH, T, N, d, w, r,
                                   float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle window_bwd failed ({rc})")
    return tuple(out)


def window_lse(q, k, T: int, N: int, w: int, r: int = 1, scale=None) -> np.ndarray:
    """Natural log-sum-exp of each query row's scaled scores over its window keys, [..., L]."""
    qf, kf = _f32(q), _f32(k)
    d = qf.shape[-1]
    lead = qf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty(qf.shape[:-1], dtype=np.float64)
    rc = _load().oracle_window_lse(_ptr(qf, ctypes.c_float), _ptr(kf, ctypes.c_float),
                                   _ptr(out, ctypes.c_double), BH, T, N, d, w, r, float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle window_lse failed ({rc})")
    return out


def rope(x, N: int, base: float = 10000.0, pos_mode: int = 0, sign: int = 1) -> np.ndarray:
    """Rotary embedding of x [..., L, d] (see oracle_rope: position l mod N or l), fp64."""
    xf = _f32(x)
    shp = xf.shape
    L, d = shp[-2], shp[-1]
    BH = int(np.prod(shp[:-2])) if len(shp) > 2 else 1
    y = np.empty(shp, dtype=np.float64)
    rc = _load().oracle_rope(_ptr(xf, ctypes.c_float), _ptr(y, ctypes.c_double), BH, L, N, d,
                             float(base), int(pos_mode), int(sign))
    if rc:
        raise ValueError("oracle_rope: bad arguments")
    return y


def e4m3_decode(code: int) -> float:
    """Value of one E4M3 code (OCP 8-bit floating point, E4M3 encoding)."""
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode(y: float) -> int:
    """Nearest E4M3 code to the float32 value y (ties to even, saturating at +-448)."""
    return int(_load().oracle_e4m3_encode(float(np.float32(y))))


def e4m3_values() -> np.ndarray:
    """float64 value of each of the 256 codes (NaN for 0x7F and 0xFF)."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def fp8_quantize_rows(x, frame_rows: int, block_rows: int, shift=None):
    """Row-block E4M3 quantisation of x [..., L, d]: blocks of block_rows rows inside frames
    of frame_rows rows. Returns (codes uint8 [..., L, d], scales float32 [..., nf, nb])."""
    xf = _f32(x)
    L, d = xf.shape[-2], xf.shape[-1]
    lead = xf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    nf = -(-L // frame_rows)
    nb = -(-frame_rows // block_rows)
    sh = None if shift is None else _f32(shift).reshape(BH, d)
    x8 = np.empty(xf.shape, dtype=np.uint8)
    sc = np.empty(lead + (nf, nb), dtype=np.float32)
    rc = _load().oracle_fp8_quantize_rows(_ptr(xf, ctypes.c_float), _ptr(sh, ctypes.c_float), BH,
                                          L, d, frame_rows, block_rows,
                                          _ptr(x8, ctypes.c_ubyte), _ptr(sc, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle fp8_quantize_rows failed ({rc})")
    return x8, sc


def fp8_quantize_channels(x):
    """Per-channel E4M3 quantisation of x [..., L, d] (one scale per head and channel).
    Returns (codes uint8 [..., L, d], scales float32 [..., d])."""
    xf = _f32(x)
    L, d = xf.shape[-2], xf.shape[-1]
    lead = xf.shape[:-2]
    BH = int(np.prod(lead)) if lead else 1
    x8 = np.empty(xf.shape, dtype=np.uint8)
    sc = np.empty(lead + (d,), dtype=np.float32)
    rc = _load().oracle_fp8_quantize_channels(_ptr(xf, ctypes.c_float), BH, L, d,
                                              _ptr(x8, ctypes.c_ubyte), _ptr(sc, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"oracle fp8_quantize_channels failed ({rc})")
    return x8, sc


def fp8_dequantize_rows(x8, scales, frame_rows: int, block_rows: int) -> np.ndarray:
    """decode(code) * scale of the code's row block, float64 [..., L, d]."""
    x8 = np.asarray(x8)
    L = x8.shape[-2]
    l = np.arange(L)
    f, j = l // frame_rows, (l % frame_rows) // block_rows
    s = np.asarray(scales, dtype=np.float64)[..., f, j]          # [..., L]
    return e4m3_values()[x8] * s[..., None]


def fp8_dequantize_channels(x8, scales) -> np.ndarray:
    """decode(code) * scale of the code's channel, float64 [..., L, d]."""
    return e4m3_values()[np.asarray(x8)] * np.asarray(scales, dtype=np.float64)[..., None, :]


def window_fp8(q8, qs, k8, ks, v8, vs, T: int, N: int, w: int, r: int, scale=None, rows=None):
    """Windowed attention (SWA when r == 1, DSWA otherwise) of E4M3 inputs: the plain
    attention of the dequantised tensors. Q blocks: 128 rows of the head; K blocks: 64-row
    runs inside each frame; V: one scale per channel. (The dequantised values are passed to
    the attention as float32, a relative rounding of 2^-24.)"""
    L = T * N
    q = fp8_dequantize_rows(q8, qs, L, 128)
    k = fp8_dequantize_rows(k8, ks, N, 64)
    v = fp8_dequantize_channels(v8, vs)
    return _window(q, k, v, T, N, w, r, r > 1, scale, rows)


def hybrid_rows(q, k, v, a, b, Hs, Hd, Hg, T, N, w_swa, w_dswa, r, rows, scale=None):
    """Softmax branches on sampled query rows only, GDN in full.

    ``rows``: query positions l (shared by every head). Returns
    (o_sw [B,Hs,len(rows),d], o_dsw [B,Hd,len(rows),d], o_gdn [B,Hg,L,d], S_final)."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    B, H, L, d = qf.shape
    rows = np.asarray(rows, dtype=np.int64)

    def flat(nh):
        return (np.arange(B * nh)[:, None] * L + rows[None, :]).reshape(-1)

    o_s = o_d = None
    if Hs:
        o_s = swa(qf[:, :Hs], kf[:, :Hs], vf[:, :Hs], T, N, w_swa, scale,
                  rows=flat(Hs)).reshape(B, Hs, rows.size, d)
    if Hd:
        s = slice(Hs, Hs + Hd)
        o_d = dswa(qf[:, s], kf[:, s], vf[:, s], T, N, w_dswa, r, scale,
                   rows=flat(Hd)).reshape(B, Hd, rows.size, d)
    o_g, S_fin = (None, None)
    if Hg:
        s = slice(Hs + Hd, H)
        o_g, S_fin = gdn(qf[:, s], kf[:, s], vf[:, s], a, b)
    return o_s, o_d, o_g, S_fin
