"""Python binding of the B200 Hybrid Linear Temporal Attention library (libhlta.so).

Argument marshalling only: every function passes device pointers, sizes and the current
CUDA stream to the C ABI declared in include/hlta.h, and raises ``HltaError`` on a non-OK
status. Tensors are torch tensors on a CUDA device (torch provides memory and streams);
no computation happens here, and there is no fallback: if the compiled library is missing,
importing this package fails.

Function names match the C entry points (``hlta_swa_fwd`` ...). The convenience wrappers
at the end (``swa``, ``dswa``, ``gdn``, ``hybrid``, ``Stream``) allocate outputs and
workspaces with torch and then call those same entry points.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhlta.so")

HLTA_OK, HLTA_ERR_INVALID_ARG, HLTA_ERR_UNSUPPORTED, HLTA_ERR_CUDA, HLTA_ERR_TIMEOUT = range(5)
HLTA_BF16, HLTA_FP32 = 0, 1
HLTA_DEVERR_ATTN_WAIT, HLTA_DEVERR_GDN_WAIT, HLTA_DEVERR_SELFTEST = 0x1, 0x2, 0x4
_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT"}


class HltaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"HLTA_ERR_{_STATUS.get(status, status)}: {msg}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python linear_video_world_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, L, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_float, ctypes.c_size_t
    sig = {
        "hlta_version": (I, []),
        "hlta_last_error": (ctypes.c_char_p, []),
        "hlta_swa_fwd": (I, [P, P, P, P, I, I, I, I, I, I, F, I, P]),
        "hlta_dswa_fwd": (I, [P, P, P, P, I, I, I, I, I, I, I, F, I, P]),
        "hlta_gdn_workspace_bytes": (Z, [I, I, L, I, I, I]),
        "hlta_gdn_chunk_fwd": (I, [P, P, P, P, P, P, P, P, I, I, L, I, I, P, Z, I, P]),
        "hlta_gdn_chunk_fwd_raw": (I, [P, P, P, P, P, F, P, P, P, I, I, L, I, I, P, Z, I, P]),
        "hlta_gdn_chunk_fwd_static": (I, [P, P, P, P, P, P, P, P, I, I, L, I, I, I, P]),
        "hlta_hybrid_workspace_bytes": (Z, [I, I, I, I, I, I, I]),
        "hlta_hybrid_fwd": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, F,
                                P, Z, I, P]),
        "hlta_hybrid_fwd_raw": (I, [P, P, P, P, P, F, P, P, P, I, I, I, I, I, I, I, I, I, I, I,
                                    F, P, Z, I, P]),
        "hlta_stream_create": (I, [ctypes.POINTER(P), I, I, I, I, I, I, I, I, I, I, F, I, P]),
        "hlta_stream_create_ex": (I, [ctypes.POINTER(P), I, I, I, I, I, I, I, I, I, I, F, I, I, P]),
        "hlta_stream_step": (I, [P, P, P, P, P, P, P, P]),
        "hlta_stream_step_frames": (I, [P, P, P, P, P, P, P, I, P]),
        "hlta_stream_state": (I, [P, ctypes.POINTER(P), ctypes.POINTER(I)]),
        "hlta_stream_destroy": (I, [P]),
        "hlta_stream_frame_counter": (I, [P, ctypes.POINTER(P)]),
        "hlta_stream_checkpoint_bytes": (Z, [P]),
        "hlta_stream_save": (I, [P, P, Z, P]),
        "hlta_stream_load": (I, [P, P, Z, P]),
        "hlta_rope": (I, [P, P, I, I, I, I, L, I, I, F, I, I, I, P]),
        "hlta_fp8_quantize_rows": (I, [P, P, I, I, L, I, L, I, P, P, P]),
        "hlta_fp8_quantize_channels": (I, [P, I, I, L, I, P, P, P]),
        "hlta_window_fp8_fwd": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "hlta_window_fwd_lse": (I, [P, P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "hlta_window_bwd_workspace_bytes": (Z, [I, I, I, I]),
        "hlta_window_bwd": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, Z, P]),
        "hlta_gdn_bwd_workspace_bytes": (Z, [I, I, L, I, I]),
        "hlta_gdn_chunk_bwd": (I, [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, L, I, I, P, Z, I,
                                   P]),
        "hlta_device_status": (I, [P, ctypes.POINTER(ctypes.c_uint)]),
        "hlta_kernel_launches": (ctypes.c_ulonglong, []),
        "hlta_wait_expiry_selftest": (I, [ctypes.c_ulonglong, P]),
        "hlta_set_profile_events": (I, [ctypes.POINTER(P)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(status: int) -> None:
    if status != HLTA_OK:
        raise HltaError(status, (_lib.hlta_last_error() or b"").decode(errors="replace"))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dt(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return HLTA_BF16
    if t.dtype == torch.float32:
        return HLTA_FP32
    raise HltaError(HLTA_ERR_INVALID_ARG, f"unsupported dtype {t.dtype}")


def _need(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise HltaError(HLTA_ERR_INVALID_ARG, f"{name} must be a contiguous CUDA tensor")


# ---- entry points (same names as the C ABI) -----------------------------------------

def hlta_version() -> int:
    return int(_lib.hlta_version())


def hlta_swa_fwd(q, k, v, o, B, H, T, N, d, w, scale=0.0, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n)
    _check(_lib.hlta_swa_fwd(_p(q), _p(k), _p(v), _p(o), B, H, T, N, d, w, float(scale),
                             _dt(q), _stream(stream)))


def hlta_dswa_fwd(q, k, v, o, B, H, T, N, d, w, r, scale=0.0, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n)
    _check(_lib.hlta_dswa_fwd(_p(q), _p(k), _p(v), _p(o), B, H, T, N, d, w, r, float(scale),
                              _dt(q), _stream(stream)))


def hlta_gdn_workspace_bytes(B, H, L, d, chunk=64, dt=HLTA_BF16) -> int:
    return int(_lib.hlta_gdn_workspace_bytes(B, H, L, d, chunk, dt))


def hlta_gdn_chunk_fwd(q, k, v, a, b, o, S0, S_out, B, H, L, d, chunk, workspace,
                       stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (a, "a"), (b, "b"), (o, "o"), (workspace, "workspace")):
        _need(t, n)
    _check(_lib.hlta_gdn_chunk_fwd(_p(q), _p(k), _p(v), _p(a), _p(b), _p(o), _p(S0), _p(S_out),
                                   B, H, L, d, chunk, _p(workspace), workspace.numel() * workspace.element_size(),
                                   _dt(q), _stream(stream)))


def hlta_gdn_chunk_fwd_raw(q, k, v, x, y, c, o, S0, S_out, B, H, L, d, chunk, workspace,
                           stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (x, "x"), (y, "y"), (o, "o"), (workspace, "workspace")):
        _need(t, n)
    _check(_lib.hlta_gdn_chunk_fwd_raw(_p(q), _p(k), _p(v), _p(x), _p(y), float(c), _p(o), _p(S0),
                                       _p(S_out), B, H, L, d, chunk, _p(workspace),
                                       workspace.numel() * workspace.element_size(), _dt(q),
                                       _stream(stream)))


HLTA_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


def hlta_gdn_chunk_fwd_static(q, k, v, a, b, o, S0, S_out, B, H, L, d, chunk, stream=None):
    """hlta_gdn_chunk_fwd without a workspace argument: the library's built-in scratch is used
    (for callers that may not allocate device memory; see include/hlta.h)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (a, "a"), (b, "b"), (o, "o")):
        _need(t, n)
    _check(_lib.hlta_gdn_chunk_fwd_static(_p(q), _p(k), _p(v), _p(a), _p(b), _p(o), _p(S0),
                                          _p(S_out), B, H, L, d, chunk, _dt(q), _stream(stream)))


def hlta_hybrid_workspace_bytes(B, Hg, T, N, d, chunk=64, dt=HLTA_BF16) -> int:
    return int(_lib.hlta_hybrid_workspace_bytes(B, Hg, T, N, d, chunk, dt))


def hlta_hybrid_fwd(q, k, v, a, b, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa, r,
                    chunk, scale, workspace, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_p(workspace), workspace.numel() * workspace.element_size())
    _check(_lib.hlta_hybrid_fwd(_p(q), _p(k), _p(v), _p(a), _p(b), _p(o), _p(S0), _p(S_out),
                                B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa, r, chunk, float(scale),
                                ws_ptr, ws_bytes, _dt(q), _stream(stream)))


def hlta_hybrid_fwd_raw(q, k, v, x, y, c, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa,
                        r, chunk, scale, workspace, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, n)
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (_p(workspace), workspace.numel() * workspace.element_size())
    _check(_lib.hlta_hybrid_fwd_raw(_p(q), _p(k), _p(v), _p(x), _p(y), float(c), _p(o), _p(S0),
                                    _p(S_out), B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa, r, chunk,
                                    float(scale), ws_ptr, ws_bytes, _dt(q), _stream(stream)))


def _need_types(x, x8, scales):
    import torch
    if x.dtype != torch.bfloat16 or x8.dtype != torch.uint8 or scales.dtype != torch.float32:
        raise HltaError(HLTA_ERR_INVALID_ARG, "FP8 quantisation takes bf16 x, uint8 codes and "
                        "float32 scales")


def hlta_fp8_quantize_rows(x, shift, B, H, L, d, frame_rows, block_rows, x8, scales,
                           stream=None):
    for t, n in ((x, "x"), (x8, "x8"), (scales, "scales")):
        _need(t, n)
    _need_types(x, x8, scales)
    if shift is not None:
        _need(shift, "shift")
    _check(_lib.hlta_fp8_quantize_rows(_p(x), _p(shift), B, H, L, d, frame_rows, block_rows,
                                       _p(x8), _p(scales), _stream(stream)))


def hlta_fp8_quantize_channels(x, B, H, L, d, x8, scales, stream=None):
    for t, n in ((x, "x"), (x8, "x8"), (scales, "scales")):
        _need(t, n)
    _need_types(x, x8, scales)
    _check(_lib.hlta_fp8_quantize_channels(_p(x), B, H, L, d, _p(x8), _p(scales),
                                           _stream(stream)))


def hlta_window_fp8_fwd(q8, qs, k8, ks, v8, vs, o, B, H, T, N, d, w, r, scale=0.0, stream=None):
    for t, n in ((q8, "q8"), (qs, "q_scales"), (k8, "k8"), (ks, "k_scales"), (v8, "v8"),
                 (vs, "v_scales"), (o, "o")):
        _need(t, n)
    _check(_lib.hlta_window_fp8_fwd(_p(q8), _p(qs), _p(k8), _p(ks), _p(v8), _p(vs), _p(o), B, H,
                                    T, N, d, w, r, float(scale), _stream(stream)))


def _need_bf16(*ts):
    import torch
    if any(t.dtype != torch.bfloat16 for t in ts):
        raise HltaError(HLTA_ERR_INVALID_ARG, "the attention training pair takes bf16 tensors")


def hlta_window_fwd_lse(q, k, v, o, lse, B, H, T, N, d, w, r, scale=0.0, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse")):
        _need(t, n)
    _need_bf16(q, k, v, o)
    _check(_lib.hlta_window_fwd_lse(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, T, N, d, w, r,
                                    float(scale), _stream(stream)))


def hlta_window_bwd_workspace_bytes(B, H, T, N) -> int:
    return int(_lib.hlta_window_bwd_workspace_bytes(B, H, T, N))


def hlta_window_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, N, d, w, r, scale, workspace,
                    stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dO, "dO"), (dq, "dq"),
                 (dk, "dk"), (dv, "dv"), (workspace, "workspace")):
        _need(t, n)
    _need_bf16(q, k, v, o, dO, dq, dk, dv)
    _check(_lib.hlta_window_bwd(_p(q), _p(k), _p(v), _p(o), _p(lse), _p(dO), _p(dq), _p(dk),
                                _p(dv), B, H, T, N, d, w, r, float(scale), _p(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def hlta_gdn_bwd_workspace_bytes(B, H, L, d=128, chunk=64) -> int:
    return int(_lib.hlta_gdn_bwd_workspace_bytes(B, H, L, d, chunk))


def hlta_rope(q, k, B, H, h0, Hr, L, N, d, base=10000.0, pos_mode=0, inverse=False,
              stream=None):
    for t, n in ((q, "q"), (k, "k")):
        if t is not None:
            _need(t, n)
    ref = q if q is not None else k
    _check(_lib.hlta_rope(_p(q), _p(k), B, H, h0, Hr, L, N, d, float(base), int(pos_mode),
                          1 if inverse else 0, _dt(ref), _stream(stream)))


def rope(q, k, N, heads=None, base=10000.0, pos_mode=0, inverse=False, stream=None):
    """Rotate q and k ([B, H, L, d]) in place; `heads` = (h0, Hr) or None for all heads."""
    ref = q if q is not None else k
    B, H, L, d = ref.shape
    h0, Hr = heads if heads is not None else (0, H)
    hlta_rope(q, k, B, H, h0, Hr, L, N, d, base, pos_mode, inverse, stream)
    return q, k


def hlta_gdn_chunk_bwd(q, k, v, a, b, S0, dO, dS_final, dq, dk, dv, da, db, dS0, B, H, L, d,
                       chunk, workspace, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (a, "a"), (b, "b"), (dO, "dO"), (dq, "dq"),
                 (dk, "dk"), (dv, "dv"), (da, "da"), (db, "db"), (workspace, "workspace")):
        _need(t, n)
    for t, n in ((S0, "S0"), (dS_final, "dS_final"), (dS0, "dS0")):
        if t is not None:
            _need(t, n)
    _check(_lib.hlta_gdn_chunk_bwd(_p(q), _p(k), _p(v), _p(a), _p(b), _p(S0), _p(dO),
                                   _p(dS_final), _p(dq), _p(dk), _p(dv), _p(da), _p(db), _p(dS0),
                                   B, H, L, d, chunk, _p(workspace),
                                   workspace.numel() * workspace.element_size(), _dt(q),
                                   _stream(stream)))


def hlta_device_status(stream=None) -> int:
    code = ctypes.c_uint(0)
    _check(_lib.hlta_device_status(_stream(stream), ctypes.byref(code)))
    return int(code.value)


def hlta_device_status_code(stream=None):
    """(status, raw device error word) without raising: hlta_device_status for callers that
    handle an expired wait themselves."""
    code = ctypes.c_uint(0)
    st = int(_lib.hlta_device_status(_stream(stream), ctypes.byref(code)))
    return st, int(code.value)


def hlta_kernel_launches() -> int:
    return int(_lib.hlta_kernel_launches())


def hlta_wait_expiry_selftest(cycles, stream=None):
    _check(_lib.hlta_wait_expiry_selftest(int(cycles), _stream(stream)))


def hlta_set_profile_events(events):
    """events: None, or 5 torch.cuda.Event objects (already created on the device)."""
    if events is None:
        _check(_lib.hlta_set_profile_events(None))
        return
    arr = (ctypes.c_void_p * 5)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib.hlta_set_profile_events(arr))


# ---- convenience wrappers (allocate with torch, then call the entry points) ----------

def _workspace(nbytes, device):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def swa(q, k, v, T, N, w, scale=0.0, out=None, stream=None):
    import torch
    B, H, _, d = q.shape
    o = torch.empty_like(q) if out is None else out
    hlta_swa_fwd(q, k, v, o, B, H, T, N, d, w, scale, stream)
    return o


def dswa(q, k, v, T, N, w, r, scale=0.0, out=None, stream=None):
    import torch
    B, H, _, d = q.shape
    o = torch.empty_like(q) if out is None else out
    hlta_dswa_fwd(q, k, v, o, B, H, T, N, d, w, r, scale, stream)
    return o


def fp8_quantize_rows(x, frame_rows, block_rows, shift=None, stream=None):
    """E4M3 codes (uint8, shape of x) and per-block scales [B, H, nframes, nblocks] of a bf16
    [B, H, L, d] tensor; blocks of block_rows rows inside frames of frame_rows rows."""
    import torch
    B, H, L, d = x.shape
    nf, nb = -(-L // frame_rows), -(-frame_rows // block_rows)
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty((B, H, nf, nb), dtype=torch.float32, device=x.device)
    hlta_fp8_quantize_rows(x, shift, B, H, L, d, frame_rows, block_rows, x8, sc, stream)
    return x8, sc


def fp8_quantize_channels(x, stream=None):
    """E4M3 codes and per-channel scales [B, H, d] of a bf16 [B, H, L, d] tensor."""
    import torch
    B, H, L, d = x.shape
    x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty((B, H, d), dtype=torch.float32, device=x.device)
    hlta_fp8_quantize_channels(x, B, H, L, d, x8, sc, stream)
    return x8, sc


def fp8_quantize_window_inputs(q, k, v, T, N, k_shift=None, stream=None):
    """The three quantisations the FP8 window attention takes: q in 128-row blocks of the
    head, k in 64-row runs of each frame (optionally minus a per-channel shift), v per channel.
    Returns (q8, qs, k8, ks, v8, vs)."""
    q8, qs = fp8_quantize_rows(q, T * N, 128, None, stream)
    k8, ks = fp8_quantize_rows(k, N, 64, k_shift, stream)
    v8, vs = fp8_quantize_channels(v, stream)
    return q8, qs, k8, ks, v8, vs


def window_fp8(q8, qs, k8, ks, v8, vs, T, N, w, r=1, scale=0.0, out=None, stream=None):
    """FP8 window attention (SWA for r = 1, DSWA otherwise); bf16 output [B, H, T*N, d]."""
    import torch
    B, H, L, d = q8.shape
    o = torch.empty((B, H, L, d), dtype=torch.bfloat16, device=q8.device) if out is None else out
    hlta_window_fp8_fwd(q8, qs, k8, ks, v8, vs, o, B, H, T, N, d, w, r, scale, stream)
    return o


def window_fwd_lse(q, k, v, T, N, w, r=1, scale=0.0, out=None, lse=None, stream=None):
    """Window attention forward that also returns the per-row log-sum-exp (for the backward)."""
    import torch
    B, H, L, d = q.shape
    o = torch.empty_like(q) if out is None else out
    ls = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if lse is None else lse
    hlta_window_fwd_lse(q, k, v, o, ls, B, H, T, N, d, w, r, scale, stream)
    return o, ls


def window_bwd(q, k, v, o, lse, dO, T, N, w, r=1, scale=0.0, grads=None, workspace=None,
               stream=None):
    """Gradients (dq, dk, dv) of the window attention for the upstream gradient dO."""
    import torch
    B, H, L, d = q.shape
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q) for _ in range(3))
    ws = workspace if workspace is not None else _workspace(
        hlta_window_bwd_workspace_bytes(B, H, T, N), q.device)
    hlta_window_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, T, N, d, w, r, scale, ws, stream)
    return dq, dk, dv


def gdn_bwd(q, k, v, a, b, dO, S0=None, dS_final=None, chunk=64, workspace=None, stream=None):
    """Gradients (dq, dk, dv, da, db, dS0) of the gated delta rule."""
    import torch
    B, H, L, d = q.shape
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    da, db = (torch.empty((B, H, L), dtype=torch.float32, device=q.device) for _ in range(2))
    dS0 = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    ws = workspace if workspace is not None else _workspace(
        hlta_gdn_bwd_workspace_bytes(B, H, L, d, chunk), q.device)
    hlta_gdn_chunk_bwd(q, k, v, a, b, S0, dO, dS_final, dq, dk, dv, da, db, dS0, B, H, L, d,
                       chunk, ws, stream)
    return dq, dk, dv, da, db, dS0


def gdn(q, k, v, a, b, S0=None, chunk=64, out=None, S_out=None, workspace=None, stream=None):
    import torch
    B, H, L, d = q.shape
    o = torch.empty_like(q) if out is None else out
    if S_out is None:
        S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(hlta_gdn_workspace_bytes(B, H, L, d, chunk, _dt(q)), q.device)
    hlta_gdn_chunk_fwd(q, k, v, a, b, o, S0, S_out, B, H, L, d, chunk, workspace, stream)
    return o, S_out


def gdn_raw(q, k, v, x, y, c, S0=None, chunk=64, out=None, S_out=None, workspace=None,
            stream=None):
    """GDN heads from raw q, k and raw gate inputs x, y (see hlta_gdn_chunk_fwd_raw)."""
    import torch
    B, H, L, d = q.shape
    o = torch.empty_like(q) if out is None else out
    if S_out is None:
        S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(hlta_gdn_workspace_bytes(B, H, L, d, chunk, _dt(q)), q.device)
    hlta_gdn_chunk_fwd_raw(q, k, v, x, y, c, o, S0, S_out, B, H, L, d, chunk, workspace, stream)
    return o, S_out


def hybrid_raw(q, k, v, x, y, c, Hs, Hd, Hg, T, N, w_swa, w_dswa, r, S0=None, chunk=64,
               scale=0.0, out=None, S_out=None, workspace=None, stream=None):
    """The hybrid operator with raw GDN inputs (see hlta_hybrid_fwd_raw)."""
    import torch
    B, H, L, d = q.shape
    o = torch.empty_like(q) if out is None else out
    if Hg and S_out is None:
        S_out = torch.empty((B, Hg, d, d), dtype=torch.float32, device=q.device)
    if Hg and workspace is None:
        workspace = _workspace(hlta_hybrid_workspace_bytes(B, Hg, T, N, d, chunk, _dt(q)), q.device)
    hlta_hybrid_fwd_raw(q, k, v, x, y, c, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa,
                        r, chunk, scale, workspace, stream)
    return o, S_out


def hybrid(q, k, v, a, b, Hs, Hd, Hg, T, N, w_swa, w_dswa, r, S0=None, chunk=64, scale=0.0,
           out=None, S_out=None, workspace=None, stream=None):
    import torch
    B, H, L, d = q.shape
    o = torch.empty_like(q) if out is None else out
    if Hg and S_out is None:
        S_out = torch.empty((B, Hg, d, d), dtype=torch.float32, device=q.device)
    if Hg and workspace is None:
        workspace = _workspace(hlta_hybrid_workspace_bytes(B, Hg, T, N, d, chunk, _dt(q)), q.device)
    hlta_hybrid_fwd(q, k, v, a, b, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa, w_dswa, r,
                    chunk, scale, workspace, stream)
    return o, S_out


class Stream:
    """Streaming cache (hlta_stream_create_ex / _step / _step_frames / _state /
    _frame_counter / _checkpoint_bytes / _save / _load / _destroy). A step may be captured into a CUDA graph and replayed for the
    following frames: the frame index lives in a device counter that every step advances."""

    def __init__(self, B, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk=64, scale=0.0,
                 dtype=None, S0=None, max_step_frames=1):
        import torch
        dt = HLTA_BF16 if dtype in (None, torch.bfloat16) else HLTA_FP32
        self._h = ctypes.c_void_p()
        _check(_lib.hlta_stream_create_ex(ctypes.byref(self._h), B, Hs, Hd, Hg, N, d, w_swa,
                                          w_dswa, r, chunk, float(scale), int(max_step_frames),
                                          dt, _p(S0)))
        self.B, self.H, self.Hg, self.N, self.d = B, Hs + Hd + Hg, Hg, N, d

    def step(self, q, k, v, a, b, out=None, stream=None):
        import torch
        o = torch.empty_like(q) if out is None else out
        _check(_lib.hlta_stream_step(self._h, _p(q), _p(k), _p(v), _p(a), _p(b), _p(o),
                                     _stream(stream)))
        return o

    def step_frames(self, q, k, v, a, b, frames, out=None, stream=None):
        """Append `frames` frames per rollout at once (inputs [B, H, frames*N, d])."""
        import torch
        o = torch.empty_like(q) if out is None else out
        _check(_lib.hlta_stream_step_frames(self._h, _p(q), _p(k), _p(v), _p(a), _p(b), _p(o),
                                            int(frames), _stream(stream)))
        return o

    def state(self):
        """(device address of the [B,Hg,d,d] fp32 state, frames appended so far)."""
        ptr, n = ctypes.c_void_p(), ctypes.c_int()
        _check(_lib.hlta_stream_state(self._h, ctypes.byref(ptr), ctypes.byref(n)))
        return ptr.value, n.value

    def frame_counter(self):
        """Device address of the cache's frame counter (an int advanced by every step, in
        stream order, replays of a captured step included)."""
        ptr = ctypes.c_void_p()
        _check(_lib.hlta_stream_frame_counter(self._h, ctypes.byref(ptr)))
        return ptr.value

    def checkpoint_bytes(self):
        return int(_lib.hlta_stream_checkpoint_bytes(self._h))

    def save(self, stream=None):
        """The cache's checkpoint image (hlta_stream_save) as a uint8 numpy array."""
        import numpy as np
        buf = np.empty(self.checkpoint_bytes(), dtype=np.uint8)
        _check(_lib.hlta_stream_save(self._h, buf.ctypes.data, buf.nbytes, _stream(stream)))
        return buf

    def load(self, image, stream=None):
        """Resume from a checkpoint image (hlta_stream_load)."""
        import numpy as np
        buf = np.ascontiguousarray(image, dtype=np.uint8)
        _check(_lib.hlta_stream_load(self._h, buf.ctypes.data, buf.nbytes, _stream(stream)))

    def state_tensor(self):
        """A torch copy of the carried state [B, Hg, d, d] fp32 (ordered on the current stream)."""
        import torch
        ptr, _ = self.state()

        class _View:   # exposes the cache's device buffer to torch without copying
            __cuda_array_interface__ = {"shape": (self.B, self.Hg, self.d, self.d),
                                        "typestr": "<f4", "data": (ptr, False), "version": 2}
        return torch.as_tensor(_View(), device="cuda").clone()

    def close(self):
        if self._h:
            _check(_lib.hlta_stream_destroy(self._h))
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
