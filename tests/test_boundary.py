"""CPU-only checks of the C ABI: the library loads, exports every entry point that
include/hlta.h declares, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hlta.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hlta_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import linear_video_world_b200 as h
    return h._lib


def test_header_declares_the_documented_calls():
    names = _declared()
    for n in ("hlta_swa_fwd", "hlta_dswa_fwd", "hlta_gdn_chunk_fwd", "hlta_hybrid_fwd",
              "hlta_stream_create", "hlta_stream_step", "hlta_stream_destroy", "hlta_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_version(lib):
    assert lib.hlta_version() >= 100


def test_null_pointers_rejected_on_host(lib):
    import linear_video_world_b200 as h
    st = lib.hlta_swa_fwd(None, None, None, None, 1, 1, 2, 16, 128, 2, 0.0, h.HLTA_BF16, None)
    assert st == h.HLTA_ERR_INVALID_ARG
    assert b"null" in lib.hlta_last_error()


def test_bad_shapes_rejected_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    assert lib.hlta_swa_fwd(p, p, p, p, 1, 1, 0, 16, 128, 2, 0.0, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_swa_fwd(p, p, p, p, 1, 1, 2, 16, 64, 2, 0.0, h.HLTA_BF16, None) == h.HLTA_ERR_UNSUPPORTED
    assert lib.hlta_dswa_fwd(p, p, p, p, 1, 1, 2, 16, 128, 2, 0, 0.0, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_dswa_fwd(p, p, p, p, 1, 1, 2, 16, 128, 0, 2, 0.0, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_swa_fwd(p, p, p, ctypes.c_void_p(264), 1, 1, 2, 16, 128, 2, 0.0, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_swa_fwd(p, p, p, p, 1, 1, 2, 16, 129, 2, 0.0, h.HLTA_FP32, None) == h.HLTA_ERR_UNSUPPORTED
    # gated delta rule: chunk other than 64 and a short workspace
    assert lib.hlta_gdn_chunk_fwd(p, p, p, p, p, p, None, None, 1, 1, 100, 128, 32, p, 1 << 30,
                                  h.HLTA_BF16, None) == h.HLTA_ERR_UNSUPPORTED
    assert lib.hlta_gdn_chunk_fwd(p, p, p, p, p, p, None, None, 1, 1, 100, 128, 64, p, 16,
                                  h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert b"workspace" in lib.hlta_last_error()


def test_raw_entry_points_validate_decay_constant_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    for c in (-0.5, float("nan"), float("inf")):
        assert lib.hlta_gdn_chunk_fwd_raw(p, p, p, p, p, c, p, None, None, 1, 1, 100, 128, 64, p,
                                          1 << 30, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
        assert b"decay" in lib.hlta_last_error()
        assert lib.hlta_hybrid_fwd_raw(p, p, p, p, p, c, p, None, None, 1, 1, 1, 1, 2, 16, 128, 2,
                                       2, 2, 64, 0.0, p, 1 << 30, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    # null gate inputs are rejected like null gates
    assert lib.hlta_gdn_chunk_fwd_raw(p, p, p, None, p, 1.0, p, None, None, 1, 1, 100, 128, 64, p,
                                      1 << 30, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG


def test_stream_create_ex_validates_frames_per_step(lib):
    import linear_video_world_b200 as h
    out = ctypes.c_void_p()
    for m in (0, -1, 5000):
        assert lib.hlta_stream_create_ex(ctypes.byref(out), 1, 1, 1, 1, 16, 128, 3, 4, 6, 64, 0.0,
                                         m, h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
        assert not out.value
    assert lib.hlta_stream_step_frames(None, None, None, None, None, None, None, 1, None) == h.HLTA_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    import linear_video_world_b200 as h
    # bf16: 4 arrays of [BH][nchunks][128][64] bf16 (W^T, Qt^T, Up^T, Op^T), 68 fp32 scalars
    # per chunk, and the segment scan's three fp32 [BH][nseg][d][d] arrays (512 chunks per
    # head: 16 segments)
    n = h.hlta_gdn_workspace_bytes(1, 8, 32760, 128, 64, h.HLTA_BF16)
    nch = (32760 + 63) // 64
    arr = 8 * nch * 64 * 128 * 2
    assert n == 4 * arr + ((8 * nch * 68 * 4 + 255) // 256) * 256 + 3 * 8 * 16 * 128 * 128 * 4
    # a head short enough for one segment needs no scan arrays
    n1 = h.hlta_gdn_workspace_bytes(1, 8, 1560, 128, 64, h.HLTA_BF16)
    assert n1 == 4 * (8 * 25 * 64 * 128 * 2) + ((8 * 25 * 68 * 4 + 255) // 256) * 256
    assert h.hlta_hybrid_workspace_bytes(1, 8, 21, 1560, 128, 64, h.HLTA_BF16) == n
    assert h.hlta_gdn_workspace_bytes(1, 1, 10, 64, 64, h.HLTA_FP32) > 5 * 64 * 64 * 4 - 1


def test_stream_create_validates_before_allocating(lib):
    import linear_video_world_b200 as h
    out = ctypes.c_void_p()
    assert lib.hlta_stream_create(ctypes.byref(out), 0, 1, 1, 1, 16, 128, 3, 4, 6, 64, 0.0,
                                  h.HLTA_BF16, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_stream_create(ctypes.byref(out), 1, 1, 1, 1, 16, 128, 3, 4, 6, 32, 0.0,
                                  h.HLTA_BF16, None) == h.HLTA_ERR_UNSUPPORTED
    assert out.value is None


def test_stream_checkpoint_validates_on_host(lib):
    import linear_video_world_b200 as h
    buf = ctypes.create_string_buffer(64)
    assert lib.hlta_stream_checkpoint_bytes(None) == 0
    assert lib.hlta_stream_save(None, buf, 64, None) == h.HLTA_ERR_INVALID_ARG
    assert lib.hlta_stream_load(None, buf, 64, None) == h.HLTA_ERR_INVALID_ARG
    assert b"null" in lib.hlta_last_error()


def test_fp8_entry_points_validate_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    odd = ctypes.c_void_p(264)
    q = lib.hlta_fp8_quantize_rows
    assert q(None, None, 1, 1, 100, 128, 100, 64, p, p, None) == h.HLTA_ERR_INVALID_ARG
    assert q(p, None, 1, 1, 100, 64, 100, 64, p, p, None) == h.HLTA_ERR_UNSUPPORTED
    assert q(p, None, 1, 1, 100, 128, 100, 0, p, p, None) == h.HLTA_ERR_INVALID_ARG
    assert q(p, None, 1, 1, 100, 128, 100, 129, p, p, None) == h.HLTA_ERR_INVALID_ARG
    assert q(p, None, 1, 1, 100, 128, 0, 64, p, p, None) == h.HLTA_ERR_INVALID_ARG
    assert q(p, odd, 1, 1, 100, 128, 100, 64, p, p, None) == h.HLTA_ERR_INVALID_ARG
    assert q(p, None, -1, 1, 100, 128, 100, 64, p, p, None) == h.HLTA_ERR_INVALID_ARG
    c = lib.hlta_fp8_quantize_channels
    assert c(p, 1, 1, 100, 128, None, p, None) == h.HLTA_ERR_INVALID_ARG
    assert c(p, 1, 1, 100, 96, p, p, None) == h.HLTA_ERR_UNSUPPORTED
    assert c(p, 1, 1, 100, 128, p, odd, None) == h.HLTA_ERR_INVALID_ARG
    a = lib.hlta_window_fp8_fwd
    assert a(p, p, p, p, p, None, p, 1, 1, 2, 16, 128, 2, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    assert a(p, p, p, p, p, p, p, 1, 1, 2, 16, 64, 2, 1, 0.0, None) == h.HLTA_ERR_UNSUPPORTED
    assert a(p, p, p, p, p, p, p, 1, 1, 0, 16, 128, 2, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    assert a(p, p, p, p, p, p, p, 1, 1, 2, 16, 128, 0, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    assert a(p, p, p, p, p, p, p, 1, 1, 2, 16, 128, 2, 0, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    assert a(p, odd, p, p, p, p, p, 1, 1, 2, 16, 128, 2, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG


def test_attention_backward_entry_points_validate_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    f = lib.hlta_window_fwd_lse
    assert f(p, p, p, p, None, 1, 1, 2, 16, 128, 2, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    assert f(p, p, p, p, p, 1, 1, 2, 16, 64, 2, 1, 0.0, None) == h.HLTA_ERR_UNSUPPORTED
    assert f(p, p, p, p, p, 1, 1, 2, 16, 128, 0, 1, 0.0, None) == h.HLTA_ERR_INVALID_ARG
    ws = lib.hlta_window_bwd_workspace_bytes(2, 3, 4, 100)
    assert ws == (2 * 3 * 4 * 100 * 4 + 255) // 256 * 256
    b = lib.hlta_window_bwd
    args = [p] * 9 + [2, 3, 4, 100, 128, 2, 1, 0.0, p, ws, None]
    bad = list(args); bad[4] = None
    assert b(*bad) == h.HLTA_ERR_INVALID_ARG
    bad = list(args); bad[18] = ws - 1
    assert b(*bad) == h.HLTA_ERR_INVALID_ARG
    assert b"workspace" in lib.hlta_last_error()
    bad = list(args); bad[13] = 96
    assert b(*bad) == h.HLTA_ERR_UNSUPPORTED
    bad = list(args); bad[7] = ctypes.c_void_p(264)
    assert b(*bad) == h.HLTA_ERR_INVALID_ARG


def test_gdn_backward_entry_point_validates_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    ws = lib.hlta_gdn_bwd_workspace_bytes(1, 2, 100, 128, 64)
    assert ws > 0 and lib.hlta_gdn_bwd_workspace_bytes(1, 2, 100, 64, 64) == 0
    f = lib.hlta_gdn_chunk_bwd
    args = [p, p, p, p, p, None, p, None, p, p, p, p, p, None, 1, 2, 100, 128, 64, p, ws, h.HLTA_BF16, None]
    bad = list(args); bad[0] = None
    assert f(*bad) == h.HLTA_ERR_INVALID_ARG
    bad = list(args); bad[20] = ws - 1
    assert f(*bad) == h.HLTA_ERR_INVALID_ARG and b"workspace" in lib.hlta_last_error()
    bad = list(args); bad[18] = 32
    assert f(*bad) == h.HLTA_ERR_UNSUPPORTED
    bad = list(args); bad[17] = 64
    assert f(*bad) == h.HLTA_ERR_UNSUPPORTED
    bad = list(args); bad[5] = ctypes.c_void_p(264)
    assert f(*bad) == h.HLTA_ERR_INVALID_ARG


def test_rope_entry_point_validates_on_host(lib):
    import linear_video_world_b200 as h
    p = ctypes.c_void_p(256)
    F = ctypes.c_float
    bad = [
        (p, p, 1, 4, 0, 4, 100, 10, 127, F(1e4), 0, 0, h.HLTA_BF16),    # odd d
        (p, p, 1, 4, 0, 4, 100, 10, 130, F(1e4), 0, 0, h.HLTA_BF16),    # d > 128
        (p, p, 1, 4, 2, 3, 100, 10, 128, F(1e4), 0, 0, h.HLTA_BF16),    # heads past H
        (p, p, 1, 4, 0, 4, 100, 10, 128, F(1.0), 0, 0, h.HLTA_BF16),    # base <= 1
        (p, p, 1, 4, 0, 4, 100, 10, 128, F(1e4), 2, 0, h.HLTA_BF16),    # pos_mode
        (p, p, 1, 4, 0, 4, 100, 0, 128, F(1e4), 0, 0, h.HLTA_BF16),     # N < 1
        (ctypes.c_void_p(264), p, 1, 4, 0, 4, 100, 10, 128, F(1e4), 0, 0, h.HLTA_BF16),
        (p, p, 1, 4, 0, 4, 100, 10, 128, F(1e4), 0, 0, 7),               # dtype
    ]
    for args in bad:
        assert lib.hlta_rope(*args, None) == h.HLTA_ERR_INVALID_ARG, args
    # nothing to rotate: accepted without touching a device
    assert lib.hlta_rope(None, None, 1, 4, 0, 4, 100, 10, 128, F(1e4), 0, 0, h.HLTA_BF16, None) == h.HLTA_OK
    assert lib.hlta_rope(p, p, 1, 4, 1, 0, 100, 10, 128, F(1e4), 0, 0, h.HLTA_BF16, None) == h.HLTA_OK


def test_static_scratch_size_matches_header():
    """The binding's copy of HLTA_STATIC_SCRATCH_BYTES is the value include/hlta.h defines."""
    import linear_video_world_b200 as h
    src = open(os.path.join(ROOT, "include", "hlta.h")).read()
    m = re.search(r"#define\s+HLTA_STATIC_SCRATCH_BYTES\s+\(([^)]*)\)", src)
    assert m, "HLTA_STATIC_SCRATCH_BYTES not defined in hlta.h"
    expr = re.sub(r"(\d+)[uUlL]+", r"\1", m.group(1))
    assert re.fullmatch(r"[\d\s*+()]+", expr), expr
    assert eval(expr) == h.HLTA_STATIC_SCRATCH_BYTES
