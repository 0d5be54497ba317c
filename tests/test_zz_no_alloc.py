"""hlta_gdn_chunk_fwd_static: the gated delta rule for callers that may not allocate device
memory (a host application that owns the device-memory budget and passes in only inputs and
outputs, or a latency-critical loop that must stay out of the allocator). It uses a scratch
array built into the library instead of a caller workspace and runs the same kernels as
hlta_gdn_chunk_fwd, so its results must equal that entry point's bit for bit; they are also
checked against the oracle's token recurrence. Collected last (file name) so that a run
stopping at its first failure has already run every other test; it passes alone in a fresh
process too.
"""
import ctypes

import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def _case(seed, H, L, dtype):
    wl = hi.Workload("t", B=1, Hs=0, Hd=0, Hg=H, d=128, T=L, N=1, w_swa=1, w_dswa=1, r=1,
                     chunk=64, dtype=dtype, decay=1.0)
    return hi.make_inputs(wl, seed=seed), hi.random_state(1, H, 128, seed=seed + 50, scale=0.1)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_static_scratch_matches_workspace_entry_point_twice(orc, dtype):
    import linear_video_world_b200 as h
    B, H, d = 1, 2, 128
    # two calls in a row: the second reuses the scratch the first left behind
    for call, (seed, L) in enumerate(((11, 1000), (12, 777))):
        x, S0 = _case(seed, H, L, dtype)
        q, k, v, a, b = (dev(x[n]) for n in "qkvab")
        o_ref, S_ref = h.gdn(q, k, v, a, b, S0=dev(S0))
        o = poison_like(q)
        S = torch.full((B, H, d, d), float("nan"), device="cuda")
        h.hlta_gdn_chunk_fwd_static(q, k, v, a, b, o, dev(S0), S, B, H, L, d, 64)
        torch.cuda.synchronize()
        assert h.hlta_device_status() == 0
        assert torch.equal(o, o_ref), call
        assert torch.equal(S, S_ref), call
        o_orc, S_orc = orc.gdn(x["q"], x["k"], x["v"], x["a"], x["b"], S0.double().numpy())
        assert maxabs(o, o_orc) <= TOL[dtype], call
        assert maxabs(S, S_orc) <= TOL[dtype], call


def test_static_scratch_rejects_oversized_problem_on_host():
    """A problem whose workspace exceeds the built-in scratch is refused before any launch."""
    import linear_video_world_b200 as h
    lib = h._lib
    p = ctypes.c_void_p(256)
    L = 1 << 20
    assert h.hlta_gdn_workspace_bytes(1, 8, L, 128) > h.HLTA_STATIC_SCRATCH_BYTES
    st = lib.hlta_gdn_chunk_fwd_static(p, p, p, p, p, p, None, None, 1, 8, L, 128, 64,
                                       h.HLTA_BF16, None)
    assert st == h.HLTA_ERR_INVALID_ARG
    assert b"scratch" in lib.hlta_last_error()
