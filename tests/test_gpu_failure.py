"""Failure detection on the device: a bounded mbarrier wait that runs out reaches the host as
HLTA_ERR_TIMEOUT with the waiting kernel's bit, clears on reading, and leaves the context
usable. The expiry is made on purpose by hlta_wait_expiry_selftest (a wait on a barrier that
nothing arrives at, with a short cycle limit); nothing faults, traps or hangs."""
import ctypes

import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like


def test_selftest_rejects_bad_limits_on_host():
    import linear_video_world_b200 as h
    for c in (0, (1 << 32) + 1):
        assert h._lib.hlta_wait_expiry_selftest(ctypes.c_ulonglong(c), None) == h.HLTA_ERR_INVALID_ARG
        assert b"cycles" in h._lib.hlta_last_error()


@pytest.mark.gpu
def test_expired_wait_reported_then_cleared_and_context_usable(orc):
    import linear_video_world_b200 as h
    assert h.hlta_device_status_code() == (h.HLTA_OK, 0)
    h.hlta_wait_expiry_selftest(1 << 22)            # about 2 ms at the B200's clock
    st, code = h.hlta_device_status_code()
    assert st == h.HLTA_ERR_TIMEOUT
    assert code == h.HLTA_DEVERR_SELFTEST
    assert b"bounded wait" in h._lib.hlta_last_error()
    assert h.hlta_device_status_code() == (h.HLTA_OK, 0)   # read once, cleared
    # the context still runs the library's kernels correctly
    wl = hi.Workload("t", B=1, Hs=1, Hd=1, Hg=1, d=128, T=3, N=100, w_swa=2, w_dswa=2, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=5)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    o, S = h.hybrid(q, k, v, a, b, 1, 1, 1, wl.T, wl.N, 2, 2, 2, out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status_code() == (h.HLTA_OK, 0)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], 1, 1, 1, wl.T, wl.N, 2, 2, 2)
    assert maxabs(o, o_ref) <= 2e-2
    assert maxabs(S, S_ref) <= 2e-2


@pytest.mark.gpu
def test_launch_counter_counts_library_kernels():
    import linear_video_world_b200 as h
    n0 = h.hlta_kernel_launches()
    h.hlta_wait_expiry_selftest(1)
    torch.cuda.synchronize()
    assert h.hlta_kernel_launches() - n0 == 1
    h.hlta_device_status_code()
