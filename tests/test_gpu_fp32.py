"""GPU parity of the fp32 path (HLTA_FP32) against the CPU oracle, max-abs <= 1e-4."""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _small(B, Hs, Hd, Hg, d, T, N, w_swa, w_dswa, r):
    return hi.Workload("t", B=B, Hs=Hs, Hd=Hd, Hg=Hg, d=d, T=T, N=N, w_swa=w_swa,
                       w_dswa=w_dswa, r=r, chunk=64, dtype="fp32", decay=1.0)


def test_tiny_fp32_workload_hybrid(h, orc):
    wl = hi.WORKLOADS["tiny_fp32"]
    x = hi.make_inputs(wl, seed=0)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    o = poison_like(q)
    o, S = h.hybrid(q, k, v, a, b, wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r,
                    out=o)
    torch.cuda.synchronize()
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(S, S_ref) <= TOL
    assert h.hlta_device_status() == 0


@pytest.mark.parametrize("T,N,d,w", [(5, 37, 64, 2), (3, 200, 128, 4), (6, 1, 32, 3), (4, 33, 100, 1)])
def test_swa_odd_shapes(h, orc, T, N, d, w):
    wl = _small(2, 2, 0, 0, d, T, N, w, 1, 1)
    x = hi.make_inputs(wl, seed=T * N)
    q, k, v = (dev(x[n]) for n in "qkv")
    o = h.swa(q, k, v, T, N, w, out=poison_like(q))
    torch.cuda.synchronize()
    assert maxabs(o, orc.swa(x["q"], x["k"], x["v"], T, N, w)) <= TOL


@pytest.mark.parametrize("T,N,d,w,r", [(9, 19, 64, 3, 3), (5, 40, 128, 4, 2), (4, 16, 64, 3, 5), (7, 3, 16, 2, 1)])
def test_dswa_odd_shapes(h, orc, T, N, d, w, r):
    wl = _small(1, 0, 3, 0, d, T, N, 1, w, r)
    x = hi.make_inputs(wl, seed=7 + T)
    q, k, v = (dev(x[n]) for n in "qkv")
    o = h.dswa(q, k, v, T, N, w, r, out=poison_like(q))
    torch.cuda.synchronize()
    assert maxabs(o, orc.dswa(x["q"], x["k"], x["v"], T, N, w, r)) <= TOL


@pytest.mark.parametrize("L,d", [(150, 64), (64, 128), (1, 32), (200, 128)])
def test_gdn_chunked_with_state(h, orc, L, d):
    wl = _small(2, 0, 0, 2, d, L, 1, 1, 1, 1)
    x = hi.make_inputs(wl, seed=L + d)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    S0 = hi.random_state(2, 2, d, seed=99, scale=0.3)
    o, S = h.gdn(q, k, v, a, b, S0=dev(S0), out=poison_like(q))
    torch.cuda.synchronize()
    o_ref, S_ref = orc.gdn(x["q"], x["k"], x["v"], x["a"], x["b"], S0.double().numpy())
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(S, S_ref) <= TOL
    # in place: S_out == S0
    S_io = dev(S0)
    h.gdn(q, k, v, a, b, S0=S_io, S_out=S_io)
    torch.cuda.synchronize()
    assert maxabs(S_io, S_ref) <= TOL


def test_stream_steps_equal_hybrid(h, orc):
    wl = _small(2, 1, 1, 1, 64, 7, 24, 3, 3, 2)
    x = hi.make_inputs(wl, seed=5)
    q, k, v, a, b = (dev(x[n]) for n in "qkvab")
    st = h.Stream(wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r,
                  dtype=torch.float32)
    outs = []
    for f in range(wl.T):
        s = slice(f * wl.N, (f + 1) * wl.N)
        outs.append(st.step(q[:, :, s].contiguous(), k[:, :, s].contiguous(),
                            v[:, :, s].contiguous(), a[:, :, s].contiguous(),
                            b[:, :, s].contiguous()))
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=2)
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["a"], x["b"], wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    assert maxabs(o, o_ref) <= TOL
    assert maxabs(st.state_tensor(), S_ref) <= TOL
    assert st.state()[1] == wl.T
    st.close()
