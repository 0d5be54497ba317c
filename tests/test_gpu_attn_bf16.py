"""GPU parity of the tensor-core windowed attention (bf16 I/O, fp32 accumulation) against the
CPU oracle: max-abs <= 2e-2. Edge shapes are compared in full; the 480P workload on sampled
query rows (every frame's first and last row plus seeded random rows, all heads)."""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _wl(B, H, T, N, w, r):
    return hi.Workload("t", B=B, Hs=0, Hd=H, Hg=0, d=128, T=T, N=N, w_swa=w, w_dswa=w, r=r,
                       chunk=64, dtype="bf16", decay=1.0)


@pytest.mark.parametrize("B,H,T,N,w", [
    (1, 1, 4, 256, 2),      # frames aligned to 128-row tiles
    (2, 3, 5, 200, 3),      # tiles straddle frames, ragged key tiles
    (1, 2, 3, 40, 2),       # several frames per query tile
    (1, 1, 6, 1, 3),        # one token per frame
    (1, 1, 2, 300, 5),      # window longer than the clip
    (1, 2, 3, 1560, 3),     # 480P frame size
])
def test_swa_bf16_full(h, orc, B, H, T, N, w):
    wl = _wl(B, H, T, N, w, 1)
    x = hi.make_inputs(wl, seed=11 + T * N)
    q, k, v = (dev(x[n]) for n in "qkv")
    o = h.swa(q, k, v, T, N, w, out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert maxabs(o, orc.swa(x["q"], x["k"], x["v"], T, N, w)) <= TOL


@pytest.mark.parametrize("B,H,T,N,w,r", [
    (1, 2, 9, 150, 3, 3),
    (1, 1, 4, 300, 4, 2),   # taps before frame 0 dropped
    (2, 1, 7, 64, 3, 1),    # r = 1 (= SWA)
    (1, 1, 13, 97, 3, 4),
])
def test_dswa_bf16_full(h, orc, B, H, T, N, w, r):
    wl = _wl(B, H, T, N, w, r)
    x = hi.make_inputs(wl, seed=23 + T * N)
    q, k, v = (dev(x[n]) for n in "qkv")
    o = h.dswa(q, k, v, T, N, w, r, out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert maxabs(o, orc.dswa(x["q"], x["k"], x["v"], T, N, w, r)) <= TOL


def test_480p_softmax_branches_sampled(h, orc):
    """The 480P workload's SWA (w=3) and DSWA (w=3, r=4) heads through the hybrid layout's
    entry points, compared on sampled rows of every head."""
    wl = hi.WORKLOADS["480p"]
    x = hi.make_inputs(wl, seed=0)
    Hs, Hd = wl.Hs, wl.Hd
    q, k, v = (dev(x[n][:, :Hs + Hd]) for n in "qkv")
    o_s = h.swa(q[:, :Hs].contiguous(), k[:, :Hs].contiguous(), v[:, :Hs].contiguous(),
                wl.T, wl.N, wl.w_swa)
    o_d = h.dswa(q[:, Hs:].contiguous(), k[:, Hs:].contiguous(), v[:, Hs:].contiguous(),
                 wl.T, wl.N, wl.w_dswa, wl.r)
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    rows = hi.sample_rows(wl.L, wl.N, 256, seed=1).numpy()
    L = wl.L
    flat_s = (np.arange(Hs)[:, None] * L + rows[None, :]).reshape(-1)
    ref_s = orc.swa(x["q"][0, :Hs], x["k"][0, :Hs], x["v"][0, :Hs], wl.T, wl.N, wl.w_swa,
                    rows=flat_s)
    got_s = o_s[0].reshape(-1, wl.d)[torch.from_numpy(flat_s).cuda()]
    assert maxabs(got_s, ref_s) <= TOL
    flat_d = (np.arange(Hd)[:, None] * L + rows[None, :]).reshape(-1)
    ref_d = orc.dswa(x["q"][0, Hs:Hs + Hd], x["k"][0, Hs:Hs + Hd], x["v"][0, Hs:Hs + Hd], wl.T,
                     wl.N, wl.w_dswa, wl.r, rows=flat_d)
    got_d = o_d[0].reshape(-1, wl.d)[torch.from_numpy(flat_d).cuda()]
    assert maxabs(got_d, ref_d) <= TOL
    assert torch.isfinite(o_s).all() and torch.isfinite(o_d).all()


def test_swa_and_dswa_heads_in_one_launch(h, orc):
    """SWA and DSWA heads of one tensor as a hybrid call without GDN heads: both branches'
    units share one persistent launch (B = 2, ragged key tiles, tiles straddling frames)."""
    B, Hs, Hd, T, N, w_s, w_d, r = 2, 2, 3, 7, 150, 3, 3, 2
    wl = hi.Workload("t", B=B, Hs=Hs, Hd=Hd, Hg=0, d=128, T=T, N=N, w_swa=w_s, w_dswa=w_d, r=r,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=5)
    q, k, v = (dev(x[n]) for n in "qkv")
    o, _ = h.hybrid(q, k, v, None, None, Hs, Hd, 0, T, N, w_s, w_d, r, out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    sub = {n: (x[n][:, :Hs].contiguous(), x[n][:, Hs:].contiguous()) for n in "qkv"}
    ref_s = orc.swa(sub["q"][0], sub["k"][0], sub["v"][0], T, N, w_s)
    ref_d = orc.dswa(sub["q"][1], sub["k"][1], sub["v"][1], T, N, w_d, r)
    assert maxabs(o[:, :Hs], ref_s) <= TOL
    assert maxabs(o[:, Hs:], ref_d) <= TOL


def test_work_counter_survives_many_launches(h):
    """More launches than the kernel has work counters, of different unit counts and on two
    streams: every launch hands out all its units (each output equals the first of its shape,
    bit for bit), so each counter is back at zero for its next use."""
    shapes = [(2, 3, 5, 200, 3), (1, 1, 2, 300, 5), (1, 2, 3, 1560, 3)]
    data, first = [], []
    for i, (B, H, T, N, w) in enumerate(shapes):
        x = hi.make_inputs(_wl(B, H, T, N, w, 1), seed=100 + i)
        q, k, v = (dev(x[n]) for n in "qkv")
        data.append((q, k, v, T, N, w))
        first.append(h.swa(q, k, v, T, N, w))
    side = torch.cuda.Stream()
    outs = []
    for it in range(150):
        q, k, v, T, N, w = data[it % 3]
        stream = side if it % 5 == 4 else torch.cuda.current_stream()
        with torch.cuda.stream(stream):
            outs.append((it % 3, h.swa(q, k, v, T, N, w, out=poison_like(q))))
        if it % 5 == 4:
            torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    for j, o in outs:
        assert torch.equal(o, first[j])
