"""Checkpoint and resume of a streaming cache (hlta_stream_save / hlta_stream_load): a cache
resumed from an image continues bit for bit as the saved one does, and images of another
cache, or damaged ones, are refused without touching the cache."""
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev

pytestmark = pytest.mark.gpu


def _wl():
    return hi.Workload("t", B=2, Hs=1, Hd=1, Hg=1, d=128, T=9, N=130, w_swa=3, w_dswa=3, r=2,
                       chunk=64, dtype="bf16", decay=1.0)


def _frame(x, f, N):
    s = slice(f * N, (f + 1) * N)
    return [x[n][:, :, s].contiguous() for n in "qkvab"]


def test_resumed_cache_continues_bit_identical():
    import linear_video_world_b200 as h
    wl = _wl()
    x = {n: dev(t) for n, t in hi.make_inputs(wl, seed=71).items()}
    args = (wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r)
    a = h.Stream(*args)
    for f in range(5):                      # past the DSWA ring's first wrap (5 slots)
        a.step(*_frame(x, f, wl.N))
    img = a.save()
    assert img.nbytes == a.checkpoint_bytes()
    assert bytes(img[:4]) == b"HLTC"
    b = h.Stream(*args)
    b.load(img)
    assert b.state()[1] == 5
    assert torch.equal(a.state_tensor(), b.state_tensor())
    for f in range(5, wl.T):
        oa = a.step(*_frame(x, f, wl.N))
        ob = b.step(*_frame(x, f, wl.N))
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), f
    # equal outputs also show the device frame counter was restored (the ring slots and taps
    # the kernels use come from it)
    assert torch.equal(a.state_tensor(), b.state_tensor())
    assert a.state()[1] == b.state()[1] == wl.T
    for st in (a, b):
        st.close()


def test_foreign_or_damaged_images_are_refused():
    import linear_video_world_b200 as h
    wl = _wl()
    x = {n: dev(t) for n, t in hi.make_inputs(wl, seed=72).items()}
    args = [wl.B, wl.Hs, wl.Hd, wl.Hg, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r]
    a = h.Stream(*args)
    a.step(*_frame(x, 0, wl.N))
    img = a.save()
    S_before = a.state_tensor()
    bad = img.copy()
    bad[0] = ord("X")                       # magic
    with pytest.raises(h.HltaError) as e:
        a.load(bad)
    assert e.value.status == h.HLTA_ERR_INVALID_ARG
    with pytest.raises(h.HltaError):
        a.load(img[:-1])                    # size
    other = h.Stream(*args[:7], wl.w_dswa, 3)   # another dilation: other ring slots
    assert other.checkpoint_bytes() != a.checkpoint_bytes()
    with pytest.raises(h.HltaError):
        other.load(img)
    same_size = h.Stream(*args, scale=0.05)     # same sizes, another scale
    assert same_size.checkpoint_bytes() == a.checkpoint_bytes()
    with pytest.raises(h.HltaError):
        same_size.load(img)
    assert torch.equal(a.state_tensor(), S_before)
    for st in (a, other, same_size):
        st.close()
