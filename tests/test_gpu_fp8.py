"""GPU parity of the FP8 (E4M3) window attention path against the CPU oracle.

Quantisation is byte work and is compared bit for bit: codes and fp32 scales.

The attention of E4M3 inputs is compared with the oracle's attention of the same codes,
dequantised (the oracle computes the scores, softmax and P V in fp64). The kernel's only
coarse rounding is that of the softmax weights to E4M3 before P V: round to nearest with
3 mantissa bits is a relative error of at most 2^-4 per weight (the weights are kept at or
above 2^-6 of the row's largest, where E4M3 is normal), so an output element may differ from
the exact one by at most 2^-4 times the same attention applied to |v|, plus the bf16 rounding
of the output (2^-8 relative) and fp32 noise. That bound, computed per element from the
oracle, is the tolerance. The error against the attention of the original bf16 inputs (the
cost of quantising q, k, v at all) is a measured figure, checked with a margin.
"""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, poison_like

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _x(B, H, L, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((B, H, L, 128), generator=g) * scale).to(torch.bfloat16).contiguous()


def _inputs(B, H, T, N, seed):
    wl = hi.Workload("t", B=B, Hs=0, Hd=H, Hg=0, d=128, T=T, N=N, w_swa=1, w_dswa=1, r=1,
                     chunk=64, dtype="bf16", decay=1.0)
    return hi.make_inputs(wl, seed=seed)


@pytest.mark.parametrize("B,H,L,frame,block,shift", [
    (1, 2, 300, 100, 64, False),        # short last run in every frame
    (2, 1, 1000, 1000, 128, False),     # query blocks: one frame, short last block
    (1, 1, 3 * 1560, 1560, 64, True),   # 480P frames, with a per-channel shift
    (1, 1, 77, 7, 5, False),            # odd sizes
    (1, 1, 1, 1, 64, False),            # one row
])
def test_quantize_rows_bit_exact(h, orc, B, H, L, frame, block, shift):
    x = _x(B, H, L, seed=L + block, scale=3.0)
    sh = None
    if shift:
        sh = torch.randn((B, H, 128), generator=torch.Generator().manual_seed(1)).float()
    x8, sc = h.fp8_quantize_rows(dev(x), frame, block, shift=None if sh is None else dev(sh))
    torch.cuda.synchronize()
    c_ref, s_ref = orc.fp8_quantize_rows(x, frame, block, shift=sh)
    assert np.array_equal(x8.cpu().numpy(), c_ref)
    assert np.array_equal(sc.cpu().numpy(), s_ref)


@pytest.mark.parametrize("B,H,L", [(1, 2, 1000), (2, 3, 257), (1, 1, 1), (1, 1, 4680)])
def test_quantize_channels_bit_exact(h, orc, B, H, L):
    x = _x(B, H, L, seed=L, scale=0.5)
    x8, sc = h.fp8_quantize_channels(dev(x))
    torch.cuda.synchronize()
    c_ref, s_ref = orc.fp8_quantize_channels(x)
    assert np.array_equal(x8.cpu().numpy(), c_ref)
    assert np.array_equal(sc.cpu().numpy(), s_ref)


def test_quantize_zero_blocks(h, orc):
    x = torch.zeros((1, 1, 200, 128), dtype=torch.bfloat16)
    x[0, 0, 100:] = _x(1, 1, 100, seed=4)[0, 0]
    x8, sc = h.fp8_quantize_rows(dev(x), 200, 64)
    v8, vs = h.fp8_quantize_channels(dev(torch.zeros((1, 1, 50, 128), dtype=torch.bfloat16)))
    torch.cuda.synchronize()
    c_ref, s_ref = orc.fp8_quantize_rows(x, 200, 64)
    assert np.array_equal(x8.cpu().numpy(), c_ref) and np.array_equal(sc.cpu().numpy(), s_ref)
    assert s_ref[0, 0, 0, 0] == 0
    assert int(v8.sum()) == 0 and float(vs.abs().sum()) == 0


def _check_fp8_attention(h, orc, x, T, N, w, r, rows=None):
    """Quantise on the CPU (oracle), run the kernel on those codes, compare with the oracle's
    attention of the dequantised codes within the per-element bound. Returns (err, bound)."""
    L = T * N
    q8, qs = orc.fp8_quantize_rows(x["q"], L, 128)
    k8, ks = orc.fp8_quantize_rows(x["k"], N, 64)
    v8, vs = orc.fp8_quantize_channels(x["v"])
    t = lambda a: dev(torch.from_numpy(np.ascontiguousarray(a)))
    o = h.window_fp8(t(q8), t(qs), t(k8), t(ks), t(v8), t(vs), T, N, w, r,
                     out=poison_like(torch.empty(x["q"].shape, dtype=torch.bfloat16, device="cuda")))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    B, H = x["q"].shape[:2]
    flat = None
    if rows is not None:
        flat = (np.arange(B * H)[:, None] * L + rows[None, :]).reshape(-1)
    ref = orc.window_fp8(q8, qs, k8, ks, v8, vs, T, N, w, r, rows=flat)
    ref_abs = orc.window_fp8(q8, qs, k8, ks, v8 & 0x7F, vs, T, N, w, r, rows=flat)
    got = o.float().cpu().numpy().astype(np.float64).reshape(-1, 128)
    if flat is not None:
        got = got[flat]
    ref = ref.reshape(-1, 128)
    ref_abs = ref_abs.reshape(-1, 128)
    err = np.abs(got - ref)
    bound = 2.0 ** -4 * ref_abs + 2.0 ** -8 * np.abs(ref) + 1e-5
    return err, bound, o


@pytest.mark.parametrize("B,H,T,N,w,r", [
    (1, 1, 4, 256, 2, 1),       # frames aligned to 128-row tiles
    (2, 3, 5, 200, 3, 1),       # tiles straddle frames, ragged key tiles
    (1, 2, 3, 40, 2, 1),        # several frames per query tile
    (1, 1, 6, 1, 3, 1),         # one token per frame
    (1, 1, 2, 300, 5, 1),       # window longer than the clip
    (1, 2, 9, 150, 3, 3),       # dilated
    (1, 1, 13, 97, 3, 4),       # dilated, taps before frame 0 dropped
])
def test_window_fp8_within_quantisation_bound(h, orc, B, H, T, N, w, r):
    x = _inputs(B, H, T, N, seed=31 + T * N)
    err, bound, o = _check_fp8_attention(h, orc, x, T, N, w, r)
    assert torch.isfinite(o).all()
    assert np.all(err <= bound), float((err / bound).max())


def test_window_fp8_end_to_end_against_bf16_attention(h, orc):
    """GPU quantisation plus FP8 attention against the attention of the unquantised bf16
    inputs. No bound follows from the format alone here (the score error depends on |q||k|),
    so the tolerance is a measured one with a margin: on a B200 this case gave max 0.054 and
    rms 0.0037 (output rms 0.069); the test allows 0.08 and 0.006."""
    B, H, T, N, w = 1, 2, 4, 300, 3
    x = _inputs(B, H, T, N, seed=5)
    q, k, v = (dev(x[n]) for n in "qkv")
    o = h.window_fp8(*h.fp8_quantize_window_inputs(q, k, v, T, N), T, N, w)
    torch.cuda.synchronize()
    ref = orc.swa(x["q"], x["k"], x["v"], T, N, w)
    err = np.abs(o.float().cpu().numpy() - ref)
    rms = float(np.sqrt((err ** 2).mean()))
    assert float(err.max()) <= 8e-2 and rms <= 6e-3, (float(err.max()), rms)


def test_480p_fp8_sampled(h, orc):
    """The 480P workload's eight SWA heads (w=3) and eight DSWA heads (w=3, r=4) in E4M3:
    GPU quantisation bit-exact with the oracle's on the whole tensors, attention within the
    bound on sampled rows of every head."""
    wl = hi.WORKLOADS["480p"]
    x = hi.make_inputs(wl, seed=0)
    rows = hi.sample_rows(wl.L, wl.N, 128, seed=2).numpy()
    for h0, nh, w, r in ((0, wl.Hs, wl.w_swa, 1), (wl.Hs, wl.Hd, wl.w_dswa, wl.r)):
        xs = {n: x[n][:, h0:h0 + nh].contiguous() for n in "qkv"}
        q, k, v = (dev(xs[n]) for n in "qkv")
        q8, qs, k8, ks, v8, vs = h.fp8_quantize_window_inputs(q, k, v, wl.T, wl.N)
        torch.cuda.synchronize()
        rk8, rks = orc.fp8_quantize_rows(xs["k"], wl.N, 64)
        assert np.array_equal(k8.cpu().numpy(), rk8) and np.array_equal(ks.cpu().numpy(), rks)
        rv8, rvs = orc.fp8_quantize_channels(xs["v"])
        assert np.array_equal(v8.cpu().numpy(), rv8) and np.array_equal(vs.cpu().numpy(), rvs)
        err, bound, o = _check_fp8_attention(h, orc, xs, wl.T, wl.N, w, r, rows=rows)
        assert torch.isfinite(o).all()
        assert np.all(err <= bound), float((err / bound).max())
