"""GPU parity of the rotary position embedding (hlta_rope) against the CPU oracle (fp64).

Tolerances: bf16 outputs are rounded once, so |got - ref| <= 2^-8 |ref| + 1e-6 covers the
half-ulp rounding (2^-9 relative) with room for the single-precision sine, cosine and
products; fp32 outputs within 1e-5 (values of order one; the angle is reduced in double
precision before a single-precision sine and cosine)."""
import numpy as np
import pytest
import torch

from gpu_util import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _close(got, ref, dtype):
    g = got.float().cpu().numpy().astype(np.float64)
    if dtype == torch.bfloat16:
        return bool(np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6))
    return float(np.abs(g - ref).max()) <= 1e-5


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("pos_mode", [0, 1])
def test_rope_head_range(h, orc, dtype, pos_mode):
    B, H, L, N, d = 2, 5, 300, 64, 128
    gen = torch.Generator().manual_seed(11 + pos_mode)
    q0 = torch.randn(B, H, L, d, generator=gen).to(dtype)
    k0 = torch.randn(B, H, L, d, generator=gen).to(dtype)
    q, k = dev(q0), dev(k0)
    h.rope(q, k, N, heads=(1, 3), base=10000.0, pos_mode=pos_mode)
    torch.cuda.synchronize()
    for got, src in ((q, q0), (k, k0)):
        ref = orc.rope(src[:, 1:4], N, base=10000.0, pos_mode=pos_mode)
        assert _close(got[:, 1:4], ref, dtype)
        assert torch.equal(got[:, 0].cpu(), src[:, 0]) and torch.equal(got[:, 4].cpu(), src[:, 4])


def test_rope_inverse_round_trip_and_small_d(h, orc):
    B, H, L, N, d = 1, 2, 77, 10, 6
    x0 = torch.randn(B, H, L, d, generator=torch.Generator().manual_seed(3))
    x = dev(x0)
    h.rope(x, None, N, base=50.0, pos_mode=0)
    torch.cuda.synchronize()
    assert _close(x, orc.rope(x0, N, base=50.0, pos_mode=0), torch.float32)
    h.rope(x, None, N, base=50.0, pos_mode=0, inverse=True)
    torch.cuda.synchronize()
    assert float((x.cpu() - x0).abs().max()) <= 1e-5


def test_rope_480p_softmax_heads(h, orc):
    """The 480P clip's 16 softmax heads (N = 1560, T = 21) rotated in place, q only: frames 0,
    9 and 20 of every rotated head against the oracle (the within-frame position restarts each
    frame), the GDN heads untouched; then the global-position mode on one head in full."""
    import hlta_inputs as hi
    wl = hi.WORKLOADS["480p"]
    x = hi.make_inputs(wl, seed=5)
    q0 = x["q"]
    q = dev(q0)
    Hsm = wl.Hs + wl.Hd
    h.rope(q, None, wl.N, heads=(0, Hsm), pos_mode=0)
    torch.cuda.synchronize()
    for f in (0, 9, 20):
        sl = slice(f * wl.N, (f + 1) * wl.N)
        ref = orc.rope(q0[:, :Hsm, sl], wl.N, pos_mode=0)
        assert _close(q[:, :Hsm, sl], ref, torch.bfloat16)
    assert torch.equal(q[:, Hsm:].cpu(), q0[:, Hsm:])
    one = dev(q0[:, :1].contiguous())
    h.rope(one, None, wl.N, pos_mode=1)
    torch.cuda.synchronize()
    assert _close(one, orc.rope(q0[:, :1], wl.N, pos_mode=1), torch.bfloat16)
