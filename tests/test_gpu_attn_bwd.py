"""GPU parity of the windowed attention's training pair (forward with log-sum-exp, backward)
against the CPU oracle (fp64 log-sum-exp and reverse-mode gradients).

Tolerances: the log-sum-exp is an fp32 by-product of the bf16 forward (scores accumulated in
fp32 from bf16 inputs): 1e-3 absolute. The gradients are bf16 outputs of products whose
operands P and dS are rounded to bf16 (2^-9 relative) and whose D = dO.o uses the bf16 forward
output; they are checked like the other bf16 outputs, 2e-2 max-abs, relative to the largest
reference gradient when that exceeds 1.
"""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, poison_like

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _inputs(B, H, T, N, seed):
    wl = hi.Workload("t", B=B, Hs=0, Hd=H, Hg=0, d=128, T=T, N=N, w_swa=1, w_dswa=1, r=1,
                     chunk=64, dtype="bf16", decay=1.0)
    x = hi.make_inputs(wl, seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    x["dO"] = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16).contiguous()
    return x


def _err(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    return float(np.abs(g - ref).max()) / max(1.0, float(np.abs(ref).max()))


CASES = [
    (1, 1, 4, 256, 2, 1),       # frames aligned to 64-row tiles
    (2, 3, 5, 200, 3, 1),       # ragged tiles
    (1, 2, 3, 40, 2, 1),        # frames shorter than a tile
    (1, 1, 6, 1, 3, 1),         # one token per frame
    (1, 1, 2, 300, 5, 1),       # window longer than the clip
    (1, 2, 9, 150, 3, 3),       # dilated
    (1, 1, 13, 97, 3, 4),       # dilated, taps before frame 0 dropped
]


@pytest.mark.parametrize("B,H,T,N,w,r", CASES)
def test_window_training_pair(h, orc, B, H, T, N, w, r):
    x = _inputs(B, H, T, N, seed=7 + T * N)
    q, k, v, dO = (dev(x[n]) for n in ("q", "k", "v", "dO"))
    o, lse = h.window_fwd_lse(q, k, v, T, N, w, r, out=poison_like(q),
                              lse=torch.full(q.shape[:-1], float("nan"), device="cuda"))
    o_plain = h.dswa(q, k, v, T, N, w, r)
    dq, dk, dv = h.window_bwd(q, k, v, o, lse, dO, T, N, w, r,
                              grads=tuple(poison_like(q) for _ in range(3)))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    assert torch.equal(o, o_plain)                    # the same forward, plus the normaliser
    lse_ref = orc.window_lse(x["q"], x["k"], T, N, w, r)
    assert float(np.abs(lse.cpu().numpy() - lse_ref).max()) <= 1e-3
    rq, rk, rv = orc.window_bwd(x["q"], x["k"], x["v"], x["dO"], T, N, w, r)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert _err(got, ref) <= TOL


def test_window_training_pair_480p_frames(h, orc):
    """Six frames of the 480P frame size (N = 1560), two SWA heads (w = 3), every gradient."""
    B, H, T, N, w, r = 1, 2, 6, 1560, 3, 1
    x = _inputs(B, H, T, N, seed=3)
    q, k, v, dO = (dev(x[n]) for n in ("q", "k", "v", "dO"))
    o, lse = h.window_fwd_lse(q, k, v, T, N, w, r)
    dq, dk, dv = h.window_bwd(q, k, v, o, lse, dO, T, N, w, r)
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    rq, rk, rv = orc.window_bwd(x["q"], x["k"], x["v"], x["dO"], T, N, w, r)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert _err(got, ref) <= TOL
