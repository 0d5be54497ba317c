"""GPU parity of the raw-input entry points (GDN prologue fused into the chunk preparation:
unit-norm q and k per token, a = exp(-c softplus(x)), b = sigmoid(y)) against the CPU oracle's
gdn_raw. Tolerances as for the other paths: 2e-2 max-abs for bf16, 1e-4 for fp32."""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev, maxabs, poison_like

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _gdn_wl(B, H, L, decay=1.0, dtype="bf16", d=128):
    return hi.Workload("t", B=B, Hs=0, Hd=0, Hg=H, d=d, T=L, N=1, w_swa=1, w_dswa=1, r=1,
                       chunk=64, dtype=dtype, decay=decay)


@pytest.mark.parametrize("B,H,L,c", [(1, 2, 150, 1.0), (1, 1, 1, 1.0), (2, 1, 1000, 0.05),
                                     (1, 1, 64, 0.0)])
def test_gdn_raw_bf16(h, orc, B, H, L, c):
    wl = _gdn_wl(B, H, L, c)
    x = hi.make_raw_inputs(wl, seed=L + 7)
    q, k, v, xx, yy = (dev(x[n]) for n in ("q", "k", "v", "x", "y"))
    S0 = hi.random_state(B, H, 128, seed=5, scale=0.1)
    o, S = h.gdn_raw(q, k, v, xx, yy, c, S0=dev(S0), out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    o_ref, S_ref = orc.gdn_raw(x["q"], x["k"], x["v"], x["x"], x["y"], c, S0.double().numpy())
    assert maxabs(o, o_ref) <= 2e-2
    assert maxabs(S, S_ref) <= 2e-2


def test_gdn_raw_fp32(h, orc):
    wl = _gdn_wl(1, 2, 200, 1.0, dtype="fp32", d=64)
    x = hi.make_raw_inputs(wl, seed=11)
    q, k, v, xx, yy = (dev(x[n]) for n in ("q", "k", "v", "x", "y"))
    o, S = h.gdn_raw(q, k, v, xx, yy, 1.0, out=poison_like(q))
    torch.cuda.synchronize()
    o_ref, S_ref = orc.gdn_raw(x["q"], x["k"], x["v"], x["x"], x["y"], 1.0)
    assert maxabs(o, o_ref) <= 1e-4
    assert maxabs(S, S_ref) <= 1e-4


def test_gdn_raw_zero_tokens_and_extreme_gates(h, orc):
    """Tokens with q = k = 0 (kept zero, no NaN) and gate inputs far in both tails."""
    wl = _gdn_wl(1, 1, 130)
    x = hi.make_raw_inputs(wl, seed=3)
    x["q"][0, 0, 5] = 0
    x["k"][0, 0, 5] = 0
    x["k"][0, 0, 70] = 0
    x["x"][0, 0, :10] = 60.0          # a ~ e^-60: the memory is wiped
    x["x"][0, 0, 10:20] = -60.0       # a ~ 1: no decay
    x["y"][0, 0, 20:30] = 60.0        # b ~ 1
    x["y"][0, 0, 30:40] = -60.0       # b ~ 0
    q, k, v, xx, yy = (dev(x[n]) for n in ("q", "k", "v", "x", "y"))
    o, S = h.gdn_raw(q, k, v, xx, yy, 1.0, out=poison_like(q))
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    o_ref, S_ref = orc.gdn_raw(x["q"], x["k"], x["v"], x["x"], x["y"], 1.0)
    assert maxabs(o, o_ref) <= 2e-2
    assert maxabs(S, S_ref) <= 2e-2


def test_gdn_raw_rejects_bad_decay_constant(h):
    wl = _gdn_wl(1, 1, 64)
    x = hi.make_raw_inputs(wl, seed=1)
    q, k, v, xx, yy = (dev(x[n]) for n in ("q", "k", "v", "x", "y"))
    for c in (-1.0, float("nan"), float("inf")):
        with pytest.raises(h.HltaError):
            h.gdn_raw(q, k, v, xx, yy, c)


def test_hybrid_raw_small_full(h, orc):
    wl = hi.Workload("t", B=1, Hs=2, Hd=2, Hg=2, d=128, T=5, N=200, w_swa=3, w_dswa=2, r=2,
                     chunk=64, dtype="bf16", decay=0.5)
    x = hi.make_raw_inputs(wl, seed=9)
    q, k, v, xx, yy = (dev(x[n]) for n in ("q", "k", "v", "x", "y"))
    o, S = h.hybrid_raw(q, k, v, xx, yy, wl.decay, wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa,
                        wl.w_dswa, wl.r, out=poison_like(q))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    o_ref, S_ref = orc.hybrid(x["q"], x["k"], x["v"], x["x"], x["y"], wl.Hs, wl.Hd, wl.Hg, wl.T,
                              wl.N, wl.w_swa, wl.w_dswa, wl.r, raw=wl.decay)
    assert maxabs(o, o_ref) <= 2e-2
    assert maxabs(S, S_ref) <= 2e-2


def test_hybrid_raw_matches_normalised_entry_point(h):
    """The fused prologue and the caller-side preprocessing of the workload recipe give the
    same result up to one extra bf16 rounding of q and k."""
    wl = hi.Workload("t", B=1, Hs=1, Hd=1, Hg=2, d=128, T=4, N=160, w_swa=2, w_dswa=2, r=2,
                     chunk=64, dtype="bf16", decay=1.0)
    raw = hi.make_raw_inputs(wl, seed=2)
    g0 = wl.Hs + wl.Hd
    qn, kn = raw["q"].float().clone(), raw["k"].float().clone()
    for t in (qn, kn):
        t[:, g0:] /= t[:, g0:].norm(dim=-1, keepdim=True).clamp_min(1e-12)
    a = torch.exp(-wl.decay * torch.nn.functional.softplus(raw["x"]))
    b = torch.sigmoid(raw["y"])
    o1, S1 = h.hybrid_raw(*(dev(raw[n]) for n in ("q", "k", "v", "x", "y")), wl.decay, wl.Hs,
                          wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    o2, S2 = h.hybrid(dev(qn.bfloat16()), dev(kn.bfloat16()), dev(raw["v"]), dev(a), dev(b),
                      wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N, wl.w_swa, wl.w_dswa, wl.r)
    torch.cuda.synchronize()
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2
    assert float((S1 - S2).abs().max()) <= 2e-2
