"""GPU parity of the gated delta rule's backward pass (chunk form, fp32 arithmetic) against
the CPU oracle's reverse-mode derivative of the token recurrence (fp64).

Tolerances, relative to the largest reference gradient when that exceeds 1: fp32 inputs 1e-4,
as the fp32 forward; bf16 inputs and gradients 2e-2, as every bf16 output (the gradients are
rounded to bf16 once, the arithmetic is fp32)."""
import numpy as np
import pytest
import torch

import hlta_inputs as hi
from gpu_util import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    import linear_video_world_b200 as h
    assert torch.cuda.is_available()
    return h


def _case(B, H, L, decay, dtype, seed):
    wl = hi.Workload("t", B=B, Hs=0, Hd=0, Hg=H, d=128, T=L, N=1, w_swa=1, w_dswa=1, r=1,
                     chunk=64, dtype=dtype, decay=decay)
    x = hi.make_inputs(wl, seed=seed)
    g = torch.Generator().manual_seed(seed + 50)
    dO = torch.randn(x["q"].shape, generator=g)
    x["dO"] = dO.to(x["q"].dtype).contiguous()
    x["S0"] = hi.random_state(B, H, 128, seed=seed + 60, scale=0.1)
    x["dSL"] = hi.random_state(B, H, 128, seed=seed + 70, scale=0.1)
    return x


def _rel(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    return float(np.abs(g - ref).max()) / max(1.0, float(np.abs(ref).max()))


@pytest.mark.parametrize("B,H,L,decay,dtype,tol,states", [
    (1, 2, 150, 1.0, "fp32", 1e-4, True),     # ragged last chunk
    (1, 1, 64, 1.0, "fp32", 1e-4, False),     # one full chunk, zero S0 and dS_final
    (1, 1, 1, 1.0, "fp32", 1e-4, True),       # one token
    (2, 1, 700, 0.05, "fp32", 1e-4, True),    # slow decay: long memory
    (1, 2, 150, 1.0, "bf16", 2e-2, True),
    (2, 2, 1000, 0.05, "bf16", 2e-2, True),
    (1, 1, 1, 1.0, "bf16", 2e-2, True),       # one token
    (1, 1, 64, 1.0, "bf16", 2e-2, False),     # one full chunk, zero S0 and dS_final
    (1, 1, 2000, 0.05, "bf16", 2e-2, True),   # 32 chunks: the state passes' rings wrap
    (1, 1, 8360, 0.05, "bf16", 2e-2, True),   # 131 chunks (ragged tail), slow decay
    (1, 2, 8320, 1.0, "bf16", 2e-2, True),    # 130 full chunks per head
])
def test_gdn_bwd(h, orc, B, H, L, decay, dtype, tol, states):
    x = _case(B, H, L, decay, dtype, seed=L + 3)
    S0 = x["S0"] if states else None
    dSL = x["dSL"] if states else None
    got = h.gdn_bwd(*(dev(x[n]) for n in ("q", "k", "v", "a", "b", "dO")),
                    S0=None if S0 is None else dev(S0), dS_final=None if dSL is None else dev(dSL))
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0
    ref = orc.gdn_bwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["dO"],
                      S0=None if S0 is None else S0.double().numpy(),
                      dS_final=None if dSL is None else dSL.double().numpy())
    names = ("dq", "dk", "dv", "da", "db", "dS0")
    errs = {n: _rel(g_, r_) for n, g_, r_ in zip(names, got, ref)}
    assert all(e <= tol for e in errs.values()), errs
