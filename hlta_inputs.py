"""Seeded synthetic inputs for the hybrid linear temporal attention operator.

This module is shared by the CPU oracle (``oracle/``), the tests and ``bench.py``.
It draws random numbers and applies the input-side preprocessing that the operator
expects its caller to have done (unit-norm q/k on the gated-delta heads, gate
activations), and nothing else: none of the operator's own arithmetic lives here.

Workloads (Kairos, "Native Unified Architecture" / Hybrid Linear Temporal Attention;
shapes and distributions are the ones the operator is specified on):

* ``tiny_fp32``   B=1, heads 1/1/1, d=64, T=8 frames x N=16 tokens, SWA w=2, DSWA w=2 r=2, fp32
* ``480p``        B=1, heads 8/8/8, d=128, T=21 x N=1560 (30x52 latent grid), SWA w=3, DSWA w=3 r=4
* ``480p_long``   as 480p with T=61, DSWA w=4 r=6 and slow decay a=exp(-0.05*softplus(x))
* ``720p_long``   T=61 x N=3600 (45x80 grid), SWA w=3, DSWA w=4 r=6
* ``stream_480p`` B=8 rollouts, one new N=1560 frame per step, SWA w=3, DSWA w=4 r=6, 200 steps

Distributions: q, k, v ~ N(0, 1); on the gated-delta (GDN) heads q and k are L2-normalised
per token; gates a = exp(-c * softplus(x)), b = sigmoid(y) with x, y ~ N(0, 1) per token per
GDN head (c = 1, or 0.05 for the long-memory workload). Token l = f*N + n (frame-major).

Random numbers come from torch's CPU Philox-based generator, one independent stream per
tensor (seed, seed+1, ...), so the same seed gives the same inputs on every machine.
bf16 workloads are rounded once (round-to-nearest-even) after generation; both the oracle
and the CUDA path consume exactly these rounded values.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hs: int          # sliding-window heads
    Hd: int          # dilated sliding-window heads
    Hg: int          # gated-delta heads
    d: int
    T: int           # frames (for the streaming workload: frames in one full clip = steps)
    N: int           # tokens per frame
    w_swa: int
    w_dswa: int
    r: int
    chunk: int
    dtype: str       # "fp32" or "bf16"
    decay: float     # c in a = exp(-c * softplus(x))
    streaming: bool = False

    @property
    def H(self) -> int:
        return self.Hs + self.Hd + self.Hg

    @property
    def L(self) -> int:
        return self.T * self.N

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, Hs=1, Hd=1, Hg=1, d=64, T=8, N=16,
                          w_swa=2, w_dswa=2, r=2, chunk=64, dtype="fp32", decay=1.0),
    "480p": Workload("480p", B=1, Hs=8, Hd=8, Hg=8, d=128, T=21, N=1560,
                     w_swa=3, w_dswa=3, r=4, chunk=64, dtype="bf16", decay=1.0),
    "480p_long": Workload("480p_long", B=1, Hs=8, Hd=8, Hg=8, d=128, T=61, N=1560,
                          w_swa=3, w_dswa=4, r=6, chunk=64, dtype="bf16", decay=0.05),
    "720p_long": Workload("720p_long", B=1, Hs=8, Hd=8, Hg=8, d=128, T=61, N=3600,
                          w_swa=3, w_dswa=4, r=6, chunk=64, dtype="bf16", decay=1.0),
    "stream_480p": Workload("stream_480p", B=8, Hs=8, Hd=8, Hg=8, d=128, T=200, N=1560,
                            w_swa=3, w_dswa=4, r=6, chunk=64, dtype="bf16", decay=1.0,
                            streaming=True),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(shape, seed: int) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed), dtype=torch.float32)


def make_inputs(wl: Workload, seed: int = 0, frames: int | None = None) -> dict:
    """Return host tensors for one workload.

    q, k, v: [B, H, L, d] (fp32, or bf16 for bf16 workloads), heads ordered SWA | DSWA | GDN.
    a, b:    [B, Hg, L] fp32 gates of the GDN heads.
    ``frames`` overrides T (used to cut short clips of a workload for tests).
    """
    T = wl.T if frames is None else int(frames)
    L = T * wl.N
    shape = (wl.B, wl.H, L, wl.d)
    q = _randn(shape, seed)
    k = _randn(shape, seed + 1)
    v = _randn(shape, seed + 2)
    x = _randn((wl.B, wl.Hg, L), seed + 3)
    y = _randn((wl.B, wl.Hg, L), seed + 4)
    g0 = wl.Hs + wl.Hd
    if wl.Hg:
        for t in (q, k):
            sub = t[:, g0:]
            sub.div_(sub.norm(dim=-1, keepdim=True).clamp_min(1e-12))
    a = torch.exp(-wl.decay * torch.nn.functional.softplus(x))
    b = torch.sigmoid(y)
    if wl.dtype == "bf16":
        q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "a": a.contiguous(), "b": b.contiguous()}


def make_raw_inputs(wl: Workload, seed: int = 0, frames: int | None = None) -> dict:
    """Host tensors for the raw-input entry points (the GDN prologue done by the operator).

    q, k, v: [B, H, L, d] as in ``make_inputs`` before any preprocessing, except that the
    GDN heads' q and k carry a seeded per-token scale (log-normal, sigma 1) so their norms
    vary; x, y: [B, Hg, L] float32 raw gate inputs (the same draws ``make_inputs`` turns into
    a and b). bf16 workloads are rounded once after generation.
    """
    T = wl.T if frames is None else int(frames)
    L = T * wl.N
    shape = (wl.B, wl.H, L, wl.d)
    q = _randn(shape, seed)
    k = _randn(shape, seed + 1)
    v = _randn(shape, seed + 2)
    x = _randn((wl.B, wl.Hg, L), seed + 3)
    y = _randn((wl.B, wl.Hg, L), seed + 4)
    g0 = wl.Hs + wl.Hd
    if wl.Hg:
        sc = torch.exp(_randn((2, wl.B, wl.Hg, L, 1), seed + 5))
        q[:, g0:] *= sc[0]
        k[:, g0:] *= sc[1]
    if wl.dtype == "bf16":
        q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "x": x.contiguous(), "y": y.contiguous()}


def random_state(B: int, Hg: int, d: int, seed: int, scale: float = 1.0) -> torch.Tensor:
    """A seeded fp32 initial GDN state [B, Hg, d, d] (rows: value dim, cols: key dim)."""
    return (_randn((B, Hg, d, d), seed) * scale).contiguous()


def sample_rows(L: int, N: int, count: int, seed: int) -> torch.Tensor:
    """Seeded query-row sample: every frame's first and last row plus ``count`` random rows."""
    T = L // N
    firsts = torch.arange(T) * N
    lasts = firsts + (N - 1)
    rnd = torch.randint(0, L, (count,), generator=_gen(seed))
    return torch.unique(torch.cat([firsts, lasts, rnd])).to(torch.int64)
