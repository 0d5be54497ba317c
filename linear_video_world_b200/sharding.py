"""Sharding the operator over the GPUs of one node: one process per GPU (torch.distributed),
each owning a share of independent units, with outputs gathered only when asked.

The operator has no exchange step between its units: the rollouts of a streaming cache evolve
independently (zhichai.net blog, section 2.3: streaming tokens), and so do the heads of the
hybrid call (each head is one branch over its own q, k, v). The researchpapers.dev summary of
Kairos reports a 480P rollout on four A800s (its results list, inference latency) without
describing the split. So a node shards them with no collective on the data
path: every rank runs the library's kernels on its own slice, on its own GPU, from its own
memory (no peer memory is ever an operand). When the caller wants every output on every rank,
one all_gather (NCCL over NVLink on GPUs; gloo in the CPU tests) collects the local results,
padded to the largest share so that every rank sends the same size.

* ``RolloutShardedStream``: rank r holds rollouts [b0, b0 + Br) of a B-rollout streaming cache.
* ``HeadShardedHybrid``: rank r runs a contiguous share of each branch's heads (SWA, DSWA,
  GDN) of the hybrid operator; the full head order is restored when gathering.
"""
from __future__ import annotations


def split_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """(start, count) of rank's contiguous share of n units, the first n % world ranks one more."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad split: n={n} world={world} rank={rank}")
    base, rem = divmod(n, world)
    return rank * base + min(rank, rem), base + (1 if rank < rem else 0)


def head_plan(Hs: int, Hd: int, Hg: int, world: int):
    """Per rank ((s0, ns), (d0, nd), (g0, ng)): its share of the SWA, DSWA and GDN heads."""
    return [tuple(split_range(n, world, r) for n in (Hs, Hd, Hg)) for r in range(world)]


def global_heads(plan_r, Hs: int, Hd: int) -> list[int]:
    """Global head indices (SWA | DSWA | GDN order) of one rank's local heads, in local order."""
    (s0, ns), (d0, nd), (g0, ng) = plan_r
    return (list(range(s0, s0 + ns)) + [Hs + i for i in range(d0, d0 + nd)] +
            [Hs + Hd + i for i in range(g0, g0 + ng)])


def assemble_heads(parts, plan, Hs: int, Hd: int):
    """Rank-ordered local outputs [B, H_r, ...] -> the full [B, H, ...] in global head order."""
    import torch
    order = [h for pr in plan for h in global_heads(pr, Hs, Hd)]
    cat = torch.cat(list(parts), dim=1)
    out = torch.empty_like(cat)
    out[:, torch.tensor(order, device=cat.device)] = cat
    return out


def all_gather_dim(local, dim: int, counts, group=None):
    """All-gather tensors that differ only in their size along `dim` (rank r's size counts[r]),
    padded to the largest so every rank sends the same bytes; returns the rank-ordered parts."""
    import torch
    import torch.distributed as dist
    mx = max(counts)
    shape = list(local.shape)
    shape[dim] = mx
    buf = local.new_zeros(shape)
    buf.narrow(dim, 0, local.shape[dim]).copy_(local)
    parts = [torch.empty_like(buf) for _ in counts]
    dist.all_gather(parts, buf, group=group)
    return [p.narrow(dim, 0, c) for p, c in zip(parts, counts)]


def _world(group):
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


class RolloutShardedStream:
    """A B-rollout streaming cache split over the ranks: this rank holds rollouts
    [b0, b0 + Br) (``self.b0``, ``self.Br``) in a local ``Stream``. ``step`` takes this rank's
    inputs ([Br, H, N, d], gates [Br, Hg, N]) and returns its outputs, or with ``gather`` the
    outputs of all B rollouts on every rank."""

    def __init__(self, B, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk=64, scale=0.0,
                 max_step_frames=1, group=None):
        import linear_video_world_b200 as h
        self.group = group
        self.world, self.rank = _world(group)
        self.B, self.H, self.Hg, self.N, self.d = B, Hs + Hd + Hg, Hg, N, d
        self.counts = [split_range(B, self.world, q)[1] for q in range(self.world)]
        self.b0, self.Br = split_range(B, self.world, self.rank)
        self.stream = (h.Stream(self.Br, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk, scale,
                                max_step_frames=max_step_frames) if self.Br else None)

    def step_frames(self, q, k, v, a, b, frames, gather=False, out=None):
        import torch
        if self.stream is not None:
            o = self.stream.step_frames(q, k, v, a, b, frames, out=out)
        else:
            o = torch.empty((0, self.H, frames * self.N, self.d), dtype=q.dtype, device=q.device)
        if not gather or self.world == 1:
            return o
        return torch.cat(all_gather_dim(o, 0, self.counts, self.group), dim=0)

    def step(self, q, k, v, a, b, gather=False, out=None):
        return self.step_frames(q, k, v, a, b, 1, gather=gather, out=out)

    def state(self, gather=False, device="cuda"):
        """The carried GDN state [Br, Hg, d, d] of this rank (or [B, Hg, d, d] gathered)."""
        import torch
        S = (self.stream.state_tensor() if self.stream is not None else
             torch.empty((0, self.Hg, self.d, self.d), device=device))
        if not gather or self.world == 1:
            return S
        return torch.cat(all_gather_dim(S, 0, self.counts, self.group), dim=0)

    def close(self):
        if self.stream is not None:
            self.stream.close()


class HeadShardedHybrid:
    """The hybrid operator with its heads split over the ranks: this rank runs heads
    ``self.heads`` (global indices, SWA | DSWA | GDN order), a contiguous share of each branch.
    ``local(t)`` cuts a full [B, H, ...] tensor (or gates [B, Hg, ...]) down to this rank's
    heads; ``forward`` takes this rank's q, k, v [B, H_r, L, d] and gates [B, Hg_r, L] and
    returns (o [B, H_r, L, d], S [B, Hg_r, d, d]), or with ``gather`` the full o [B, H, L, d]
    and S [B, Hg, d, d] on every rank."""

    def __init__(self, Hs, Hd, Hg, T, N, w_swa, w_dswa, r, chunk=64, scale=0.0, group=None):
        self.group = group
        self.world, self.rank = _world(group)
        self.Hs, self.Hd, self.Hg, self.T, self.N = Hs, Hd, Hg, T, N
        self.w_swa, self.w_dswa, self.r, self.chunk, self.scale = w_swa, w_dswa, r, chunk, scale
        self.plan = head_plan(Hs, Hd, Hg, self.world)
        (self.s0, self.ns), (self.d0, self.nd), (self.g0, self.ng) = self.plan[self.rank]
        self.heads = global_heads(self.plan[self.rank], Hs, Hd)

    def local(self, t, gates=False):
        """This rank's heads of a full tensor (a contiguous copy)."""
        import torch
        idx = (list(range(self.g0, self.g0 + self.ng)) if gates else self.heads)
        return t.index_select(1, torch.tensor(idx, device=t.device)).contiguous()

    def forward(self, q, k, v, a, b, S0=None, gather=False):
        import torch
        import linear_video_world_b200 as h
        if len(self.heads):
            o, S = h.hybrid(q, k, v, a, b, self.ns, self.nd, self.ng, self.T, self.N,
                            self.w_swa, self.w_dswa, self.r, S0=S0, chunk=self.chunk,
                            scale=self.scale)
        else:
            o = torch.empty_like(q)
            S = None
        B, d = q.shape[0], q.shape[3]
        if S is None:
            S = torch.zeros((B, self.ng, d, d), dtype=torch.float32, device=q.device)
        if not gather or self.world == 1:
            return o, S
        hcounts = [len(global_heads(pr, self.Hs, self.Hd)) for pr in self.plan]
        o_full = assemble_heads(all_gather_dim(o, 1, hcounts, self.group), self.plan, self.Hs, self.Hd)
        gcounts = [pr[2][1] for pr in self.plan]
        S_full = torch.cat(all_gather_dim(S, 1, gcounts, self.group), dim=1)
        return o_full, S_full
