"""Sharding over several GPUs (linear_video_world_b200/sharding.py), on CPU: the partition of
rollouts and heads, and the gather that restores the full outputs, run as gloo process groups
of 2 and 3 ranks (uneven shares). The kernels themselves run only on GPUs; here every rank
holds synthetic local outputs whose values name the global unit they belong to."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_split_range_covers_every_unit_once_balanced():
    from linear_video_world_b200.sharding import split_range
    for n in (0, 1, 5, 8, 24, 25):
        for world in (1, 2, 3, 4, 8):
            parts = [split_range(n, world, r) for r in range(world)]
            units = [i for s, c in parts for i in range(s, s + c)]
            assert units == list(range(n))
            assert max(c for _, c in parts) - min(c for _, c in parts) <= 1
    with pytest.raises(ValueError):
        split_range(4, 2, 2)


def test_head_plan_partitions_each_branch():
    from linear_video_world_b200.sharding import global_heads, head_plan
    for (Hs, Hd, Hg) in ((8, 8, 8), (1, 2, 3), (0, 5, 1), (3, 0, 0)):
        for world in (1, 2, 3, 8):
            plan = head_plan(Hs, Hd, Hg, world)
            heads = sorted(h for pr in plan for h in global_heads(pr, Hs, Hd))
            assert heads == list(range(Hs + Hd + Hg))
            for pr in plan:           # each rank's share of a branch is contiguous
                g = global_heads(pr, Hs, Hd)
                assert g == sorted(g)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from linear_video_world_b200.sharding import (all_gather_dim, assemble_heads, global_heads,
                                                  head_plan, split_range)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    res = {}
    # heads: local outputs [B, H_r, L, d] whose values are the global head index
    Hs, Hd, Hg, B = 3, 2, 4, 2
    plan = head_plan(Hs, Hd, Hg, world)
    mine = global_heads(plan[rank], Hs, Hd)
    o = torch.tensor(mine, dtype=torch.float32).view(1, -1, 1, 1).expand(B, len(mine), 5, 4).contiguous()
    counts = [len(global_heads(pr, Hs, Hd)) for pr in plan]
    full = assemble_heads(all_gather_dim(o, 1, counts), plan, Hs, Hd)
    res["heads"] = bool(torch.equal(full, torch.arange(Hs + Hd + Hg, dtype=torch.float32).view(1, -1, 1, 1).expand(B, -1, 5, 4)))
    # the GDN states: contiguous shares, gathered in rank order
    g0, ng = plan[rank][2]
    S = torch.arange(g0, g0 + ng, dtype=torch.float32).view(1, -1, 1, 1).expand(B, ng, 3, 3).contiguous()
    Sf = torch.cat(all_gather_dim(S, 1, [pr[2][1] for pr in plan]), dim=1)
    res["states"] = bool(torch.equal(Sf, torch.arange(Hg, dtype=torch.float32).view(1, -1, 1, 1).expand(B, -1, 3, 3)))
    # rollouts: local [Br, ...] with the global rollout index
    Bt = 5
    b0, Br = split_range(Bt, world, rank)
    x = torch.arange(b0, b0 + Br, dtype=torch.float32).view(-1, 1, 1).expand(Br, 3, 2).contiguous()
    xf = torch.cat(all_gather_dim(x, 0, [split_range(Bt, world, r)[1] for r in range(world)]), dim=0)
    res["rollouts"] = bool(torch.equal(xf, torch.arange(Bt, dtype=torch.float32).view(-1, 1, 1).expand(Bt, 3, 2)))
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, res))


@pytest.mark.parametrize("world", [2, 3])
def test_gather_restores_global_order_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r in res:
        assert r == {"heads": True, "states": True, "rollouts": True}, (rank, r)
