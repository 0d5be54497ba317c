"""The N > 1 path of the benchmark on CPU: world size 2 over gloo.

The operator shards into independent replicas (no exchange step between GPUs), so the only
multi-process logic is the bench's plumbing: barriers around the timed region, the max over
ranks of the device-timed duration, the whole-job value, per-rank seeding of the inputs, and
the reference arm running on rank 0 alone under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_worker(rank: int, world: int, port: int, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import hlta_inputs as hi
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    rep = bench.Replicas(world, torch.device("cpu"))
    rep.barrier()
    ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
    ms_max = rep.allmax(ms)
    value = rep.job_value(1000, ms_max)
    x = hi.make_inputs(hi.WORKLOADS["tiny_fp32"], seed=rank)
    rep.barrier()
    dist.destroy_process_group()
    out.put((rank, ms_max, value, float(x["q"].sum())))


def test_replicas_max_over_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_replica_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value, _ in res:
        assert ms_max == 15.0                   # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 1000 / 0.015)
    # replicas get their own inputs (seed = rank), reproducibly
    assert res[0][3] != res[1][3]
    sys.path.insert(0, ROOT)
    import hlta_inputs as hi
    assert float(hi.make_inputs(hi.WORKLOADS["tiny_fp32"], seed=1)["q"].sum()) == res[1][3]


def test_single_rank_plumbing_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    rep = bench.Replicas(1, torch.device("cpu"))
    rep.barrier()
    assert rep.allmax(3.25) == 3.25
    assert rep.job_value(500, 2.0) == pytest.approx(250000.0)


def test_reference_arm_runs_on_rank0_only_under_torchrun():
    """`bench.py --impl reference` launched as two ranks prints one line (rank 0)."""
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "tiny_fp32", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
