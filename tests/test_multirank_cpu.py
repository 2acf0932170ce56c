"""The N > 1 bench path on CPU: world size 2 over gloo.

The bifocal path shards into independent sequences, so the only collective is
the max-over-ranks reduction of each timing; the whole-job value is the units
of all ranks over the slowest rank's time (weak scaling).  Also checks that the
reference arm runs on rank 0 only.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world)       # rank 1 is the slow one
    v = bench.weak_scaling_value(1.0e12, world, t)
    out.put((rank, t, v))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in res:
        assert t == 15.0                                   # both ranks see the slowest time
        assert abs(v - 2 * 1.0e12 / 15.0e-3) < 1.0          # units of both ranks / max time


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, ref_rows = 1, 0, 1
    assert bench.run_reference(A()) is None
