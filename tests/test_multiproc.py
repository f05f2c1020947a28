"""Host-side logic of the multi-GPU benchmark (replicas, no data-path
collective), run as two gloo ranks on the CPU: the step time is the max over
ranks and every rank takes the same collective steps."""
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


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        mx = bench.aggregate_over_ranks(local_ms, "max")
        total = bench.aggregate_over_ranks(1.0, "sum")
        q.put((rank, ws, r, local, mx, total))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, ws, r, local, mx, total in out:
        assert ws == 2 and r == rank and local == rank
        assert mx == 15.0          # max over ranks, seen by every rank
        assert total == 2.0


def test_single_process_aggregate_is_identity():
    import bench
    assert bench.aggregate_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_exit_without_work(capsys, monkeypatch):
    """Under torchrun the reference arm (the CPU oracle) runs on rank 0 only:
    every other rank returns 0 at once and prints nothing, without loading the
    oracle."""
    import argparse
    import sys

    import bench
    monkeypatch.delitem(sys.modules, "oracle", raising=False)
    args = argparse.Namespace(config="c1_tiny_dualscale", steps=1, warmup=0, gpus=2)
    assert bench.main_reference(args, 2, 1) == 0
    assert capsys.readouterr().out == ""
    assert "oracle" not in sys.modules
