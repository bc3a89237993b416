"""Multi-rank plumbing of bench.py on the CPU (gloo, world size 2): the timing
reduction is a max over ranks, and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        mx = bench.max_over_ranks(10.0 + 5 * rank, world)
        bench.barrier(world)

        class A:
            views = 2
            warmup = 0
            steps = 1
        res, r = bench.run_reference(A())
        q.put((rank, mx, res is None, r))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank0_reference_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[1] for o in out] == [15.0, 15.0]        # max over ranks on every rank
    assert out[0][2] is False and out[1][2] is True   # only rank 0 produces the reference line
