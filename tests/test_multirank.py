"""Host-side logic of the multi-GPU bench path, on CPU with gloo ranks (world size 2).

Heads are independent, so ranks exchange nothing on the data path: each rank
runs its own batch, and the only collective is the max of the elapsed time.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        bench.dist_init(world, "gloo")
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        elapsed = 10.0 + 5.0 * rank                    # rank 1 is the slower one
        m = bench.max_over_ranks(elapsed, world)
        bench.barrier(world)
        value = bench.weak_scaling_value(1000, world, m / 1e3)
        q.put((rank, m, value))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, value in res:
        assert m == 15.0                                # max over ranks, the same on every rank
        assert abs(value - 2 * 1000 / 0.015) < 1e-6     # all ranks' tokens over the slowest time


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100, 1, 0.5) == 200.0
