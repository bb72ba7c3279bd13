"""Host-side logic of the multi-GPU bench on CPU: two gloo ranks.

The operator shards by rows (rows are independent): each rank owns a
contiguous block of rows and no collective touches the data; the only
collective is the max-over-ranks reduction of the timing."""
import os
import socket

import pytest

import bench

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, rows, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = bench.shard_rows(rows, world, rank)
        mine = torch.zeros(rows, dtype=torch.int64)
        mine[lo:hi] = 1
        dist.all_reduce(mine)  # test-only check that the shards tile the rows
        slowest = bench.max_over_ranks(10.0 + rank * 5.5, dist, torch.device("cpu"))
        out.put((rank, mine.tolist(), slowest))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("rows", [1, 5, 2048])
def test_two_rank_sharding_and_max_time(rows):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rows, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, cover, slowest in res:
        assert cover == [1] * rows  # every row owned by exactly one rank
        assert slowest == 15.5


def test_shard_rows_single():
    assert bench.shard_rows(7, 1, 0) == (0, 7)
    assert [bench.shard_rows(7, 3, r) for r in range(3)] == [(0, 3), (3, 5), (5, 7)]
