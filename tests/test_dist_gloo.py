"""Multi-rank host logic on CPU (gloo, world size 2): request partitioning and the
max-over-ranks timing reduction used by the bench. The decode path itself has no collective."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_recurrent_state_gated_b200 import dist as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as tdist
    info = D.init("gloo", timeout_s=30)
    assert (info.rank, info.world) == (rank, world)
    start, stop = D.partition(n, world, rank)
    shares = [None] * world
    tdist.all_gather_object(shares, (start, stop))
    mx = D.max_over_ranks(1.5 + rank)
    total = D.sum_over_ranks(stop - start)
    D.barrier()
    D.finalize()
    q.put((rank, shares, mx, total))


@pytest.mark.parametrize("n", [7, 64, 1])
def test_partition_and_reductions_two_ranks(n):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, n, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = [q.get(timeout=120) for _ in ps]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shares, mx, total in res:
        assert shares[0][0] == 0 and shares[-1][1] == n
        assert shares[0][1] == shares[1][0]
        assert mx == 2.5 and total == n


def test_partition_covers_exactly():
    for n in range(0, 40):
        for world in range(1, 9):
            parts = [D.partition(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for a, b in zip(parts, parts[1:]):
                assert a[1] == b[0]
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
