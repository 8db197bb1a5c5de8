"""The multi-rank logic of bench.py on CPU ranks (gloo, world size 2): the max-over-ranks
timing, independent layers per rank, the weak-scaling value."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    t = bench.max_over_ranks(0.25 * (rank + 1), world)
    q.put((rank, t, bench.rank_seed(rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_layers():
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
    assert [t for _, t, _ in out] == [0.5, 0.5]          # every rank sees the slowest rank
    assert len({s for _, _, s in out}) == 2              # different layers per rank


def test_weak_scaling_value():
    import bench
    assert bench.weak_scaling_value(1, 4096 * 4096, 0.01) == pytest.approx(4096 * 4096 / 0.01)
    assert bench.weak_scaling_value(8, 4096 * 4096, 0.02) == pytest.approx(8 * 4096 * 4096 / 0.02)
