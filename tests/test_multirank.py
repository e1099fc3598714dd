"""World-size-2 gloo check (CPU) of the benchmark's multi-rank timing rule:
every rank's device time is gathered, the slowest rank's time divides all
ranks' work (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [100.0, 125.0][rank]          # rank 1 is the slow one
    all_ms = bench.gather_floats(ms, world)
    value, ms_per_step = bench.aggregate(all_ms, [3.5e12 * 10] * world, 10)
    q.put((rank, all_ms, value, ms_per_step))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, all_ms, value, ms_per_step in res:
        assert all_ms == [100.0, 125.0]
        assert ms_per_step == 12.5
        assert value == pytest.approx(2 * 3.5e13 / 0.125)
