"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
replica; the job time is the max over ranks and the whole-job value counts
every rank's units over that time.  No data-path collective exists."""
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
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    my_ms = [12.5, 20.0][rank]
    mx = bench.max_over_ranks(my_ms, world, device="cpu")
    val = bench.job_throughput(1000.0, world, mx)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, val))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]
    assert all(abs(r[2] - 2 * 1000.0 / 0.020) < 1e-6 for r in res)
