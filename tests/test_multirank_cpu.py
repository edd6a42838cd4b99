"""The benchmark's multi-rank logic on CPU with two gloo ranks: every rank processes its own
clip (no data-path collective), and the job's time is the slowest rank's."""
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


def _rank(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    ms_local = 10.0 * (rank + 1)  # rank 1 is the slow one
    value, ms = bench.job_throughput(1000, ms_local, world, device="cpu")
    # a decision one rank takes (e.g. "skip the end-to-end leg", "device error") reaches all
    flag = bench.max_over_ranks(1.0 if rank == 1 else 0.0, world, device="cpu")
    q.put((rank, value, ms, flag))
    dist.barrier()
    dist.destroy_process_group()


def test_job_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms, flag in res:
        assert ms == pytest.approx(20.0)                    # the slowest rank's time
        assert value == pytest.approx(2 * 1000 / 20e-3)     # units of all ranks / that time
        assert flag == 1.0                                  # every rank sees rank 1's decision


def test_single_rank_needs_no_collective():
    import bench
    value, ms = bench.job_throughput(500, 5.0, 1)
    assert ms == 5.0 and value == pytest.approx(500 / 5e-3)
