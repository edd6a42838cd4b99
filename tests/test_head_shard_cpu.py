"""The head-sharded split of one clip over ranks (host logic, CPU): the head ranges partition the
heads, and with gloo ranks each computing its own heads (the fp64 oracle stands in for the
per-rank library call, which needs a GPU) the all-gathered outputs and states equal the oracle on
the whole clip, in head order, also for ragged and empty ranges."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from frame_wise_gated_deltanet_b200.parallel import head_range


def test_head_ranges_partition_the_heads():
    for H in range(1, 41):
        for world in range(1, 10):
            ranges = [head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0  # contiguous, in rank order
            sizes = [b - a for a, b in ranges]
            assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)  # longer ranges first
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, H, q):
    import datetime
    import sys
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import gdn_inputs
    import oracle
    from frame_wise_gated_deltanet_b200.parallel import gather_heads, shard_heads
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, T, N, D = 2, 4, 9, 16
        x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=77, state_std=0.3)
        f = lambda t: t.float().numpy().astype(np.float64)
        ks = 0.05
        # this rank's heads, as a column-parallel projection would hand them over
        loc = {n: shard_heads(x[n], world, rank, 3) for n in ("q", "k", "v")}
        loc.update({n: shard_heads(x[n], world, rank, 2) for n in ("gamma", "beta")})
        loc["state"] = shard_heads(x["state"], world, rank, 1)
        if loc["q"].shape[3] > 0:
            o, s = oracle.gdn_frame_forward(f(loc["q"]), f(loc["k"]), f(loc["v"]),
                                            f(loc["gamma"]), f(loc["beta"]), f(loc["state"]), ks)
        else:
            o, s = np.zeros((B, T, N, 0, D)), np.zeros((B, 0, D, D))
        out = gather_heads(torch.from_numpy(o), H, 3)
        st = gather_heads(torch.from_numpy(s), H, 1)
        o_ref, s_ref = oracle.gdn_frame_forward(f(x["q"]), f(x["k"]), f(x["v"]), f(x["gamma"]),
                                                f(x["beta"]), f(x["state"]), ks)
        q.put((rank, bool(np.array_equal(out.numpy(), o_ref)),
               bool(np.array_equal(st.numpy(), s_ref)), tuple(out.shape)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,H", [(2, 5), (2, 4), (3, 2)], ids=["ragged", "even", "empty_rank"])
def test_gathered_head_shards_equal_the_whole_clip(world, H):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, H, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, out_ok, st_ok, shape in res:
        assert shape == (2, 4, 9, H, 16)
        assert out_ok and st_ok, f"rank {rank}: gathered output {out_ok}, state {st_ok}"
