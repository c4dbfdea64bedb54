"""The bench's multi-rank host logic on two gloo ranks (CPU): every rank gets
its own tokens against the same weights, and step times reduce to the
slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        wl = bench.rank_workload(rank)
        x0 = float(wl["x"][:4, :4].float().sum())
        w0 = float(wl["w1"][:4, :4].float().sum())
        out.put((rank, ms, x0, w0))
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_weights_shard_tokens_and_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, ms, x0, w0 = q.get(timeout=240)
        res[r] = (ms, x0, w0)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 15.0          # the slowest rank's time
    assert res[0][2] == res[1][2]                  # same weights
    assert res[0][1] != res[1][1]                  # different tokens


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
