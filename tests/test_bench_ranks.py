"""The multi-GPU bookkeeping of the benchmark on two CPU ranks (gloo): every
rank reports its own time, the job uses the slowest, the throughput counts
every rank's tokens, and each replica decodes its own tokens with the same
layer."""
import os
import socket
import sys

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                        # rank 1 is the slower one
        slowest = bench.max_over_ranks(ms, "cpu")
        rate = bench.whole_job_rate(1000 * 3, world, slowest)
        x0 = np.arange(12, dtype=np.float32).reshape(3, 4)
        xt = bench.rank_tokens(x0, rank)
        out[rank] = (slowest, rate, xt.copy(), bench.rank_env()[:2])
    finally:
        dist.destroy_process_group()


def test_two_ranks_slowest_time_and_whole_job_rate():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        slowest, rate, _, env = res[r]
        assert slowest == 15.0                       # max over ranks, the same on every rank
        assert abs(rate - 2 * 3000 / 0.015) < 1e-6   # both ranks' tokens over the slowest time
        assert env == (r, world)
    x_r0, x_r1 = res[0][2], res[1][2]
    assert np.array_equal(x_r0, np.arange(12, dtype=np.float32).reshape(3, 4))
    assert x_r1.shape == x_r0.shape and not np.array_equal(x_r1, x_r0)


def test_single_rank_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(100, 1, 50.0) == 2000.0
