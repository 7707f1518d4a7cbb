"""Host logic of the multi-GPU bench on the CPU: two gloo ranks.

Replicas shard the job with no data-path collective: each rank generates its own
sequence (start token seeded by its rank), and the only exchange is the max over
ranks of the measured times, outside the timed region.  The whole-job value is
all ranks' tokens over the slowest rank's time.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from long_convolution_sequence_b200 import synth
    try:
        got = bench.max_over_ranks(times[rank], world, "cpu")
        x0 = synth.start_token(1, 8, seed=bench.rank_seed(rank))
        q.put((rank, got, x0))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_distinct_sequences():
    world = 2
    times = [12.5, 20.25]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, x0 = q.get(timeout=120)
        res[rank] = (got, x0)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == max(times)
    assert not np.array_equal(res[0][1], res[1][1])   # independent start tokens


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    # weak scaling: N replicas of B*L tokens over the slowest rank's milliseconds
    assert bench.job_tokens_per_s(4, 1, 1 << 17, 500.0) == 4 * (1 << 17) / 0.5
