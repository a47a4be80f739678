"""The N-GPU bench path's host logic on CPU: two gloo ranks.

bench.py runs independent replicas (no collective on the data path); the
only cross-rank steps are the slowest-rank time and the launch total, which
these ranks exercise with the gloo backend."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from mixture_experts_routing_top_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = [12.5, 30.25][rank]            # rank 1 is the slow one
        launches = [100, 120][rank]
        t, n = bench.reduce_over_ranks(elapsed, launches, "cpu")
        q.put((rank, t, n, bench.throughput(world, 8192, 10, t)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_total_launches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, n, v in res:
        assert t == 30.25 and n == 220
        assert v == pytest.approx(2 * 8192 * 10 / 0.03025)


def test_single_process_reduction_is_identity():
    assert bench.reduce_over_ranks(7.0, 3, "cpu") == (7.0, 3)


def test_ranks_get_their_own_batch_and_share_the_model():
    w = W.TINY
    a, b = bench.rank_batch(w, 0), bench.rank_batch(w, 1)
    assert not np.array_equal(W.make_logits(a), W.make_logits(b))
    assert not np.array_equal(W.make_x(a), W.make_x(b))
    assert a.T == b.T and a.E == b.E
    # the model (weights) is generated from the workload, not the rank's batch
    assert np.array_equal(W.make_weights(w)[0], W.make_weights(w)[0])
