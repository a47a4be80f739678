"""The N-GPU bench path's host logic on CPU: two gloo ranks.

bench.py runs independent replicas (no collective on the data path); the
cross-rank steps are the slowest-rank time, the launch total and, once after
the timed steps, the sum of the ranks' routing histograms (co-selection or
transition counts are sums over tokens, so the sum over token shards is the
whole job's histogram).  These ranks exercise them with the gloo backend."""
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


def _routing(T, E, k, seed):
    from oracle import oracle as O
    from mixture_experts_routing_top_b200 import synth

    idx1, _ = O.route_topk(synth.normal_f32(seed, 1, (T, E)), k)
    idx2, _ = O.route_topk(synth.normal_f32(seed, 2, (T, E)), 1)
    return idx1, idx2


def _hist_rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    from oracle import oracle as O
    from mixture_experts_routing_top_b200 import layer as Lyr

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, E, k = 600, 16, 3
        idx1, idx2 = _routing(T, E, k, 9)
        # even token shards through the bench's record (totals must agree)
        lo, hi = rank * T // world, (rank + 1) * T // world
        cos = torch.from_numpy(O.coselect(idx1[lo:hi], E))
        job_c, rec_c = bench.job_histogram("coselect", cos, world, torch.device("cpu"))
        # ragged shards (250 / 350 tokens) through the library call, transitions
        cut = [0, 250, T][rank:rank + 2]
        top1 = idx1[cut[0]:cut[1], :1]
        tr = Lyr.reduce_histogram(torch.from_numpy(O.transition(top1, idx2[cut[0]:cut[1]], E)))
        q.put((rank, job_c.numpy(), rec_c, cos.numpy(), tr.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_their_histograms_to_the_jobs():
    from oracle import oracle as O

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_hist_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted((q.get(timeout=10) for _ in range(2)), key=lambda r: r[0])
    T, E, k = 600, 16, 3
    idx1, idx2 = _routing(T, E, k, 9)
    full_c = O.coselect(idx1, E)
    full_t = O.transition(idx1[:, :1], idx2, E)
    for rank, job_c, rec, local_c, tr in res:
        assert np.array_equal(job_c, full_c) and np.array_equal(tr, full_t)
        assert rec["consistent"] and rec["total"] == T * k * k and rec["ranks"] == 2
        assert rec["collective"] == "all_reduce sum int32" and rec["bytes"] == E * E * 4
        assert not np.array_equal(local_c, full_c)                   # each rank saw only its shard
    assert np.array_equal(res[0][3] + res[1][3], full_c)


def test_one_rank_histogram_is_its_own():
    import torch

    cos = torch.arange(16, dtype=torch.int32).view(4, 4)
    job, rec = bench.job_histogram("coselect", cos, 1, torch.device("cpu"))
    assert torch.equal(job, cos) and rec["consistent"] and rec["allreduce_us"] == 0.0
    assert rec["collective"] == "none (one rank)"


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
