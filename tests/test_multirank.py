"""The multi-GPU path on the CPU: two gloo ranks.

The attention path shards into independent problems (each rank runs its own
batch; there is no exchange step), so what a multi-rank run adds is host
logic: each rank draws its own seeded batch, the per-rank time is reduced to
the slowest rank, and rank 0 alone reports.  These tests run that logic as
world_size-2 gloo process groups with the float64 oracle standing in for the
kernels, and check that the sharded results equal the results of running
each shard alone."""

import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    import oracle
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs, shrink
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = shrink(WORKLOADS["tiny_causal"], Tq=16, Tk=16)
        x = make_inputs(w, seed=bench.shard_seed(w, rank))
        out, stat, _ = oracle.attention_fwd(x["q"], x["k"], x["v"], w.scale,
                                            "entmax15", True)
        # the slowest rank's time wins
        ms = bench.max_over_ranks(10.0 + rank, dist, "cpu")
        # collect every shard on every rank (test only; the path never does)
        got = [None] * world
        dist.all_gather_object(got, (rank, out.tolist(), stat.tolist()))
        q.put((rank, ms, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_shards():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from alternative_normalizers_b200.workloads import WORKLOADS, make_inputs, shrink
    w = shrink(WORKLOADS["tiny_causal"], Tq=16, Tk=16)
    for rank, ms, got in res:
        assert ms == 11.0                      # max over ranks
        shards = {r: (np.array(o), np.array(s)) for r, o, s in got}
        assert set(shards) == {0, 1}
        for r in (0, 1):
            x = make_inputs(w, seed=bench.shard_seed(w, r))
            o, s, _ = oracle.attention_fwd(x["q"], x["k"], x["v"], w.scale,
                                           "entmax15", True)
            np.testing.assert_array_equal(shards[r][0], o)
            np.testing.assert_array_equal(shards[r][1], s)
        # the two ranks really hold different problems
        assert not np.array_equal(shards[0][0], shards[1][0])
