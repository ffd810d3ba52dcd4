"""The multi-rank path of bench.py on CPU with two gloo ranks: each rank
draws its own batch (weak scaling, no data-path collective), the step time is
the maximum over ranks, and the job's value aggregates every rank's
positions.  No GPU is touched."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        t_max = bench.max_over_ranks(local_ms, "cpu")
        w = bench.make_rank_workload(1, rank)
        value = bench.aggregate_value(world, w.positions, 100, t_max)
        q.put((rank, t_max, value, int(w.tokens.sum()), float(w.uniforms.sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_aggregate_positions():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, v0, tok0, u0), (r1, t1, v1, tok1, u1) = res
    assert t0 == t1 == 15.0                        # max over ranks
    assert v0 == v1 == 2 * 16 * 100 / 0.015         # 2 ranks x 16 positions (B=4, k=4) x 100 steps
    assert (tok0, u0) != (tok1, u1)                 # each rank verifies its own batch


def test_single_process_helpers():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_seed(2, 0) != bench.rank_seed(2, 1)
    assert np.isclose(bench.aggregate_value(1, 512, 10, 1.0), 512 * 10 / 1e-3)
