"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Sequences are independent, so ranks share nothing on the data path; what must agree across ranks
is the timing (maximum over ranks) and the per-rank inputs (distinct seeds)."""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        w = bench.rank_workload("mlra4_n8_l32k", rank)
        v = bench.weak_scaling_value(w.batch, world, t)
        q.put((rank, t, w.seed, v))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_draw_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, t0, s0, v0), (r1, t1, s1, v1) = res
    assert t0 == t1 == 15.0            # both ranks report the slower rank's time
    assert s0 != s1                    # distinct inputs per rank
    assert v0 == v1 == pytest.approx(2 * 8 / 15e-3)  # both batches over the max time
