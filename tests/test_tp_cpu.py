"""Branch-parallel decode (the branches spread over devices, the sum over branches by an all-reduce
after step 3) on CPU: gloo ranks on 127.0.0.1 -- four ranks with one branch each, and two ranks
with two branches each (the layout of ``bench.py --parallel branch --gpus 2``).

Each rank takes its shard from ``bench.branch_layout``, cuts its blocks with the package's sharding
helpers and runs the package's ``BranchShardStep.__call__`` (local share, then the all-reduce); the
local share itself is the oracle's decode of the rank's branches and step 3 on the rank's blocks
(the CUDA kernels need a GPU).  The reduced result must equal the oracle's four-branch decode
followed by step 3 on the full arrays: that pins the column blocks, the per-branch independence of
the softmax, the branch scale and the reduction together."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

BRANCHES = 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    import workloads
    w = workloads.small(batch=3, heads=4, num_branches=BRANCHES, d_latent=64, d_rope=16, seq_len=40,
                        ragged=True, min_seq_len=1, seed=31)
    inp = workloads.make_inputs(w)
    g = torch.Generator().manual_seed(32)
    w_uv = (torch.randn(w.heads, 32, w.d_latent, generator=g) / w.d_latent ** 0.5).to(torch.bfloat16)
    return w, inp, w_uv


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from latent_kv_cache_mlra_b200 import tp

        w, inp, w_uv = _inputs()
        shard, shards, per_device = bench.branch_layout(BRANCHES, world, rank)

        class OracleShard(tp.BranchShardStep):
            """The rank's local share from the oracle (test only); reduction as in the package."""

            def __init__(self, q_lat_b, c_b, w_uv_b):
                self.group, self.reduce = None, True
                self.args = (q_lat_b, c_b, w_uv_b)

            def local(self):
                q_lat_b, c_b, w_uv_b = self.args
                o_b, _ = oracle.decode(q_lat_b, inp.q_rope, c_b, inp.k_rope, inp.seq_lens, None,
                                       per_device, w.sigma, 1.0 / BRANCHES,
                                       max_seq_len=inp.max_seq_len)
                return torch.from_numpy(oracle.project(o_b, w_uv_b.float()))

        step = OracleShard(tp.shard_queries(inp.q_lat, shard, shards),
                           tp.shard_latent(inp.c_kv, shard, shards), tp.shard_wuv(w_uv, shard, shards))
        y = step()
        q.put((rank, y.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [4, 2])
def test_branch_ranks_sum_to_the_full_decode_and_projection(world):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w, inp, w_uv = _inputs()
    o, _ = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None, BRANCHES,
                         w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    ref = oracle.project(o, w_uv.float())
    for r in range(world):  # every rank holds the same, full result
        np.testing.assert_allclose(got[r], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_branch_blocks():
    from latent_kv_cache_mlra_b200 import tp
    assert tp.branch_block(512, 3, 4) == slice(384, 512)
    c = torch.arange(2 * 8).view(2, 8)
    assert torch.equal(tp.shard_latent(c, 1, 4), c[:, 2:4])
    with pytest.raises(ValueError):
        tp.branch_block(510, 0, 4)
    with pytest.raises(ValueError):
        tp.branch_block(512, 4, 4)


def test_branch_layout():
    import bench
    assert bench.branch_layout(4, 1, 0) == (0, 1, 4)
    assert bench.branch_layout(4, 2, 1) == (1, 2, 2)
    assert bench.branch_layout(4, 4, 3) == (3, 4, 1)
    with pytest.raises(ValueError):
        bench.branch_layout(4, 3, 0)      # three devices cannot split four branches evenly
    with pytest.raises(ValueError):
        bench.branch_layout(4, 8, 0)      # more devices than branches
