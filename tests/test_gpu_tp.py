"""Branch-parallel decode on one GPU: the B branch shards (``tp.BranchShardStep`` without the
all-reduce) run one after another on the same device and their shares are summed here; the sum
must match the oracle's B-branch decode followed by step 3 on the full arrays (the path's
tolerance).  The reduction across devices itself is covered by the gloo test on CPU."""
import pytest
import torch

import oracle
from latent_kv_cache_mlra_b200 import tp
from tests.gpu_helpers import assert_close, to_dev
from tests.test_gpu_parity import small_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,page_size", [(4, 0), (2, 0), (4, 64)])
def test_branch_shards_sum_to_the_full_step(B, page_size):
    inp = small_inputs(B=B, lens=[300, 1, 129, 700], heads=64, page_size=page_size, seed=41)
    w = inp.workload
    q, qr, c, kr, lens, pt = to_dev(inp)
    g = torch.Generator().manual_seed(42)
    w_uv = (torch.randn(w.heads, 128, w.d_latent, generator=g) / w.d_latent ** 0.5).to(torch.bfloat16)
    y = torch.zeros(len(inp.seq_lens), w.heads, 128, device="cuda")
    for b in range(B):
        step = tp.BranchShardStep(tp.shard_queries(q, b, B), qr, tp.shard_latent(c, b, B), kr, lens,
                                  pt, tp.shard_wuv(w_uv.cuda(), b, B), num_branches=B,
                                  softmax_scale=w.sigma, max_seq_len=inp.max_seq_len,
                                  page_size=page_size, reduce=False)
        y += step()
    torch.cuda.synchronize()
    o, _ = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, inp.page_table,
                         B, w.sigma, w.gamma, max_seq_len=inp.max_seq_len, page_size=page_size)
    assert_close(y, oracle.project(o, w_uv.float()), f"B={B} paged={page_size}")


def test_branch_bench_step_on_one_device_matches_the_oracle():
    """The step that ``bench.py --parallel branch`` times, on one device (all B branches there,
    no all-reduce): steps 2 and 3 against the oracle's decode followed by step 3."""
    import bench
    inp = small_inputs(B=4, lens=[513, 1, 129, 700], heads=64, page_size=64, seed=43)
    w = inp.workload
    step, w_uv, per_device = bench.branch_step(w, inp, torch.device("cuda", 0), world=1, rank=0)
    assert per_device == 4
    y = step()
    torch.cuda.synchronize()
    o, _ = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, inp.page_table,
                         4, w.sigma, w.gamma, max_seq_len=inp.max_seq_len, page_size=64)
    assert_close(y, oracle.project(o, w_uv.float()), "branch step, one device")
