"""Seeded input generation: determinism and layout invariants (host only)."""
import math

import torch

import workloads


def test_deterministic_and_shapes():
    w = workloads.small(batch=2, seq_len=100)
    a, b = workloads.make_inputs(w), workloads.make_inputs(w)
    for x, y in [(a.q_lat, b.q_lat), (a.c_kv, b.c_kv), (a.k_rope, b.k_rope), (a.q_rope, b.q_rope)]:
        assert torch.equal(x, y)
    assert a.q_lat.shape == (2, 64, 512) and a.q_rope.shape == (2, 64, 64)
    assert a.c_kv.shape == (200, 512) and a.k_rope.shape == (200, 64)
    assert a.c_kv.dtype == torch.bfloat16 and a.page_table is None


def test_paged_pool_is_a_permutation():
    w = workloads.small(batch=5, seq_len=1000, min_seq_len=10, ragged=True, page_size=64)
    inp = workloads.make_inputs(w)
    lens = inp.seq_lens.tolist()
    assert all(10 <= l <= 1000 for l in lens)
    used = []
    for s, l in enumerate(lens):
        n = (l + 63) // 64
        row = inp.page_table[s].tolist()
        assert all(p >= 0 for p in row[:n]) and all(p == -1 for p in row[n:])
        used += row[:n]
    assert len(set(used)) == len(used)
    assert max(used) < inp.cache_rows // 64


def test_named_workloads_recipe():
    w = workloads.get("mlra4_n8_l32k")
    assert (w.d_blk, w.num_branches) == (128, 4)
    assert math.isclose(w.sigma, 1 / math.sqrt(192)) and w.gamma == 0.25
    assert math.isclose(w.latent_scale, 1 / math.sqrt(2))
    mla = workloads.get("mla_n8_l32k")
    assert mla.seed == w.seed and mla.latent_scale == w.latent_scale and mla.gamma == 1.0
    t = workloads.get("tiny_mlra4_f32")
    assert t.dtype == "f32" and math.isclose(t.sigma, 1 / math.sqrt(48)) and t.latent_scale == 1.0
    assert math.isclose(workloads.get("long_mlra2_l128k").latent_scale, 0.5)


def test_tp4_shard_workload_is_one_branch_of_mlra4():
    full, shard = workloads.get("mlra4_n8_l32k"), workloads.get("mlra4_tp4_shard_n8_l32k")
    assert shard.num_branches == 1 and shard.d_latent == full.d_blk
    assert shard.d_rope == full.d_rope and shard.batch == full.batch and shard.seq_len == full.seq_len
    assert math.isclose(shard.sigma, full.sigma) and math.isclose(shard.gamma, full.gamma)
    assert math.isclose(shard.latent_scale, full.latent_scale)
    # bytes per cached token: 192 elements against MLRA-4's (and MLA's) 576 on one device
    assert (shard.d_latent + shard.d_rope) * 3 == full.d_latent + full.d_rope
