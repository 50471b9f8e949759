"""CUDA path (through the C ABI) against the CPU oracle on identical seeded inputs.

Small sizes span several 64-position tiles and ragged tails; every kernel variant, the
split-K merge, the paged layout, the summed output mode and the log-sum-exp output are
covered.  Index work (page resolution, page shuffles, branch independence) is compared
bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import assert_close, assert_lse_close, run_gpu, run_oracle, to_dev

pytestmark = pytest.mark.gpu

EDGE_LENS = [300, 1, 65, 0, 128, 64, 1000, 63]


def small_inputs(B=4, d_latent=512, d_rope=64, lens=EDGE_LENS, heads=64, page_size=0, seed=11,
                 dtype="bf16"):
    w = workloads.small(batch=len(lens), heads=heads, num_branches=B, d_latent=d_latent,
                        d_rope=d_rope, seq_len=max(lens), page_size=page_size, seed=seed,
                        dtype=dtype)
    return workloads.make_inputs(w, seq_lens=torch.tensor(lens, dtype=torch.int32))


def test_tiny_mlra4_fp32():
    """fp32 inputs, d_blk = 32, d_R = 16, 8 heads: device cast + padding path."""
    inp = workloads.make_inputs(workloads.get("tiny_mlra4_f32"))
    out, lse = run_gpu(inp)
    # strict: oracle on the bf16-rounded values the kernel computes with
    rounded = workloads.Inputs(inp.workload, inp.q_lat.bfloat16(), inp.q_rope.bfloat16(),
                               inp.c_kv.bfloat16(), inp.k_rope.bfloat16(), inp.seq_lens, None,
                               inp.max_seq_len)
    ref, ref_lse = run_oracle(inp, f32_source=rounded)
    assert_close(out, ref, "tiny vs bf16-rounded oracle")
    assert_lse_close(lse, ref_lse, "tiny lse")
    # and against the original fp32 values
    ref32, _ = run_oracle(inp)
    assert_close(out, ref32, "tiny vs fp32 oracle")


@pytest.mark.parametrize("B,d_latent,d_rope", [
    (4, 512, 64),    # MLRA-4, two branches per CTA
    (2, 512, 64),    # MLRA-2, one 256-wide branch per CTA
    (1, 512, 64),    # MLA
    (8, 512, 64),    # 64-wide branches, two per CTA
    (1, 128, 64),    # one 128-wide branch
    (3, 192, 32),    # odd branch count, padded widths (repack path)
])
def test_variants_small(B, d_latent, d_rope):
    inp = small_inputs(B=B, d_latent=d_latent, d_rope=d_rope)
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"B={B}")
    assert_lse_close(lse, ref_lse, f"B={B}")


@pytest.mark.parametrize("num_ranges", [0, 1, 2, 7, 64, 400])
def test_split_counts(num_ranges):
    """Any number of work ranges (1 = no split; many = most sequences split) agrees."""
    inp = small_inputs()
    out, lse = run_gpu(inp, num_ranges=num_ranges)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"R={num_ranges}")
    assert_lse_close(lse, ref_lse, f"R={num_ranges}")


@pytest.mark.parametrize("B,d_latent", [(4, 512), (2, 512), (1, 512), (8, 512), (1, 128)])
@pytest.mark.parametrize("lens,num_ranges", [([128], 1), ([2048], 8), ([2048], 1), ([300, 192], 2)])
def test_multi_tile_segments(B, d_latent, lens, num_ranges):
    """Segments of several tiles whose last tile is full: the epilogue must wait for the last
    output MMAs of the segment (a parity wait one phase behind would pass early)."""
    inp = small_inputs(B=B, d_latent=d_latent, lens=lens, seed=13)
    out, lse = run_gpu(inp, num_ranges=num_ranges)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"B={B} lens={lens} R={num_ranges}")
    assert_lse_close(lse, ref_lse, f"B={B}")


def test_summed_mode():
    inp = small_inputs(B=4)
    out, lse = run_gpu(inp, out_mode="summed")
    ref, ref_lse = run_oracle(inp, out_mode="summed")
    assert_close(out, ref, "summed")
    assert_lse_close(lse, ref_lse, "summed lse")


def test_few_heads_and_empty():
    inp = small_inputs(heads=5, lens=[0, 70, 0])
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    assert (out[0] == 0).all() and (out[2] == 0).all()
    assert torch.isneginf(lse[0]).all()
    assert_close(out, ref, "H=5")
    assert_lse_close(lse, ref_lse, "H=5 lse")


def test_paged_shuffle_is_bitwise_contiguous():
    """Same rows stored in shuffled pages give the same bits as the contiguous layout."""
    cont = small_inputs(lens=[300, 65, 1000, 1], seed=5)
    w = cont.workload
    P = 64
    N = len(cont.seq_lens)
    pages = [(int(l) + P - 1) // P for l in cont.seq_lens]
    n_pages = sum(pages) + 2
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(n_pages, generator=g)
    max_pages = (cont.max_seq_len + P - 1) // P
    pt = torch.full((N, max_pages), -1, dtype=torch.int32)
    c_pool = torch.full((n_pages * P, w.d_latent), float("nan")).bfloat16()
    kr_pool = torch.full((n_pages * P, w.d_rope), float("nan")).bfloat16()
    k = 0
    for s in range(N):
        for pg in range(pages[s]):
            pid = int(perm[k]); k += 1
            pt[s, pg] = pid
            src = s * cont.max_seq_len + pg * P
            c_pool[pid * P:(pid + 1) * P] = cont.c_kv[src:src + P]
            kr_pool[pid * P:(pid + 1) * P] = cont.k_rope[src:src + P]
    pw = workloads.Workload(**{**w.__dict__, "page_size": P})
    paged = workloads.Inputs(pw, cont.q_lat, cont.q_rope, c_pool, kr_pool, cont.seq_lens, pt,
                             max_pages * P)
    for R in (0, 3):
        a, la = run_gpu(cont, num_ranges=R)
        b, lb = run_gpu(paged, num_ranges=R)
        assert torch.equal(a, b) and torch.equal(la, lb), f"R={R}"
    ref, _ = run_oracle(cont)
    assert_close(b, ref, "paged")


def test_branch_independence_bitwise():
    inp = small_inputs(B=4, lens=[500, 77])
    base, lb = run_gpu(inp)
    d = 128
    for bp in (0, 3):
        c2 = inp.c_kv.clone()
        c2[:, bp * d:(bp + 1) * d] = torch.randn(c2.shape[0], d, generator=torch.Generator().manual_seed(bp)).bfloat16()
        mod = workloads.Inputs(inp.workload, inp.q_lat, inp.q_rope, c2, inp.k_rope, inp.seq_lens, None,
                               inp.max_seq_len)
        out, lo = run_gpu(mod)
        for b in range(4):
            same = torch.equal(out[..., b * d:(b + 1) * d], base[..., b * d:(b + 1) * d])
            assert same == (b != bp), (bp, b)


def test_nonfinite_rows_past_the_end_are_ignored():
    """Cache rows after a sequence's last position (same tile) may hold NaN/Inf."""
    w = workloads.small(batch=2, seq_len=128, seed=3)  # 128-row slot per sequence
    inp = workloads.make_inputs(w, seq_lens=torch.tensor([100, 30], dtype=torch.int32))
    c = inp.c_kv.clone()
    kr = inp.k_rope.clone()
    for s, L in enumerate([100, 30]):
        lo, hi = s * inp.max_seq_len + L, s * inp.max_seq_len + ((L + 63) // 64) * 64
        c[lo:hi] = float("nan")
        kr[lo:hi] = float("inf")
    mod = workloads.Inputs(inp.workload, inp.q_lat, inp.q_rope, c, kr, inp.seq_lens, None, inp.max_seq_len)
    out, lse = run_gpu(mod)
    ref, ref_lse = run_oracle(mod)
    assert_close(out, ref, "nan tail")
    assert_lse_close(lse, ref_lse, "nan tail lse")


def test_closed_forms():
    """Zero queries: gamma * mean of each block; constant latent: gamma * constant."""
    inp = small_inputs(lens=[700, 64, 1])
    zq = workloads.Inputs(inp.workload, torch.zeros_like(inp.q_lat), torch.zeros_like(inp.q_rope),
                          inp.c_kv, inp.k_rope, inp.seq_lens, None, inp.max_seq_len)
    out, lse = run_gpu(zq)
    for s, L in enumerate([700, 64, 1]):
        rows = inp.c_kv[s * inp.max_seq_len:s * inp.max_seq_len + L].double()
        expect = (0.25 * rows.mean(0)).numpy()
        np.testing.assert_allclose(out[s].cpu().double().numpy(), np.broadcast_to(expect, (64, 512)),
                                   rtol=0, atol=2e-3 * max(1.0, np.abs(expect).max()))
        np.testing.assert_allclose(lse[s].cpu().numpy(), math.log(L), rtol=1e-5, atol=1e-4)
    cc = workloads.Inputs(inp.workload, inp.q_lat, inp.q_rope, torch.full_like(inp.c_kv, 1.5),
                          inp.k_rope, inp.seq_lens, None, inp.max_seq_len)
    out, _ = run_gpu(cc)
    np.testing.assert_allclose(out.cpu().numpy(), 0.375, rtol=0, atol=0.375 * 8e-3)


def test_shared_576_wide_rows():
    """c_kv and k_rope as two column ranges of one [rows, 576] cache: same bits as separate."""
    inp = small_inputs(lens=[333, 90])
    dev = to_dev(inp)
    packed = torch.cat([dev[2], dev[3]], dim=1).contiguous()
    a, la = run_gpu(inp, dev_tensors=dev)
    b, lb = run_gpu(inp, dev_tensors=(dev[0], dev[1], packed[:, :512], packed[:, 512:], dev[4], dev[5]))
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_resolve_rows_bit_exact():
    w = workloads.small(batch=6, seq_len=5000, min_seq_len=1, ragged=True, page_size=128, seed=4)
    inp = workloads.make_inputs(w)
    lens = inp.seq_lens.cuda()
    pt = inp.page_table.cuda()
    dims = mlra.dims_for(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, lens, pt, 4, page_size=128)
    pitch = 5000
    rows = mlra.resolve_rows(lens, pt, dims, pitch).cpu()
    for s, L in enumerate(inp.seq_lens.tolist()):
        ref = oracle.resolve_rows(L, s, inp.page_table.numpy(), 128, 0)
        assert np.array_equal(rows[s, :L].numpy(), ref)
        assert (rows[s, L:] == -1).all()
    cdims = mlra.make_dims(batch=3, heads=64, num_branches=4, d_latent=512, d_rope=64,
                           max_seq_len=700, cache_rows=2100)
    clens = torch.tensor([700, 5, 0], dtype=torch.int32, device="cuda")
    crow = mlra.resolve_rows(clens, None, cdims, 700).cpu()
    for s, L in enumerate([700, 5, 0]):
        assert np.array_equal(crow[s, :L].numpy(), oracle.resolve_rows(L, s, None, 0, 700))


def test_status_flags():
    inp = small_inputs(lens=[200, 100], page_size=64, seed=8)
    dev = list(to_dev(inp))
    dec = mlra.Decoder(*dev, num_branches=4, softmax_scale=inp.workload.sigma,
                       max_seq_len=inp.max_seq_len, page_size=64)
    dec()
    assert dec.status() == (mlra.MLRA_OK, 0)
    bad_pt = dev[5].clone()
    bad_pt[1, 0] = 10 ** 6                                 # page id beyond the pool
    dec(args=(dev[0], dev[1], dev[2], dev[3], dev[4], bad_pt))
    rc, flags = dec.status()
    assert rc == mlra.MLRA_ERR_BAD_PAGE and flags == mlra.FLAG_BAD_PAGE
    assert torch.isfinite(dec.out).all()
    # a clamped over-long length also reaches the unused (-1) page-table entries
    bad_len = torch.tensor([200, 10 ** 7], dtype=torch.int32, device="cuda")
    dec(args=(dev[0], dev[1], dev[2], dev[3], bad_len, dev[5]))
    rc, flags = dec.status()
    assert rc == mlra.MLRA_ERR_BAD_PAGE and flags == mlra.FLAG_BAD_PAGE | mlra.FLAG_BAD_LENGTH
    dec()
    assert dec.status() == (mlra.MLRA_OK, 0)               # the word is per call
    # contiguous layout: lengths outside [0, max_seq_len] alone
    cont = small_inputs(lens=[200, 100], seed=8)
    cdev = list(to_dev(cont))
    cdec = mlra.Decoder(*cdev, num_branches=4, softmax_scale=cont.workload.sigma,
                        max_seq_len=cont.max_seq_len)
    for lens in ([200, 201], [-1, 100]):
        cdec(args=(*cdev[:4], torch.tensor(lens, dtype=torch.int32, device="cuda"), None))
        assert cdec.status() == (mlra.MLRA_ERR_BAD_LENGTH, mlra.FLAG_BAD_LENGTH)
        assert torch.isfinite(cdec.out).all()


@pytest.mark.parametrize("N,R", [(65, 0), (80, 7), (96, 300)])
def test_more_sequences_than_the_in_kernel_plan(N, R):
    """Batches above the in-kernel plan's limit take the prep-kernel path (one more launch);
    results, empty sequences and the status word behave the same."""
    rnd = np.random.default_rng(N)
    lens = [int(x) for x in rnd.choice([0, 1, 17, 64, 128, 129, 300, 700], size=N)]
    inp = small_inputs(lens=lens, heads=8, seed=N)
    q, qr, c, kr, dlens, pt = to_dev(inp)
    w = inp.workload
    plan = mlra.query_plan(mlra.dims_for(q, qr, c, kr, dlens, pt, w.num_branches,
                                         max_seq_len=inp.max_seq_len, num_ranges=R))
    assert plan.launches == 3
    out, lse = run_gpu(inp, num_ranges=R)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"N={N} R={R}")
    assert_lse_close(lse, ref_lse, f"N={N} R={R}")
    empty = [i for i, L in enumerate(lens) if L == 0]
    assert (out[empty] == 0).all() and torch.isinf(lse[empty]).all()
    bad = dlens.clone()
    bad[3] = -5
    dec = mlra.Decoder(q, qr, c, kr, dlens, pt, num_branches=w.num_branches, softmax_scale=w.sigma,
                       max_seq_len=inp.max_seq_len, num_ranges=R)
    dec(args=(q, qr, c, kr, bad, pt))
    assert dec.status() == (mlra.MLRA_ERR_BAD_LENGTH, mlra.FLAG_BAD_LENGTH)
    dec()
    assert dec.status() == (mlra.MLRA_OK, 0)


def test_repeat_calls_are_deterministic():
    inp = small_inputs()
    dev = to_dev(inp)
    dec = mlra.Decoder(*dev, num_branches=4, softmax_scale=inp.workload.sigma,
                       max_seq_len=inp.max_seq_len, with_lse=True)
    a = dec().clone()
    for _ in range(3):
        assert torch.equal(dec(), a)


# ----------------------------------------------------------------------------- full sizes
def _sampled(name, seqs, heads, R=0):
    inp = workloads.make_inputs(workloads.get(name))
    out, lse = run_gpu(inp, num_ranges=R)
    ref, ref_lse = run_oracle(inp, seqs=seqs, heads=heads)
    got = out[seqs][:, heads]
    assert_close(got, ref, name)
    assert_lse_close(lse[seqs][:, heads], ref_lse, name)
    assert torch.isfinite(out).all()
    return out


@pytest.mark.parametrize("B,heads,page_size", [(1, 128, 0), (4, 128, 0), (4, 128, 64), (2, 96, 64),
                                               (1, 72, 0)])
def test_head_groups(B, heads, page_size):
    """More than 64 heads: one CTA per (range, branch, 64-head group); a partial last group."""
    inp = small_inputs(B=B, heads=heads, lens=[300, 1, 129, 700], page_size=page_size, seed=71)
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"B={B} H={heads}")
    assert_lse_close(lse, ref_lse, f"B={B} H={heads}")


def test_128_heads_in_one_cta():
    """128 heads with 128-wide branches read in place: one CTA per (range, branch) carries both
    head groups as 128-row products (the plan counts B CTAs per range, not 2 B); against the
    oracle with ragged lengths, forced ranges, summed output and a replanned call."""
    inp = small_inputs(B=4, heads=128, lens=[1, 700, 129, 2049, 64], seed=73)
    w = inp.workload
    q, qr, c, kr, lens, pt = to_dev(inp)
    dims = mlra.dims_for(q, qr, c, kr, lens, pt, 4, max_seq_len=inp.max_seq_len, num_ranges=9)
    assert mlra.query_plan(dims).ctas == 9 * 4
    out, lse = run_gpu(inp, num_ranges=9)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, "128 heads, 9 ranges")
    assert_lse_close(lse, ref_lse, "128 heads lse")
    outs, _ = run_gpu(inp, out_mode="summed")
    refs, _ = run_oracle(inp, out_mode="summed")
    assert_close(outs, refs, "128 heads, summed")


@pytest.mark.parametrize("name,seqs,heads", [
    ("mla_h128_n8_l32k", [0, 7], [0, 63, 64, 127]),
    ("mlra4_h128_n8_l32k", [0, 5], [0, 63, 64, 127]),
    ("mlra4_n8_l32k", [0, 5, 7], [0, 17, 33, 63]),
    ("mla_n8_l32k", [1, 6], [2, 40, 63]),
    ("long_mlra4_l128k", [0], [0, 9, 31, 62]),
    ("long_mlra2_l128k", [0], [1, 30, 63]),
    ("serving_mlra4_n64_paged", [0, 13, 37, 63], [0, 21, 63]),
])
def test_full_size_sampled(name, seqs, heads):
    _sampled(name, seqs, heads)


@pytest.mark.parametrize("B,paged", [(4, False), (2, True)])
def test_replan_path(B, paged, monkeypatch):
    """The attention kernel plans its work range before its dependency wait and keeps that plan
    when the lengths read after the wait are unchanged; otherwise it lets the loads it issued on
    the stale plan land, resets its barriers and re-plans.  The environment variable
    MLRA_TEST_FORCE_REPLAN makes every call take that second path: the result must still match
    the oracle, and equal bit for bit the result of the normal path."""
    inp = small_inputs(B=B, lens=[300, 1, 65, 0, 1000, 63], page_size=64 if paged else 0, seed=19)
    base, base_lse = run_gpu(inp)
    monkeypatch.setenv("MLRA_TEST_FORCE_REPLAN", "1")
    out, lse = run_gpu(inp)
    monkeypatch.delenv("MLRA_TEST_FORCE_REPLAN")
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, f"re-plan B={B} paged={paged}")
    assert_lse_close(lse, ref_lse, "re-plan lse")
    assert torch.equal(out, base) and torch.equal(lse, base_lse)


@pytest.mark.parametrize("page_size", [0, 64])
def test_large_batch(page_size):
    """700 short ragged sequences (some empty): the prep kernel's plan over many sequences, and
    work ranges that each run through about twenty segments (a query load and an epilogue each)."""
    g = torch.Generator().manual_seed(41)
    lens = torch.randint(0, 160, (700,), generator=g)
    lens[::97] = 0
    inp = small_inputs(B=4, lens=lens.tolist(), page_size=page_size, seed=42)
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    empty = (lens == 0).nonzero().flatten()
    assert (out[empty] == 0).all() and torch.isneginf(lse[empty]).all()
    assert_close(out, ref, f"N=700 paged={page_size}")
    assert_lse_close(lse, ref_lse, f"N=700 paged={page_size} lse")


def test_128_heads_through_the_prep_kernel():
    """80 sequences with 128 heads: the 128-row kernel (all heads of a branch in one CTA) reading the
    prep kernel's plan."""
    g = torch.Generator().manual_seed(43)
    lens = torch.randint(0, 400, (80,), generator=g).tolist()
    inp = small_inputs(B=4, heads=128, lens=lens, page_size=64, seed=44)
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, "H=128, N=80")
    assert_lse_close(lse, ref_lse, "H=128, N=80 lse")


def test_plan_in_workspace_scratch():
    """2600 sequences: past the 2400 whose plan the prep kernel keeps in shared memory, so its
    prefixes and part ranges live in the workspace instead."""
    g = torch.Generator().manual_seed(45)
    lens = torch.randint(0, 40, (2600,), generator=g)
    lens[::50] = 0
    inp = small_inputs(B=4, heads=8, lens=lens.tolist(), seed=46)
    out, lse = run_gpu(inp)
    ref, ref_lse = run_oracle(inp)
    assert_close(out, ref, "N=2600")
    assert_lse_close(lse, ref_lse, "N=2600 lse")
