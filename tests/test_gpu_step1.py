"""Step 1 (mlra_absorb, mlra_pack_wuk) and the new token's RoPE and cache append
(mlra_rope_append), through the C ABI, against the oracle; and steps 1 -> 2 -> 3 chained."""
import numpy as np
import pytest
import torch

import oracle
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

BF16_REL = 2.0 ** -8   # one bf16 rounding of the result


@pytest.mark.parametrize("N,H,d_head,d_latent", [(8, 64, 128, 512), (3, 5, 64, 192), (70, 2, 128, 256),
                                                  (5, 32, 128, 512), (64, 64, 128, 512)])
def test_absorb_matches_oracle(N, H, d_head, d_latent):
    g = torch.Generator().manual_seed(N + H)
    q = torch.randn(N, H, d_head, generator=g)
    w = (torch.randn(H, d_head, d_latent, generator=g) / d_head ** 0.5).to(torch.bfloat16)
    q_lat = mlra.absorb(q.cuda(), mlra.pack_wuk(w.cuda()))
    torch.cuda.synchronize()
    assert q_lat.dtype == torch.bfloat16 and q_lat.shape == (N, H, d_latent)
    ref = oracle.absorb(q.to(torch.bfloat16).float(), w.float())      # the kernel rounds q
    got = q_lat.float().cpu().double().numpy()
    err = np.abs(got - ref)
    assert err.max() <= BF16_REL * np.abs(ref).max(), err.max() / np.abs(ref).max()
    assert_close(q_lat.float(), oracle.absorb(q, w.float()), "absorb vs unrounded q")


def test_pack_wuk_is_the_transpose():
    H, d_head, d_latent = 2, 64, 128
    w = torch.arange(H * d_head * d_latent, dtype=torch.float32).remainder(241).to(torch.bfloat16)
    w = w.view(H, d_head, d_latent).cuda()
    packed = mlra.pack_wuk(w).view(-1).cpu()
    wt = w.cpu().transpose(1, 2)                                     # A_h = w[h]^T: [d_latent, d_head]
    KB, mt = d_head // 64, d_latent // 64
    for (h, m, kb, r, j) in [(0, 0, 0, 0, 0), (1, 1, 0, 63, 7), (1, 0, 0, 9, 2)]:
        box = (h * mt + m) * KB + kb
        pos = j ^ (r % 8)
        got = packed[box * 4096 + r * 64 + pos * 8: box * 4096 + r * 64 + pos * 8 + 8]
        want = wt[h, m * 64 + r, kb * 64 + 8 * j: kb * 64 + 8 * j + 8]
        assert torch.equal(got, want), (h, m, kb, r, j)


def _cache(rows, d_c, d_R, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, d_c, generator=g).to(torch.bfloat16),
            torch.randn(rows, d_R, generator=g).to(torch.bfloat16))


@pytest.mark.parametrize("case", ["contiguous", "paged", "paged_far"])
def test_rope_append_matches_oracle(case):
    """Rotations against the float64 oracle (one bf16 rounding), the appended rows against the
    oracle's append (latent bit-exact, key within a bf16 rounding), every other row untouched.
    paged_far puts the new tokens at positions up to 131071 (angles of 10^5 radians)."""
    N, H, d_R, d_c, P = 4, 6, 64, 512, 64
    g = torch.Generator().manual_seed(3)
    if case == "contiguous":
        lens = torch.tensor([0, 63, 64, 255], dtype=torch.int32)
        pt, max_len, rows = None, 256, 4 * 256
    else:
        lens = torch.tensor([0, 63, 64, 300] if case == "paged" else [5, 65535, 100000, 131071],
                            dtype=torch.int32)
        max_pages = 2048 if case == "paged_far" else 5
        pt = torch.full((N, max_pages), -1, dtype=torch.int32)
        for s_, L in enumerate(lens.tolist()):            # the page holding the new position
            pt[s_, L // P] = [2, 0, 5, 3][s_]
        max_len, rows = 0, 6 * P
    c_kv, k_rope = _cache(rows, d_c, d_R, 4)
    q_in = torch.randn(N, H, d_R, generator=g)
    k_new = torch.randn(N, d_R, generator=g)
    c_new = torch.randn(N, d_c, generator=g)
    dc, dk = c_kv.cuda(), k_rope.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_out = mlra.rope_append(q_in.cuda(), k_new.cuda(), c_new.cuda(), lens.cuda(),
                             None if pt is None else pt.cuda(), dc, dk,
                             max_seq_len=max_len if pt is None else None,
                             page_size=0 if pt is None else P, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pos = lens.double().numpy()
    q_ref = oracle.rope(q_in, pos[:, None], 10000.0)
    err = np.abs(q_out.float().cpu().double().numpy() - q_ref)
    assert err.max() <= BF16_REL * np.abs(q_ref).max() + 1e-6, err.max()
    k_ref = oracle.rope(k_new, pos, 10000.0)
    c_ref, kr_ref, _ = oracle.append_token(c_kv.float(), k_rope.float(), lens,
                                           None if pt is None else pt.numpy(), P, max_len,
                                           c_new.to(torch.bfloat16).float(), k_ref)
    gc, gk = dc.float().cpu().double().numpy(), dk.float().cpu().double().numpy()
    changed = set(np.nonzero((gc != c_kv.float().double().numpy()).any(1) |
                             (gk != k_rope.float().double().numpy()).any(1))[0].tolist())
    want_rows = [int(oracle.resolve_rows(L + 1, s_, None if pt is None else pt.numpy(), P,
                                         max_len)[L]) for s_, L in enumerate(lens.tolist())]
    assert changed <= set(want_rows), (changed, want_rows)          # nothing else was written
    for r in want_rows:
        assert np.array_equal(gc[r], c_ref[r])                       # bf16(c_new), exact
        assert np.abs(gk[r] - kr_ref[r]).max() <= BF16_REL * np.abs(kr_ref[r]).max() + 1e-6


def test_rope_append_flags_and_skips():
    N, H, d_R, d_c, P = 2, 2, 64, 128, 64
    c_kv, k_rope = _cache(4 * P, d_c, d_R, 6)
    dc, dk = c_kv.cuda(), k_rope.cuda()
    pt = torch.tensor([[0, 9], [1, -1]], dtype=torch.int32).cuda()   # page 9 is past the pool
    lens = torch.tensor([64, 200], dtype=torch.int32).cuda()         # bad page; past max pages
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    z = torch.zeros
    mlra.rope_append(z(N, H, d_R).cuda(), z(N, d_R).cuda(), z(N, d_c).cuda(), lens, pt, dc, dk,
                     page_size=P, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == mlra.FLAG_BAD_PAGE | mlra.FLAG_BAD_LENGTH
    assert torch.equal(dc.cpu(), c_kv) and torch.equal(dk.cpu(), k_rope)


def test_steps_1_2_3_chained():
    """absorb -> rope_append -> decode -> project on the CUDA path against the oracle's chain."""
    N, H, B, d_head, d_c, d_R, L = 3, 8, 4, 128, 512, 64, 200
    g = torch.Generator().manual_seed(11)
    w_uk = (torch.randn(H, d_head, d_c, generator=g) / d_head ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(H, d_head, d_c, generator=g) / d_c ** 0.5).to(torch.bfloat16)
    q_nope = torch.randn(N, H, d_head, generator=g)
    q_rope_in = torch.randn(N, H, d_R, generator=g)
    k_new, c_new = torch.randn(N, d_R, generator=g), torch.randn(N, d_c, generator=g) * 0.7
    c_kv, k_rope = _cache(N * L, d_c, d_R, 12)
    c_kv = (c_kv.float() * 0.7).to(torch.bfloat16)
    lens = torch.tensor([17, 0, 150], dtype=torch.int32)
    sigma, gamma = 1 / (d_head + d_R) ** 0.5, 1.0 / B
    # CUDA path
    dc, dk, dl = c_kv.cuda(), k_rope.cuda(), lens.cuda()
    q_lat = mlra.absorb(q_nope.cuda(), mlra.pack_wuk(w_uk.cuda()))
    q_rope = mlra.rope_append(q_rope_in.cuda(), k_new.cuda(), c_new.cuda(), dl, None, dc, dk,
                              max_seq_len=L)
    out, _ = mlra.decode(q_lat, q_rope, dc, dk, dl + 1, None, num_branches=B, softmax_scale=sigma,
                         branch_scale=gamma, max_seq_len=L)
    y = mlra.project(out.contiguous(), mlra.pack_wuv(w_uv.cuda()))
    # oracle chain (float64 throughout; the cache holds what the append wrote, in bf16)
    q_lat_ref = oracle.absorb(q_nope, w_uk.float())
    pos = lens.double().numpy()
    q_rope_ref = oracle.rope(q_rope_in, pos[:, None], 10000.0)
    k_ref = oracle.rope(k_new, pos, 10000.0)
    c2, k2, lens2 = oracle.append_token(c_kv.float(), k_rope.float(), lens, None, 0, L,
                                        c_new.to(torch.bfloat16).float(),
                                        torch.from_numpy(k_ref).to(torch.bfloat16).float())
    out_ref, _ = oracle.decode(q_lat_ref, q_rope_ref, c2, k2, lens2, None, B, sigma, gamma,
                               max_seq_len=L)
    assert_close(y, oracle.project(out_ref, w_uv.float()), "steps 1-2-3")


def test_layer_chain_full_size_sampled():
    """RoPE/append -> absorb -> decode -> project at the mlra4_n8_l32k shapes (8 x 32768 tokens,
    64 heads, d_c = 512, d_head = 128) on the CUDA path, against the oracle's chain on sampled
    sequences (their cache rows cut out: the contiguous layout keeps a sequence's rows together)."""
    import workloads
    w = workloads.get("mlra4_n8_l32k")
    inp = workloads.make_inputs(w)
    N, H, d_c, d_R, d_head, L = w.batch, w.heads, w.d_latent, w.d_rope, 128, inp.max_seq_len
    g = torch.Generator().manual_seed(13)
    w_uk = (torch.randn(H, d_head, d_c, generator=g) / d_head ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(H, d_head, d_c, generator=g) / d_c ** 0.5).to(torch.bfloat16)
    q_nope = torch.randn(N, H, d_head, generator=g)
    q_rope_in = torch.randn(N, H, d_R, generator=g)
    k_new, c_new = torch.randn(N, d_R, generator=g), torch.randn(N, d_c, generator=g) * 0.7
    lens_in = inp.seq_lens - 1  # the new token takes the last row of each sequence's space
    # CUDA path
    dc, dk = inp.c_kv.cuda(), inp.k_rope.cuda()
    q_rope = mlra.rope_append(q_rope_in.cuda(), k_new.cuda(), c_new.cuda(), lens_in.cuda(), None,
                              dc, dk, max_seq_len=L)
    q_lat = mlra.absorb(q_nope.cuda(), mlra.pack_wuk(w_uk.cuda()))
    out, _ = mlra.decode(q_lat, q_rope, dc, dk, inp.seq_lens.cuda(), None, num_branches=w.num_branches,
                         softmax_scale=w.sigma, branch_scale=w.gamma, max_seq_len=L)
    y = mlra.project(out.contiguous(), mlra.pack_wuv(w_uv.cuda())).cpu()
    # oracle chain on the sampled sequences
    seqs = [0, 5]
    rows = torch.cat([torch.arange(s * L, (s + 1) * L) for s in seqs])
    c_sub, k_sub = inp.c_kv[rows].float(), inp.k_rope[rows].float()
    pos = lens_in[seqs].double().numpy()
    k_ref = oracle.rope(k_new[seqs], pos, 10000.0)
    c2, k2, lens2 = oracle.append_token(c_sub, k_sub, lens_in[seqs], None, 0, L,
                                        c_new[seqs].to(torch.bfloat16).float(),
                                        torch.from_numpy(k_ref).to(torch.bfloat16).float())
    out_ref, _ = oracle.decode(oracle.absorb(q_nope[seqs], w_uk.float()),
                               oracle.rope(q_rope_in[seqs], pos[:, None], 10000.0), c2, k2, lens2,
                               None, w.num_branches, w.sigma, w.gamma, max_seq_len=L)
    assert_close(y[seqs], oracle.project(out_ref, w_uv.float()), "layer chain, full size")
