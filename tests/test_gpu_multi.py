"""Several query tokens per sequence (``mlra_decode_multi``) against the oracle's
``decode_multi``: token t of sequence s attends positions 0 .. seq_lens[s] - q + t."""
import pytest
import torch

import oracle
import workloads
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu


def multi_inputs(q, lens, B=4, d_latent=512, heads=64, page_size=0, seed=51):
    w = workloads.small(batch=len(lens), heads=heads, num_branches=B, d_latent=d_latent, d_rope=64,
                        seq_len=max(lens), page_size=page_size, seed=seed)
    inp = workloads.make_inputs(w, seq_lens=torch.tensor(lens, dtype=torch.int32))
    g = torch.Generator().manual_seed(seed + 1)
    q_lat = torch.randn(len(lens), q, heads, d_latent, generator=g).to(torch.bfloat16)
    q_rope = torch.randn(len(lens), q, heads, 64, generator=g).to(torch.bfloat16)
    return w, inp, q_lat, q_rope


def run_multi(w, inp, q_lat, q_rope, **kw):
    pt = None if inp.page_table is None else inp.page_table.cuda()
    return mlra.decode_multi(q_lat.cuda(), q_rope.cuda(), inp.c_kv.cuda(), inp.k_rope.cuda(),
                             inp.seq_lens.cuda(), pt, num_branches=w.num_branches,
                             softmax_scale=w.sigma, branch_scale=w.gamma,
                             max_seq_len=inp.max_seq_len, page_size=w.page_size, with_lse=True, **kw)


@pytest.mark.parametrize("q,lens,B,page_size", [
    (2, [2, 300, 129, 1000], 4, 0),
    (3, [3, 64, 65, 700, 1], 4, 0),      # the last sequence is shorter than q: flagged
    (4, [4, 129, 2000], 1, 0),
    (2, [5, 190, 1500], 4, 64),
    (8, [8, 256, 4000], 2, 64),
])
def test_multi_token_matches_oracle(q, lens, B, page_size):
    w, inp, q_lat, q_rope = multi_inputs(q, lens, B=B, page_size=page_size)
    out, lse = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens,
                                       inp.page_table, w.num_branches, w.sigma, w.gamma,
                                       page_size=page_size, max_seq_len=inp.max_seq_len)
    assert out.shape == (len(lens), q, w.heads, w.d_latent)
    assert_close(out, ref, f"q={q}")
    assert_lse_close(lse, ref_lse, f"q={q} lse")  # empty tokens: -inf on both sides


def test_multi_token_through_the_prep_kernel():
    """40 sequences x 2 tokens = 80 virtual sequences: more than the attention kernel plans itself,
    so the prep kernel plans them (virtual lengths from the caller's lengths there too)."""
    g = torch.Generator().manual_seed(91)
    lens = (torch.randint(2, 400, (40,), generator=g)).tolist()
    w, inp, q_lat, q_rope = multi_inputs(2, lens, B=4, heads=8, d_latent=256, seed=92)
    out, lse = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None,
                                       w.num_branches, w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    assert_close(out, ref, "80 virtual sequences")
    assert_lse_close(lse, ref_lse, "80 virtual sequences lse")


def test_short_sequence_is_flagged():
    """seq_lens[s] < q - 1 leaves some tokens with a negative length: MLRA_FLAG_BAD_LENGTH, and
    their outputs are empty (zeros); the other sequences are unaffected."""
    q, lens = 4, [1, 50]
    w, inp, q_lat, q_rope = multi_inputs(q, lens, heads=8, d_latent=128, B=4)
    pt = None
    dims = mlra.dims_for(q_lat[:, 0].cuda(), q_rope[:, 0].cuda(), inp.c_kv.cuda(), inp.k_rope.cuda(),
                         inp.seq_lens.cuda(), pt, w.num_branches, max_seq_len=inp.max_seq_len)
    ws = torch.zeros(mlra.workspace_size_multi(dims, q), dtype=torch.uint8, device="cuda")
    out, _ = run_multi(w, inp, q_lat, q_rope, workspace=ws)
    rc, flags = mlra.read_status(ws)
    assert flags & mlra.FLAG_BAD_LENGTH
    assert torch.count_nonzero(out[0, :3]) == 0          # lengths -2, -1 and 0: nothing to see
    ref, _ = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None,
                                 w.num_branches, w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    assert_close(out[1], ref[1], "the other sequence")
    assert_close(out[0, 3], ref[0, 3], "the token at position 0")


def test_multi_token_full_size_sampled():
    """q = 2 at the mlra4_n8_l32k shapes (8 x 32768 tokens, 64 heads, 4 x 128 + 64)."""
    w = workloads.get("mlra4_n8_l32k")
    inp = workloads.make_inputs(w)
    q = 2
    g = torch.Generator().manual_seed(61)
    q_lat = torch.randn(w.batch, q, w.heads, w.d_latent, generator=g).to(torch.bfloat16)
    q_rope = torch.randn(w.batch, q, w.heads, w.d_rope, generator=g).to(torch.bfloat16)
    out, _ = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    seqs, heads = [0, 6], [0, 31, 63]
    for t in range(q):
        lens_t = inp.seq_lens - (q - 1 - t)
        ref, _ = oracle.decode(q_lat[:, t], q_rope[:, t], inp.c_kv, inp.k_rope, lens_t, None,
                               w.num_branches, w.sigma, w.gamma, max_seq_len=inp.max_seq_len,
                               seqs=seqs, heads=heads)
        assert_close(out[seqs][:, t][:, heads], ref, f"token {t}")


# Two tokens of 64 heads per CTA (the 128-row attention kernel): an even number of tokens, 64
# heads and 128-wide branches read in place.
@pytest.mark.parametrize("q,lens,page_size", [
    (4, [4, 5, 129, 1000, 3], 0),       # a sequence of 3: its first token has length 0
    (2, [1, 2, 64, 65, 128, 129, 777], 64),
    (6, [6, 300, 2049], 0),
])
def test_two_tokens_per_cta_match_oracle(q, lens, page_size):
    w, inp, q_lat, q_rope = multi_inputs(q, lens, B=4, page_size=page_size, seed=71)
    out, lse = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens,
                                       inp.page_table, w.num_branches, w.sigma, w.gamma,
                                       page_size=page_size, max_seq_len=inp.max_seq_len)
    assert_close(out, ref, f"q={q}")
    assert_lse_close(lse, ref_lse, f"q={q} lse")


def test_two_tokens_per_cta_summed_and_replanned(monkeypatch):
    """Summed output mode (every result goes through the combine kernel) and the attention
    kernel's re-plan path, on the 128-row kernel."""
    q, lens = 2, [2, 300, 129, 1000]
    w, inp, q_lat, q_rope = multi_inputs(q, lens, B=4, seed=73)
    monkeypatch.setenv("MLRA_TEST_FORCE_REPLAN", "1")
    out, lse = run_multi(w, inp, q_lat, q_rope, out_mode="summed")
    torch.cuda.synchronize()
    monkeypatch.delenv("MLRA_TEST_FORCE_REPLAN")
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None,
                                       w.num_branches, w.sigma, w.gamma,
                                       max_seq_len=inp.max_seq_len, out_mode="summed")
    assert_close(out, ref, "summed")
    assert_lse_close(lse, ref_lse, "summed lse")


def test_two_tokens_per_cta_through_the_prep_kernel():
    """80 sequences x 2 tokens = 80 units of two tokens: the prep kernel plans them."""
    g = torch.Generator().manual_seed(93)
    lens = (torch.randint(1, 300, (80,), generator=g)).tolist()
    lens[5] = 0                                   # first token -1 (flagged), second 0
    w, inp, q_lat, q_rope = multi_inputs(2, lens, B=4, seed=94)
    pt = None
    dims = mlra.dims_for(q_lat[:, 0].cuda(), q_rope[:, 0].cuda(), inp.c_kv.cuda(), inp.k_rope.cuda(),
                         inp.seq_lens.cuda(), pt, w.num_branches, max_seq_len=inp.max_seq_len)
    ws = torch.zeros(mlra.workspace_size_multi(dims, 2), dtype=torch.uint8, device="cuda")
    out, lse = run_multi(w, inp, q_lat, q_rope, workspace=ws)
    rc, flags = mlra.read_status(ws)
    assert flags & mlra.FLAG_BAD_LENGTH
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None,
                                       w.num_branches, w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    assert torch.count_nonzero(out[5]) == 0
    assert_close(out, ref, "80 units")
    assert_lse_close(lse, ref_lse, "80 units lse")


def test_two_token_units_through_the_prep_kernel():
    """100 sequences x 2 tokens with 64 heads and 128-wide branches: 100 two-token units, more than
    the attention kernel plans itself, so the 128-row kernel reads the prep kernel's plan."""
    g = torch.Generator().manual_seed(93)
    lens = torch.randint(2, 300, (100,), generator=g).tolist()
    w, inp, q_lat, q_rope = multi_inputs(2, lens, B=4, heads=64, d_latent=512, page_size=64, seed=94)
    out, lse = run_multi(w, inp, q_lat, q_rope)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens,
                                       inp.page_table, w.num_branches, w.sigma, w.gamma,
                                       page_size=64, max_seq_len=inp.max_seq_len)
    assert_close(out, ref, "100 two-token units")
    assert_lse_close(lse, ref_lse, "100 two-token units lse")
