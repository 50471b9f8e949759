"""Softmax scales off the usual path: negative and zero.

The attention kernels take a tile's row maximum on the raw dot products and fold the scale into
each exponent, so a negative scale takes the row minimum instead; that branch is compared with
the oracle here for both attention kernels.  A zero scale makes every probability 1: each branch
output is then gamma times the plain mean of the branch's latent block over the sequence's
positions and the log-sum-exp is ln L -- a closed form checked from the inputs directly."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import assert_close, assert_lse_close, to_dev

pytestmark = pytest.mark.gpu

LENS = [300, 1, 1000, 129, 64]


def inputs(lens, B=4, heads=64, page_size=0, seed=81):
    w = workloads.small(batch=len(lens), heads=heads, num_branches=B, d_latent=512, d_rope=64,
                        seq_len=max(lens), page_size=page_size, seed=seed)
    return workloads.make_inputs(w, seq_lens=torch.tensor(lens, dtype=torch.int32))


def decode_both(inp, sigma, num_ranges=0):
    w = inp.workload
    q, qr, c, kr, sl, pt = to_dev(inp)
    out, lse = mlra.decode(q, qr, c, kr, sl, pt, num_branches=w.num_branches, softmax_scale=sigma,
                           branch_scale=w.gamma, max_seq_len=inp.max_seq_len,
                           page_size=w.page_size, with_lse=True, num_ranges=num_ranges)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens,
                                 inp.page_table, w.num_branches, sigma, w.gamma,
                                 page_size=w.page_size, max_seq_len=inp.max_seq_len)
    return out, lse, ref, ref_lse


@pytest.mark.parametrize("B,heads,page_size,num_ranges", [
    (4, 64, 0, 0), (4, 64, 64, 7), (2, 64, 0, 0), (1, 64, 0, 3), (8, 64, 0, 0),
    (4, 128, 0, 0),                  # 128 heads: the 128-row kernel
])
def test_negative_scale(B, heads, page_size, num_ranges):
    inp = inputs(LENS, B=B, heads=heads, page_size=page_size)
    sigma = -inp.workload.sigma
    out, lse, ref, ref_lse = decode_both(inp, sigma, num_ranges)
    assert_close(out, ref, f"sigma<0 B={B} H={heads}")
    assert_lse_close(lse, ref_lse, f"sigma<0 B={B} H={heads} lse")


def test_negative_scale_two_tokens():
    lens = [2, 300, 1000, 129]
    inp = inputs(lens, seed=83)
    w = inp.workload
    g = torch.Generator().manual_seed(84)
    q_lat = torch.randn(len(lens), 2, w.heads, 512, generator=g).to(torch.bfloat16)
    q_rope = torch.randn(len(lens), 2, w.heads, 64, generator=g).to(torch.bfloat16)
    _, _, c, kr, sl, _ = to_dev(inp)
    out, lse = mlra.decode_multi(q_lat.cuda(), q_rope.cuda(), c, kr, sl, None, num_branches=4,
                                 softmax_scale=-w.sigma, branch_scale=w.gamma,
                                 max_seq_len=inp.max_seq_len, with_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.decode_multi(q_lat, q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None, 4,
                                       -w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    assert_close(out, ref, "two tokens, sigma<0")
    assert_lse_close(lse, ref_lse, "two tokens, sigma<0 lse")


@pytest.mark.parametrize("B,heads", [(4, 64), (1, 64), (4, 128)])
def test_zero_scale_is_the_mean(B, heads):
    lens = [300, 1, 1000, 129]
    inp = inputs(lens, B=B, heads=heads, seed=85)
    w = inp.workload
    out, lse, ref, ref_lse = decode_both(inp, 0.0)
    c = inp.c_kv.double().numpy()
    d_blk = w.d_latent // B
    for s, L in enumerate(lens):
        rows = c[s * inp.max_seq_len: s * inp.max_seq_len + L]       # contiguous cache layout
        mean = w.gamma * rows.mean(axis=0)                          # [d_latent], branches side by side
        expect = np.broadcast_to(mean, (w.heads, w.d_latent))
        got = out[s].double().cpu().numpy()
        assert np.abs(got - expect).max() <= 1e-3 * max(np.abs(expect).max(), 1e-6), (s, L)
        assert np.allclose(lse[s].cpu().numpy(), np.log(L), atol=1e-4), (s, L)
    assert_close(out, ref, f"sigma=0 B={B}")
    assert_lse_close(lse, ref_lse, f"sigma=0 B={B} lse")
    assert d_blk * B == w.d_latent
