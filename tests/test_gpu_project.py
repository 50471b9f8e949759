"""Step 3 (mlra_project, through the C ABI) against the oracle's ``project``.

The kernel rounds o to bf16 before the tensor-core product (fp32 accumulation): against the oracle
on the same rounded o it agrees to accumulation order; against the unrounded o it stays within the
path's tolerance (max |err| <= 1e-2 max |ref|, mean |err| <= 2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import assert_close, run_gpu, to_dev
from tests.test_gpu_parity import small_inputs

pytestmark = pytest.mark.gpu


def rand_project(N, H, d_latent, d_head, seed):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(N, H, d_latent, generator=g) * 0.5
    w = (torch.randn(H, d_head, d_latent, generator=g) / d_latent ** 0.5).to(torch.bfloat16)
    return o, w


@pytest.mark.parametrize("N,H,d_latent,d_head", [
    (8, 64, 512, 128),     # the MLRA-4 / MLA decode shapes, d_h = 128
    (1, 3, 64, 64),        # one box of each
    (70, 5, 256, 192),     # two sequence tiles, three row tiles
    (130, 2, 512, 64),     # three sequence tiles, the last ragged
])
def test_project_matches_oracle(N, H, d_latent, d_head):
    o, w = rand_project(N, H, d_latent, d_head, seed=N + H)
    y = mlra.project(o.cuda(), mlra.pack_wuv(w.cuda()))
    torch.cuda.synchronize()
    ref_rounded = oracle.project(o.to(torch.bfloat16).float(), w.float())
    yd = y.cpu().double().numpy()
    err = np.abs(yd - ref_rounded).max() / np.abs(ref_rounded).max()
    assert err <= 1e-5, f"vs oracle on bf16-rounded o: rel {err:.2e}"
    assert_close(y, oracle.project(o, w.float()), f"N={N} H={H}")


def test_project_after_decode_matches_oracle():
    """decode -> project on the CUDA path against the oracle's decode -> project."""
    inp = small_inputs(lens=[300, 1, 129, 64], heads=8, seed=21)
    out, _ = run_gpu(inp)
    w = inp.workload
    g = torch.Generator().manual_seed(5)
    w_uv = (torch.randn(8, 128, w.d_latent, generator=g) / w.d_latent ** 0.5).to(torch.bfloat16)
    y = mlra.project(out.contiguous(), mlra.pack_wuv(w_uv.cuda()))
    ref_out, _ = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, None,
                               w.num_branches, w.sigma, w.gamma, max_seq_len=inp.max_seq_len)
    assert_close(y, oracle.project(ref_out, w_uv.float()), "decode + project")


def test_project_rejects():
    o = torch.zeros(2, 2, 96, device="cuda")
    w = torch.zeros(2, 64, 96, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(2, 2, 64, device="cuda")
    lib = mlra.lib()
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    args = [ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(y.data_ptr()),
            2, 2, 96, 64, None, ctypes.c_void_p(st)]
    assert lib.mlra_project(*args) == mlra.MLRA_ERR_UNSUPPORTED        # d_latent not a multiple of 64
    args[5], args[6] = 128, 96
    assert lib.mlra_project(*args) == mlra.MLRA_ERR_UNSUPPORTED        # d_head not a multiple of 64
    args[3] = 0
    assert lib.mlra_project(*args) == mlra.MLRA_ERR_INVALID_ARG


def test_pack_wuv_layout():
    """The packed image puts W[h, m*64 + r, kb*64 + 8j .. +7] at box (h*(d_head/64) + m)*KB + kb,
    row r, 16-byte chunk j ^ (r % 8) (the 128-byte swizzled K-major tensor-core layout)."""
    H, d_head, d_latent = 3, 128, 192
    w = torch.arange(H * d_head * d_latent, dtype=torch.float32).remainder(251).to(torch.bfloat16)
    w = w.view(H, d_head, d_latent).cuda()
    packed = mlra.pack_wuv(w).view(-1).cpu()
    wc = w.cpu()
    KB, mt = d_latent // 64, d_head // 64
    for (h, m, kb, r, j) in [(0, 0, 0, 0, 0), (2, 1, 2, 63, 7), (1, 0, 1, 5, 3), (1, 1, 0, 9, 6)]:
        box = (h * mt + m) * KB + kb
        pos = j ^ (r % 8)
        got = packed[box * 4096 + r * 64 + pos * 8: box * 4096 + r * 64 + pos * 8 + 8]
        want = wc[h, m * 64 + r, kb * 64 + 8 * j: kb * 64 + 8 * j + 8]
        assert torch.equal(got, want), (h, m, kb, r, j)


@pytest.mark.parametrize("B,d_latent,lens,page_size,num_ranges", [
    (4, 512, [300, 1, 65, 0, 1000, 63, 2049], 0, 0),    # splits, an empty sequence
    (1, 512, [129, 700, 5], 64, 0),                    # MLA, paged
    (2, 512, [3000, 17], 0, 9),                        # forced ranges: many parts
    (4, 256, [40] * 70, 64, 0),                        # more than 64 sequences: prep kernel
])
def test_decode_project_matches_oracle(B, d_latent, lens, page_size, num_ranges):
    """mlra_decode_project: the attention kernel, then step 3 merging the split sequences itself
    (no combine kernel), against the oracle's decode followed by its step 3."""
    inp = small_inputs(B=B, d_latent=d_latent, lens=lens, page_size=page_size, seed=23)
    w = inp.workload
    q, qr, c, kr, sl, pt = to_dev(inp)
    g = torch.Generator().manual_seed(24)
    w_uv = (torch.randn(w.heads, 128, d_latent, generator=g) / d_latent ** 0.5).to(torch.bfloat16)
    dims = mlra.dims_for(q, qr, c, kr, sl, pt, B, max_seq_len=inp.max_seq_len,
                         page_size=page_size, num_ranges=num_ranges)
    ws = torch.full((mlra.workspace_size_project(dims),), 0xFF, dtype=torch.uint8, device="cuda")
    y = mlra.decode_project(q, qr, c, kr, sl, pt, mlra.pack_wuv(w_uv.cuda()), num_branches=B,
                            softmax_scale=w.sigma, branch_scale=w.gamma,
                            max_seq_len=inp.max_seq_len, page_size=page_size,
                            num_ranges=num_ranges, workspace=ws)
    torch.cuda.synchronize()
    rc, flags = mlra.read_status(ws)
    assert rc == mlra.MLRA_OK, flags
    o, _ = oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, inp.page_table,
                         B, w.sigma, w.gamma, max_seq_len=inp.max_seq_len, page_size=page_size)
    assert_close(y, oracle.project(o, w_uv.float()), f"B={B} lens={len(lens)}")
