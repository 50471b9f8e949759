"""The bounded-wait time-out path of the attention kernels, run for real.

Every wait inside the attention kernels gives up after a time limit: the waiting warp sets the
time-out bit in the call's status word and raises its CTA's abort flag, the other warps leave
their loops, the producer waits (bounded) for the copies it already issued, the issuers wait for
their tensor-core products, and TMEM is released.  The environment variable
MLRA_TEST_FORCE_TIMEOUT makes each CTA's producer wait, with a 1 ms limit, on a barrier nothing
arrives at, just before it would issue its first non-speculative copy; the calls use 3 work
ranges so that every CTA has copies left after its speculative ones.  A forced call must report
MLRA_ERR_TIMEOUT with the time-out bit, and must leave the context usable: the next call on the
same workspace reports success and returns bit for bit the result of a call made before."""
import pytest
import torch

import workloads
from latent_kv_cache_mlra_b200 import mlra
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu

HOOK = "MLRA_TEST_FORCE_TIMEOUT"
RANGES = 3


def inputs(lens, B=4, heads=64, page_size=0, seed=71):
    w = workloads.small(batch=len(lens), heads=heads, num_branches=B, d_latent=512, d_rope=64,
                        seq_len=max(lens), page_size=page_size, seed=seed)
    return workloads.make_inputs(w, seq_lens=torch.tensor(lens, dtype=torch.int32))


def forced_then_normal(call, workspace, monkeypatch):
    base = [t.clone() for t in call()]
    assert mlra.read_status(workspace) == (mlra.MLRA_OK, 0)
    monkeypatch.setenv(HOOK, "1")
    try:
        call()
        rc, flags = mlra.read_status(workspace)
    finally:
        monkeypatch.delenv(HOOK)
    assert rc == mlra.MLRA_ERR_TIMEOUT and flags & mlra.FLAG_TIMEOUT, (rc, flags)
    again = call()
    assert mlra.read_status(workspace) == (mlra.MLRA_OK, 0)
    for a, b in zip(again, base):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,lens,page_size", [
    (4, [2000, 700, 1300], 0),        # 128-column branch blocks, in-kernel plan
    (4, [1500, 1, 900], 64),          # ... paged
    (2, [1800, 640], 0),              # 256-column blocks
    (1, [1200, 300], 0),              # MLA: 512 columns, 64-position tiles
    (8, [1000, 2000], 0),             # 64-column blocks
    (4, [400] * 70, 0),               # more sequences than the in-kernel plan takes: prep kernel
])
def test_decode_timeout_path(B, lens, page_size, monkeypatch):
    inp = inputs(lens, B=B, page_size=page_size)
    w = inp.workload
    q, qr, c, kr, sl, pt = to_dev(inp)
    dims = mlra.dims_for(q, qr, c, kr, sl, pt, B, max_seq_len=inp.max_seq_len, page_size=page_size,
                         num_ranges=RANGES)
    ws = torch.zeros(mlra.workspace_size(dims), dtype=torch.uint8, device="cuda")

    def call():
        out, lse = mlra.decode(q, qr, c, kr, sl, pt, num_branches=B, softmax_scale=w.sigma,
                               branch_scale=w.gamma, max_seq_len=inp.max_seq_len,
                               page_size=page_size, with_lse=True, workspace=ws,
                               num_ranges=RANGES)
        return out, lse

    forced_then_normal(call, ws, monkeypatch)


@pytest.mark.parametrize("q_len,heads,lens", [
    (2, 64, [2000, 1000, 600]),       # two query tokens per CTA (128-row products)
    (1, 128, [1500, 900]),            # 128 heads in one CTA
])
def test_m128_timeout_path(q_len, heads, lens, monkeypatch):
    inp = inputs(lens, heads=heads, seed=73)
    w = inp.workload
    g = torch.Generator().manual_seed(74)
    q_lat = torch.randn(len(lens), q_len, heads, 512, generator=g).to(torch.bfloat16).cuda()
    q_rope = torch.randn(len(lens), q_len, heads, 64, generator=g).to(torch.bfloat16).cuda()
    _, _, c, kr, sl, _ = to_dev(inp)
    dims = mlra.dims_for(q_lat[:, 0], q_rope[:, 0], c, kr, sl, None, 4, max_seq_len=inp.max_seq_len,
                         num_ranges=RANGES)
    if q_len == 1:
        info = mlra.query_plan(dims)
        assert info.ctas == 4 * info.num_ranges      # one CTA per (range, branch): all 128 heads
        ws = torch.zeros(mlra.workspace_size(dims), dtype=torch.uint8, device="cuda")

        def call():
            return mlra.decode(q_lat[:, 0], q_rope[:, 0], c, kr, sl, None, num_branches=4,
                               softmax_scale=w.sigma, branch_scale=w.gamma,
                               max_seq_len=inp.max_seq_len, with_lse=True, workspace=ws,
                               num_ranges=RANGES)
    else:
        ws = torch.zeros(mlra.workspace_size_multi(dims, q_len), dtype=torch.uint8, device="cuda")

        def call():
            return mlra.decode_multi(q_lat, q_rope, c, kr, sl, None, num_branches=4,
                                     softmax_scale=w.sigma, branch_scale=w.gamma,
                                     max_seq_len=inp.max_seq_len, with_lse=True, workspace=ws,
                               num_ranges=RANGES)

    forced_then_normal(call, ws, monkeypatch)


def test_decode_project_timeout_path(monkeypatch):
    """Steps 2 and 3 in one call: the step-3 product folds the attention CTAs' status bits into the
    call's status word, so a time-out inside the attention kernel reaches the caller there too."""
    inp = inputs([2000, 700, 1300], seed=75)
    w = inp.workload
    q, qr, c, kr, sl, pt = to_dev(inp)
    g = torch.Generator().manual_seed(76)
    w_uv = (torch.randn(w.heads, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16).cuda()
    wp = mlra.pack_wuv(w_uv)
    dims = mlra.dims_for(q, qr, c, kr, sl, pt, 4, max_seq_len=inp.max_seq_len, num_ranges=RANGES)
    ws = torch.zeros(mlra.workspace_size_project(dims), dtype=torch.uint8, device="cuda")

    def call():
        return (mlra.decode_project(q, qr, c, kr, sl, pt, wp, num_branches=4, softmax_scale=w.sigma,
                                    branch_scale=w.gamma, max_seq_len=inp.max_seq_len,
                                    num_ranges=RANGES, workspace=ws),)

    forced_then_normal(call, ws, monkeypatch)
