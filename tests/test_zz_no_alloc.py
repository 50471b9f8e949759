"""mlra_decode_static_scratch: the decode for callers that cannot give the library device memory.

Some hosts own every device allocation through their own pool and offer plug-ins no allocator;
some serving paths must not allocate at all.  This entry point takes no workspace and runs the
decode on a scratch array built into the library.  Called here through the C ABI, twice in a row
(the array keeps the previous call's contents), it must give what mlra_decode gives with a
caller workspace, within the parity tolerance of the GPU tests.  The file is named to run last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from latent_kv_cache_mlra_b200 import mlra

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_ABS = 1e-2, 2e-3


def _close(a, b):
    a, b = a.detach().cpu().double().numpy(), b.detach().cpu().double().numpy()
    err = np.abs(a - b)
    assert np.isfinite(a).all()
    assert err.max() <= MAX_REL * max(np.abs(b).max(), 1e-30) and err.mean() <= MEAN_ABS


def _call(lib, dev, w, dims, out, lse):
    scales = mlra.Scales(w.sigma, w.gamma)
    st = torch.cuda.current_stream().cuda_stream
    q, qr, c, kr, lens, pt = dev
    return lib.mlra_decode_static_scratch(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(qr.data_ptr()), ctypes.c_void_p(c.data_ptr()),
        ctypes.c_void_p(kr.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
        None if pt is None else ctypes.c_void_p(pt.data_ptr()), w.num_branches,
        ctypes.byref(scales), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.byref(dims), ctypes.c_void_p(st))


@pytest.mark.parametrize("paged", [False, True])
def test_static_scratch_matches_workspace_entry_point(paged):
    w = workloads.small(batch=5, seq_len=3000, ragged=True, min_seq_len=1,
                        page_size=64 if paged else 0, seed=31)
    inp = workloads.make_inputs(w)
    dev = [t.cuda() for t in (inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens)]
    dev.append(None if inp.page_table is None else inp.page_table.cuda())
    ref, ref_lse = mlra.decode(*dev, num_branches=w.num_branches, softmax_scale=w.sigma,
                               branch_scale=w.gamma, max_seq_len=inp.max_seq_len,
                               page_size=w.page_size, with_lse=True)
    dims = mlra.dims_for(*dev, w.num_branches, max_seq_len=inp.max_seq_len, page_size=w.page_size)
    lib = mlra.lib()
    for _ in range(2):  # two calls in a row share the built-in scratch
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _call(lib, dev, w, dims, out, lse) == mlra.MLRA_OK
        torch.cuda.synchronize()
        _close(out, ref)
        _close(lse, ref_lse)


def test_static_scratch_rejects_problems_beyond_its_size():
    # fp32 inputs need padded copies of the whole cache: far beyond the built-in scratch
    w = workloads.small(batch=8, seq_len=20000, dtype="f32", seed=3)
    dims = mlra.make_dims(batch=8, heads=64, num_branches=4, d_latent=512, d_rope=64,
                          max_seq_len=20000, cache_rows=8 * 20000, dtype="f32")
    lib = mlra.lib()
    q = torch.zeros(8, 64, 512, device="cuda")
    qr = torch.zeros(8, 64, 64, device="cuda")
    c = torch.zeros(8 * 20000, 512, device="cuda")
    kr = torch.zeros(8 * 20000, 64, device="cuda")
    lens = torch.full((8,), 100, dtype=torch.int32, device="cuda")
    out = torch.zeros(8, 64, 512, device="cuda")
    lse = torch.zeros(8, 64, 4, device="cuda")
    rc = _call(lib, (q, qr, c, kr, lens, None), w, dims, out, lse)
    assert rc == mlra.MLRA_ERR_SCRATCH_LIMIT
    assert "scratch" in mlra.status_string(rc)
