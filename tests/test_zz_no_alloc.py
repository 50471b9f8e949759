"""mlra_decode_static_scratch: the decode for callers that cannot give the library device memory.

Some hosts own every device allocation through their own pool and offer plug-ins no allocator;
some serving paths must not allocate at all.  This entry point takes no workspace and runs the
decode on a scratch array built into the library, which every call shares and which keeps the
previous call's contents.

Called here through the C ABI several times in a row with problems of different shapes (a small
contiguous batch planned inside the attention kernel, then 80 ragged paged sequences planned by
the prep kernel, then the first problem again over the scratch the second one left), each result
must match the CPU oracle within the parity tolerance of the GPU tests, and also what mlra_decode
gives with a caller workspace.  The file is named to run last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from latent_kv_cache_mlra_b200 import mlra

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_ABS = 1e-2, 2e-3


def _close(a, b, what):
    a = a.detach().cpu().double().numpy() if hasattr(a, "detach") else np.asarray(a)
    b = b.detach().cpu().double().numpy() if hasattr(b, "detach") else np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    assert np.isfinite(a).all(), f"{what}: non-finite output"
    err = np.abs(a - b)
    assert err.max() <= MAX_REL * max(np.abs(b).max(), 1e-30), f"{what}: max err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean err {err.mean():.3e}"


def _lse_close(a, b, what):
    a = a.detach().cpu().double().numpy()
    b = b.detach().cpu().double().numpy() if hasattr(b, "detach") else np.asarray(b)
    fin = np.isfinite(b)
    assert (np.isneginf(a) == np.isneginf(b)).all(), f"{what}: -inf pattern"
    assert (np.abs(a[fin] - b[fin]) <= 1e-3 + 1e-4 * np.abs(b[fin])).all(), what


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


class _Problem:
    """One decode problem: device inputs, the oracle's answer and mlra_decode's answer."""

    def __init__(self, w, seq_lens=None):
        self.w = w
        inp = workloads.make_inputs(w, seq_lens=seq_lens)
        self.inp = inp
        self.dev = [t.cuda() for t in (inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens)]
        self.dev.append(None if inp.page_table is None else inp.page_table.cuda())
        self.ref, self.ref_lse = oracle.decode(
            inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, inp.page_table,
            w.num_branches, w.sigma, w.gamma, page_size=w.page_size, max_seq_len=inp.max_seq_len)
        self.ws_out, self.ws_lse = mlra.decode(
            *self.dev, num_branches=w.num_branches, softmax_scale=w.sigma, branch_scale=w.gamma,
            max_seq_len=inp.max_seq_len, page_size=w.page_size, with_lse=True)
        self.dims = mlra.dims_for(*self.dev, w.num_branches, max_seq_len=inp.max_seq_len,
                                  page_size=w.page_size)

    def check(self, lib, what):
        out = torch.full_like(self.ws_out, float("nan"))
        lse = torch.full_like(self.ws_lse, float("nan"))
        assert _call(lib, self.dev, self.w, self.dims, out, lse) == mlra.MLRA_OK
        torch.cuda.synchronize()
        _close(out, self.ref, f"{what} vs oracle")
        _lse_close(lse, self.ref_lse, f"{what} lse vs oracle")
        _close(out, self.ws_out, f"{what} vs mlra_decode")
        _lse_close(lse, self.ws_lse, f"{what} lse vs mlra_decode")


def test_static_scratch_consecutive_calls_of_different_shapes():
    small = _Problem(workloads.small(batch=5, seq_len=3000, ragged=True, min_seq_len=1, seed=31))
    # more than 64 sequences: the prep kernel plans the call; paged, ragged, one empty sequence
    lens = workloads.draw_seq_lens(
        workloads.small(batch=80, seq_len=900, ragged=True, min_seq_len=1, seed=32),
        torch.Generator().manual_seed(32))
    lens[17] = 0
    big = _Problem(workloads.small(batch=80, seq_len=900, ragged=True, min_seq_len=1,
                                   page_size=64, seed=33), seq_lens=lens)
    assert mlra.query_plan(big.dims).launches == 3  # prep kernel in the call

    lib = mlra.lib()
    small.check(lib, "first call (5 contiguous sequences)")
    big.check(lib, "second call (80 paged sequences)")
    small.check(lib, "third call (the first problem again)")


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
