"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle, compare.

Tolerance (bf16 inputs, fp32 accumulation, bf16 probabilities in the output contraction):
  max |out - ref| <= 1e-2 * max |ref|   and   mean |out - ref| <= 2e-3.
lse: |lse - ref| <= 1e-3 + 1e-4 |ref| (scores are exact bf16 products summed in fp32).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
from latent_kv_cache_mlra_b200 import mlra

MAX_REL, MEAN_ABS = 1e-2, 2e-3


def to_dev(inp: workloads.Inputs, dev="cuda"):
    pt = None if inp.page_table is None else inp.page_table.to(dev)
    return (inp.q_lat.to(dev), inp.q_rope.to(dev), inp.c_kv.to(dev), inp.k_rope.to(dev),
            inp.seq_lens.to(dev), pt)


def poisoned_workspace(dims) -> torch.Tensor:
    """Workspace whose every byte is 0xFF (fp32 NaN): a partial slot the kernels read without
    having written it shows up as a non-finite output instead of hiding behind zeros."""
    return torch.full((mlra.workspace_size(dims),), 0xFF, dtype=torch.uint8, device="cuda")


def run_gpu(inp: workloads.Inputs, dev_tensors=None, **kw):
    w = inp.workload
    q, qr, c, kr, lens, pt = dev_tensors if dev_tensors is not None else to_dev(inp)
    dims = mlra.dims_for(q, qr, c, kr, lens, pt, w.num_branches, max_seq_len=inp.max_seq_len,
                         page_size=w.page_size, out_mode=kw.get("out_mode", "branches"),
                         num_ranges=kw.get("num_ranges", 0))
    out, lse = mlra.decode(q, qr, c, kr, lens, pt, num_branches=w.num_branches,
                           softmax_scale=w.sigma, branch_scale=w.gamma,
                           max_seq_len=inp.max_seq_len, page_size=w.page_size, with_lse=True,
                           workspace=poisoned_workspace(dims), **kw)
    torch.cuda.synchronize()
    return out, lse


def run_oracle(inp: workloads.Inputs, seqs=None, heads=None, out_mode="branches", f32_source=None):
    w = inp.workload
    src = f32_source if f32_source is not None else inp
    return oracle.decode(src.q_lat, src.q_rope, src.c_kv, src.k_rope, inp.seq_lens, inp.page_table,
                         w.num_branches, w.sigma, w.gamma, page_size=w.page_size,
                         max_seq_len=inp.max_seq_len, out_mode=out_mode, seqs=seqs, heads=heads)


def assert_close(out, ref, what=""):
    out = out.detach().cpu().double().numpy() if hasattr(out, "detach") else np.asarray(out)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref)
    scale = max(np.abs(ref).max(), 1e-30)
    assert err.max() <= MAX_REL * scale, f"{what}: max err {err.max():.3e} > {MAX_REL} * {scale:.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean err {err.mean():.3e}"
    return err.max() / scale, err.mean()


def assert_lse_close(lse, ref, what=""):
    lse = lse.detach().cpu().double().numpy()
    fin = np.isfinite(ref)
    assert (np.isneginf(lse) == np.isneginf(ref)).all(), f"{what}: -inf pattern"
    d = np.abs(lse[fin] - ref[fin])
    assert (d <= 1e-3 + 1e-4 * np.abs(ref[fin])).all(), f"{what}: lse err {d.max():.3e}"
