"""Seeded synthetic inputs for MLRA single-token decode attention.

This module only draws random numbers and lays them out.  It holds none of the
attention arithmetic, so that both the CPU oracle (``oracle/``) and the CUDA
path can take their inputs from it without sharing any computation.

Shapes follow the decode workloads of "Multi-Head Low-Rank Attention"
(yunpan.plus page, section 1.3 three-step decode and section 3.1 MLRA-4): a
latent cache ``c_kv`` of width ``d_c`` split into ``B`` branch blocks, a shared
RoPE key cache ``k_rope`` of width ``d_R``, and per-head absorbed queries
``q_lat`` (width ``d_c``) and RoPE queries ``q_rope`` (width ``d_R``).

Recipe (every workload):
  * one ``torch.Generator`` on the CPU, seeded with the workload's seed;
  * draws in this order: sequence lengths (serving mix only), ``q_lat``,
    ``q_rope``, ``c_kv``, ``k_rope``, page permutation (paged only);
  * every tensor is fp32 N(0, 1); ``c_kv`` is multiplied by the
    variance-matching factor ``alpha = sqrt(d_R / d_blk)`` (the pages ask for
    the latent state to be scaled so that the NoPE and RoPE score terms have
    matching variance, section 3.3; they print no number, so this is the
    plain reading for unit-variance inputs) and is then rounded;
  * bf16 workloads round to bf16 with round-to-nearest-even (``Tensor.to``);
  * the contiguous layout stores sequence ``s`` token ``j`` at cache row
    ``s * max_seq_len + j``; the paged layout stores it at row
    ``page_table[s, j // P] * P + j % P`` with the pages of all sequences
    drawn as one random permutation of the pool.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["Workload", "Inputs", "WORKLOADS", "get", "make_inputs", "small"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """A decode-attention problem: shapes, scales and the input recipe."""

    name: str
    batch: int
    heads: int
    num_branches: int
    d_latent: int
    d_rope: int
    seq_len: int                 # every sequence's length, or the upper bound when ``ragged``
    dtype: str = "bf16"          # "bf16" or "f32"
    page_size: int = 0           # 0: contiguous cache; else paged with this page size
    ragged: bool = False         # lengths log-uniform in [min_seq_len, seq_len]
    min_seq_len: int = 0
    seed: int = 0
    softmax_scale: Optional[float] = None   # default 1/sqrt(d_h + d_R), d_h = 128
    branch_scale: Optional[float] = None    # default 1/B
    alpha: Optional[float] = None           # default sqrt(d_R / d_blk)
    head_dim: int = 128                     # d_h of the explicit (decompressed) form

    @property
    def d_blk(self) -> int:
        return self.d_latent // self.num_branches

    @property
    def sigma(self) -> float:
        if self.softmax_scale is not None:
            return self.softmax_scale
        return 1.0 / math.sqrt(self.head_dim + self.d_rope)

    @property
    def gamma(self) -> float:
        return self.branch_scale if self.branch_scale is not None else 1.0 / self.num_branches

    @property
    def latent_scale(self) -> float:
        return self.alpha if self.alpha is not None else math.sqrt(self.d_rope / self.d_blk)


# The decode workloads.  Sizes are those of the MLRA decode study (Qwen3-32B-like
# heads: 64 query heads, latent 512, RoPE key 64, contexts up to 128k).
WORKLOADS = {
    "tiny_mlra4_f32": Workload(
        name="tiny_mlra4_f32", batch=1, heads=8, num_branches=4, d_latent=128, d_rope=16,
        seq_len=256, dtype="f32", seed=1001, softmax_scale=1.0 / math.sqrt(32 + 16),
        branch_scale=0.25, alpha=1.0),
    "mlra4_n8_l32k": Workload(
        name="mlra4_n8_l32k", batch=8, heads=64, num_branches=4, d_latent=512, d_rope=64,
        seq_len=32768, seed=1002),
    # Same cache bytes (same seed, same alpha) as mlra4_n8_l32k, read as one block.
    "mla_n8_l32k": Workload(
        name="mla_n8_l32k", batch=8, heads=64, num_branches=1, d_latent=512, d_rope=64,
        seq_len=32768, seed=1002, alpha=math.sqrt(64 / 128), branch_scale=1.0),
    "long_mlra4_l128k": Workload(
        name="long_mlra4_l128k", batch=1, heads=64, num_branches=4, d_latent=512, d_rope=64,
        seq_len=131072, seed=1004),
    "long_mlra2_l128k": Workload(
        name="long_mlra2_l128k", batch=1, heads=64, num_branches=2, d_latent=512, d_rope=64,
        seq_len=131072, seed=1004),
    # One device's share of mlra4_n8_l32k when the 4 branches sit on 4 devices (tensor
    # parallelism, one branch each): its 128-column latent block and the shared RoPE key, i.e.
    # d_R + d_c / 4 = 192 cached elements per token instead of 576.  Same scales as MLRA-4.
    "mlra4_tp4_shard_n8_l32k": Workload(
        name="mlra4_tp4_shard_n8_l32k", batch=8, heads=64, num_branches=1, d_latent=128,
        d_rope=64, seq_len=32768, seed=1006, alpha=math.sqrt(64 / 128), branch_scale=0.25),
    # MLA with 128 query heads (DeepSeek-V3-like attention: latent 512, RoPE key 64, head dim 128).
    "mla_h128_n8_l32k": Workload(
        name="mla_h128_n8_l32k", batch=8, heads=128, num_branches=1, d_latent=512, d_rope=64,
        seq_len=32768, seed=1007),
    # MLRA-4 with 128 heads (both head groups as one 128-row product per cache tile)
    "mlra4_h128_n8_l32k": Workload(
        name="mlra4_h128_n8_l32k", batch=8, heads=128, num_branches=4, d_latent=512, d_rope=64,
        seq_len=32768, seed=1008),
    "serving_mlra4_n64_paged": Workload(
        name="serving_mlra4_n64_paged", batch=64, heads=64, num_branches=4, d_latent=512,
        d_rope=64, seq_len=65536, min_seq_len=1024, ragged=True, page_size=64, seed=1005),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def small(name: str = "small", *, batch=3, heads=64, num_branches=4, d_latent=512, d_rope=64,
          seq_len=300, page_size=0, ragged=False, min_seq_len=1, seed=7, dtype="bf16",
          softmax_scale=None, branch_scale=None, alpha=None) -> Workload:
    """A workload small enough for the oracle to finish in well under a second."""
    return Workload(name=name, batch=batch, heads=heads, num_branches=num_branches,
                    d_latent=d_latent, d_rope=d_rope, seq_len=seq_len, dtype=dtype,
                    page_size=page_size, ragged=ragged, min_seq_len=min_seq_len, seed=seed,
                    softmax_scale=softmax_scale, branch_scale=branch_scale, alpha=alpha)


@dataclasses.dataclass
class Inputs:
    """Host tensors of one workload.  Floating tensors are in the workload dtype."""

    workload: Workload
    q_lat: torch.Tensor        # [N, H, d_c]
    q_rope: torch.Tensor       # [N, H, d_R]
    c_kv: torch.Tensor         # [rows, d_c]
    k_rope: torch.Tensor       # [rows, d_R]
    seq_lens: torch.Tensor     # int32 [N]
    page_table: Optional[torch.Tensor]  # int32 [N, max_pages] or None (contiguous)
    max_seq_len: int           # row pitch of the contiguous layout / bound on lengths

    @property
    def cache_rows(self) -> int:
        return int(self.c_kv.shape[0])

    @property
    def max_pages(self) -> int:
        return 0 if self.page_table is None else int(self.page_table.shape[1])


def draw_seq_lens(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """Per-sequence lengths: fixed, or round(exp(U[ln lo, ln hi])) when ragged."""
    if not w.ragged:
        return torch.full((w.batch,), w.seq_len, dtype=torch.int32)
    lo, hi = math.log(max(1, w.min_seq_len)), math.log(w.seq_len)
    u = torch.rand(w.batch, generator=gen, dtype=torch.float64)
    lens = torch.exp(lo + (hi - lo) * u).round().to(torch.int64)
    return lens.clamp(max(1, w.min_seq_len), w.seq_len).to(torch.int32)


def _round(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t.contiguous()


def make_inputs(w: Workload, *, seq_lens: Optional[torch.Tensor] = None,
                spare_pages: int = 3) -> Inputs:
    """Draw the inputs of ``w`` from its seed (see the module docstring)."""
    gen = torch.Generator().manual_seed(w.seed)
    lens = draw_seq_lens(w, gen) if seq_lens is None else seq_lens.to(torch.int32).clone()
    n, h = w.batch, w.heads
    q_lat = torch.randn(n, h, w.d_latent, generator=gen)
    q_rope = torch.randn(n, h, w.d_rope, generator=gen)
    if w.page_size == 0:
        max_len = int(max(w.seq_len, int(lens.max()) if n else 0))
        rows = n * max_len
        page_table = None
    else:
        p = w.page_size
        pages_per_seq = [(int(l) + p - 1) // p for l in lens.tolist()]
        max_pages = max([1] + [(w.seq_len + p - 1) // p])
        n_pages = sum(pages_per_seq) + spare_pages
        rows = n_pages * p
        max_len = max_pages * p
    c_kv = torch.randn(rows, w.d_latent, generator=gen)
    c_kv.mul_(w.latent_scale)
    k_rope = torch.randn(rows, w.d_rope, generator=gen)
    if w.page_size != 0:
        perm = torch.randperm(n_pages, generator=gen).to(torch.int32)
        page_table = torch.full((n, max_pages), -1, dtype=torch.int32)
        k = 0
        for s, np_s in enumerate(pages_per_seq):
            page_table[s, :np_s] = perm[k:k + np_s]
            k += np_s
    return Inputs(workload=w, q_lat=_round(q_lat, w.dtype), q_rope=_round(q_rope, w.dtype),
                  c_kv=_round(c_kv, w.dtype), k_rope=_round(k_rope, w.dtype), seq_lens=lens,
                  page_table=page_table, max_seq_len=max_len)
