"""CPU float64 oracle for MLRA single-token decode attention (step 2, absorbed form).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path and must never be used as a fallback for it.

What it computes (sources: "Multi-Head Low-Rank Attention", yunpan.plus page):
  * section 1.3, steps 1-3 of MLA's efficient decode: the absorbed query
    ``q~`` is dotted with the cached latent vectors directly, as MQA-style
    attention with the latent as the shared key/value, and the value
    up-projection comes afterwards (step 3: ``project`` below; step 1, the
    absorption, and the decoupled RoPE with the cache append: ``absorb``,
    ``rope`` and ``append_token`` below);
  * section 2: the per-head NoPE key is a sum of B block projections of the
    latent, so splitting ``c_t`` into B column blocks ``c_{t,b}`` is exact;
  * section 3 / 3.1 (MLRA-4): the block sum moves behind the attention; each
    branch b runs its own attention over its block with its own softmax over
    positions, and the RoPE key ``k^R_t`` is shared by all branches;
  * section 3.3: the sum of the branch outputs is scaled (``gamma``).

For sequence s, head h, branch b and position j < L_s (row(s, j) from the page
table or the contiguous layout):

    score[j] = sigma * ( q_lat[s,h,b-block] . c[row, b-block]  +  q_rope[s,h] . k_rope[row] )
    p        = softmax over j of score          (independent per branch)
    out[s,h,b-block] = gamma * sum_j p[j] * c[row, b-block]

Readings where the pages are silent: one RoPE query
per head shared by all branches; ``sigma`` and ``gamma`` are parameters; the
current token is already in the cache and no other mask applies; an empty
sequence gives a zero output and ``lse = -inf``; ``lse = log sum_j exp(score_j)``
per (s, h, b); "summed" output mode adds the B scaled branch outputs.

Every function below is written in float64 with NumPy; matrix products use
``numpy.matmul``.  Parity of the reconstructed MLRA-4 formula against the
published paper is unpinned (the equation is missing from the pages); the
oracle is pinned by the identities and closed forms in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

__all__ = ["resolve_rows", "decode", "decode_heads", "branch_probabilities", "to_f64"]


def to_f64(x) -> np.ndarray:
    """Convert a tensor/array to a float64 NumPy array (exact for bf16 and fp32)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def resolve_rows(seq_len: int, s: int, page_table, page_size: int, max_seq_len: int) -> np.ndarray:
    """Cache row of every position j < seq_len of sequence s.

    Contiguous layout (no page table): row = s * max_seq_len + j.
    Paged layout: row = page_table[s, j // P] * P + j % P.
    """
    j = np.arange(seq_len, dtype=np.int64)
    if page_table is None:
        return s * np.int64(max_seq_len) + j
    pt = np.asarray(page_table, dtype=np.int64)
    return pt[s, j // page_size] * page_size + j % page_size


def _rope_scores(q_rope_s: np.ndarray, kr: np.ndarray) -> np.ndarray:
    """Shared RoPE term q^R_h . k^R_j for all heads h and positions j: [H, L]."""
    return q_rope_s @ kr.T


def _branch_scores(q_blk: np.ndarray, c_blk: np.ndarray, rope: np.ndarray, sigma: float) -> np.ndarray:
    """sigma * (q~_{h,b} . c_{j,b} + q^R_h . k^R_j): [H, L]."""
    return sigma * (q_blk @ c_blk.T + rope)


def _softmax_positions(scores: np.ndarray):
    """Softmax over positions (last axis) with the row max subtracted; returns (p, lse)."""
    m = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - m)
    z = e.sum(axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def _apply_probs(p: np.ndarray, c_blk: np.ndarray) -> np.ndarray:
    """sum_j p[h, j] c_{j,b}: [H, d_blk]."""
    return p @ c_blk


def _gather(seq_len, s, c_kv, k_rope, page_table, page_size, max_seq_len):
    """The sequence's cache rows, converted to float64 after gathering (tensor or array)."""
    rows = resolve_rows(seq_len, s, page_table, page_size, max_seq_len)
    if hasattr(c_kv, "detach"):
        import torch
        idx = torch.from_numpy(rows)
        return to_f64(c_kv[idx]), to_f64(k_rope[idx])
    return to_f64(np.asarray(c_kv)[rows]), to_f64(np.asarray(k_rope)[rows])


def decode_heads(q_lat_s, q_rope_s, c_rows, kr_rows, num_branches, sigma, gamma,
                 out_mode="branches", with_probs=False):
    """Decode for one sequence whose cache rows are already gathered.

    q_lat_s [H', d_c], q_rope_s [H', d_R] (any subset of heads), c_rows [L, d_c],
    kr_rows [L, d_R].  Returns (out, lse[, probs]) with out [H', d_c] in
    "branches" mode or [H', d_blk] in "summed" mode, lse [H', B] and, on request,
    probs [B, H', L].
    """
    hq, d_c = q_lat_s.shape
    B = num_branches
    d = d_c // B
    L = c_rows.shape[0]
    if L == 0:
        out = np.zeros((hq, d_c if out_mode == "branches" else d))
        lse = np.full((hq, B), -np.inf)
        return (out, lse, np.zeros((B, hq, 0))) if with_probs else (out, lse)
    rope = _rope_scores(q_rope_s, kr_rows)
    outs, lses, probs = [], [], []
    for b in range(B):
        cols = slice(b * d, (b + 1) * d)
        scores = _branch_scores(q_lat_s[:, cols], c_rows[:, cols], rope, sigma)
        p, lse = _softmax_positions(scores)
        outs.append(gamma * _apply_probs(p, c_rows[:, cols]))
        lses.append(lse)
        probs.append(p)
    out = np.concatenate(outs, axis=1) if out_mode == "branches" else np.sum(outs, axis=0)
    lse = np.stack(lses, axis=1)
    return (out, lse, np.stack(probs)) if with_probs else (out, lse)


def decode(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches, sigma, gamma,
           page_size=0, max_seq_len=0, out_mode="branches", seqs=None, heads=None):
    """Decode attention for a batch.

    q_lat [N, H, d_c], q_rope [N, H, d_R], c_kv [rows, d_c], k_rope [rows, d_R],
    seq_lens [N], page_table [N, max_pages] or None.  ``seqs`` / ``heads`` pick a
    subset (default: all).  Returns (out [n, h, ...], lse [n, h, B]) in float64.
    """
    q_lat, q_rope = to_f64(q_lat), to_f64(q_rope)
    lens = np.asarray(seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens, dtype=np.int64)
    pt = None if page_table is None else np.asarray(
        page_table.tolist() if hasattr(page_table, "tolist") else page_table, dtype=np.int64)
    seqs = range(q_lat.shape[0]) if seqs is None else seqs
    heads = slice(None) if heads is None else heads
    outs, lses = [], []
    for s in seqs:
        c_rows, kr_rows = _gather(int(lens[s]), s, c_kv, k_rope, pt, page_size, max_seq_len)
        o, l = decode_heads(q_lat[s][heads], q_rope[s][heads], c_rows, kr_rows, num_branches,
                            sigma, gamma, out_mode)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def decode_multi(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches, sigma, gamma,
                 page_size=0, max_seq_len=0, out_mode="branches"):
    """Decode attention for the q newest tokens of every sequence at once (a speculative or
    chunked-prefill step; the absorbed step 2 of section 1.3 for each of them).

    q_lat [N, q, H, d_c], q_rope [N, q, H, d_R]: token t of sequence s is at position
    seq_lens[s] - q + t; all q tokens are already in the cache (seq_lens counts them).  Token t
    attends positions 0 .. seq_lens[s] - q + t (causal among the new tokens), i.e. it is the
    single-token decode with the length seq_lens[s] - (q - 1 - t) over the same cache rows.
    Returns (out [N, q, H, ...], lse [N, q, H, B]).
    """
    q_lat, q_rope = to_f64(q_lat), to_f64(q_rope)
    lens = np.asarray(seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens, dtype=np.int64)
    q = q_lat.shape[1]
    outs, lses = [], []
    for t in range(q):
        lens_t = np.maximum(lens - (q - 1 - t), 0)
        o, l = decode(q_lat[:, t], q_rope[:, t], c_kv, k_rope, lens_t, page_table, num_branches,
                      sigma, gamma, page_size=page_size, max_seq_len=max_seq_len,
                      out_mode=out_mode)
        outs.append(o)
        lses.append(l)
    return np.stack(outs, axis=1), np.stack(lses, axis=1)


def branch_probabilities(q_lat_s, q_rope_s, c_rows, kr_rows, num_branches, sigma):
    """Attention weights p[b, h, j] of one sequence (for the sum-to-one checks)."""
    _, _, probs = decode_heads(to_f64(q_lat_s), to_f64(q_rope_s), to_f64(c_rows), to_f64(kr_rows),
                               num_branches, sigma, 1.0, with_probs=True)
    return probs


def project(out, w_uv):
    """Step 3 of the absorbed decode (section 1.3; the branch sum of sections 3 and 3.3).

    out [N, H, d_c]: the branch-mode output of ``decode`` (gamma * o_b, branch b in columns
    b*d_blk .. (b+1)*d_blk).  w_uv [H, d_h, d_c]: head h's value up-projections side by side,
    W^UV_{h,b} = w_uv[h, :, b*d_blk:(b+1)*d_blk].  The per-branch projections summed over the
    branches are one product with the concatenation:

        y[s, h] = sum_b W^UV_{h,b} out[s, h, b-block] = w_uv[h] @ out[s, h]      -> [N, H, d_h]
    """
    return np.einsum("hkd,shd->shk", to_f64(w_uv), to_f64(out))


def absorb(q_nope, w_uk):
    """Step 1 of the absorbed decode (section 1.3): the query absorbs the key up-projections.

    q_nope [N, H, d_head]: each head's query before the keys' up-projection.  w_uk
    [H, d_head, d_c]: head h's key up-projections side by side, W^UK_{h,b} = w_uk[h, :, b-block],
    so that head h's key for branch b is W^UK_{h,b} c_b (section 2).  Then
        q_lat[s, h, b-block] = (W^UK_{h,b})^T q_nope[s, h]      -> [N, H, d_c]
    and q_lat[s, h, b-block] . c_b equals the head's query dotted with its branch-b key.
    """
    return np.einsum("hkd,shk->shd", to_f64(w_uk), to_f64(q_nope))


def rope(x, positions, base=10000.0):
    """Rotary position embedding of the decoupled RoPE vectors (the page's section on DeepSeek's
    decoupled RoPE; the rotation itself is the standard one, the pages give no variant).

    x [..., d] with d even; positions broadcast against x[..., 0].  Pair (2i, 2i+1) of a vector at
    position p is rotated by the angle p * base^(-2i/d):
        y[2i]   = x[2i] cos(a) - x[2i+1] sin(a)
        y[2i+1] = x[2i] sin(a) + x[2i+1] cos(a)
    """
    x = to_f64(x)
    d = x.shape[-1]
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    a = np.asarray(positions, dtype=np.float64)[..., None] * theta
    c, s_ = np.cos(a), np.sin(a)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s_
    y[..., 1::2] = x0 * s_ + x1 * c
    return y


def append_token(c_kv, k_rope, seq_lens, page_table, page_size, max_seq_len, c_new, kr_new):
    """The new token of every sequence goes into the cache at position p = seq_lens[s] (its
    row by the same addressing as the decode: page table or contiguous), latent c_new[s] and
    RoPE key kr_new[s] (already rotated).  Returns updated copies of (c_kv, k_rope) and the new
    lengths."""
    c_kv, k_rope = to_f64(c_kv).copy(), to_f64(k_rope).copy()
    lens = np.asarray(seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens, dtype=np.int64)
    pt = None if page_table is None else np.asarray(
        page_table.tolist() if hasattr(page_table, "tolist") else page_table, dtype=np.int64)
    c_new, kr_new = to_f64(c_new), to_f64(kr_new)
    for s in range(len(lens)):
        p = int(lens[s])
        row = int(resolve_rows(p + 1, s, pt, page_size, max_seq_len)[p])
        c_kv[row, :c_new.shape[1]] = c_new[s]
        k_rope[row, :kr_new.shape[1]] = kr_new[s]
    return c_kv, k_rope, lens + 1
