"""Checks that pin the CPU oracle to facts fixed outside of it.

Each ``pin_*`` takes the oracle module (so that the same checks can be run
against copies with a planted mistake, see test_oracle_mutants.py) and raises
AssertionError when the oracle disagrees.  None of them retypes the oracle's
formula: they compare it with an independent library routine (PyTorch's
scaled-dot-product attention, SciPy's logsumexp), with pure-Python brute force,
with closed forms, or with invariants.

Sources ("Multi-Head Low-Rank Attention", yunpan.plus page):
  * section 1.3: absorbed three-step decode equals attention with the
    decompressed keys/values;
  * section 2: the NoPE key is a sum of block projections;
  * section 3 / 3.1: per-branch attention with its own softmax, shared RoPE key,
    branch outputs summed;
  * section 3.3: the branch sum is scaled.
"""
from __future__ import annotations

import math
import pathlib

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

GOLDEN = pathlib.Path(__file__).parent / "golden"


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _one_seq(orc, q_lat, q_rope, c, kr, B, sigma, gamma, out_mode="branches"):
    out, lse = orc.decode(q_lat[None], q_rope[None], c, kr, [c.shape[0]], None, B, sigma, gamma,
                          max_seq_len=c.shape[0], out_mode=out_mode)
    return out[0], lse[0]


# --------------------------------------------------------------------------- explicit form
def explicit_mlra(q_nope, q_rope, c, kr, W_uk, W_uv, sigma, gamma):
    """Per-branch attention with decompressed keys/values (SDPA, float64).

    q_nope [H, B, d_h], q_rope [H, d_R], c [L, d_c], kr [L, d_R],
    W_uk / W_uv [H, B, d_h, d_blk].  Branch b keys: [W_uk[h,b] c_{j,b} ; k^R_j],
    values W_uv[h,b] c_{j,b}; the branch outputs are summed and scaled.
    """
    H, B, d_h, d_blk = W_uk.shape
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    y = torch.zeros(H, d_h, dtype=torch.float64)
    for b in range(B):
        cb = t(c[:, b * d_blk:(b + 1) * d_blk])                       # [L, d_blk]
        k_nope = torch.einsum("hkd,ld->hlk", t(W_uk[:, b]), cb)        # [H, L, d_h]
        v = torch.einsum("hkd,ld->hlk", t(W_uv[:, b]), cb)             # [H, L, d_h]
        k = torch.cat([k_nope, t(kr)[None].expand(H, -1, -1)], dim=-1)
        q = torch.cat([t(q_nope[:, b]), t(q_rope)], dim=-1)[:, None]   # [H, 1, d_h+d_R]
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], scale=sigma)[0, :, 0]
        y += o
    return (gamma * y).numpy()


def pin_absorbed_equals_explicit(orc, seed=0, H=6, B=4, d_blk=8, d_R=4, d_h=5, L=37):
    """Step 1 absorption + step 2 + step 3 (the oracle's ``project``) == explicit decompressed
    attention (section 1.3, 2, 3)."""
    rng = np.random.default_rng(seed)
    W_uk, W_uv = _rand(rng, H, B, d_h, d_blk), _rand(rng, H, B, d_h, d_blk)
    q_nope, q_rope = _rand(rng, H, B, d_h), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, B * d_blk), _rand(rng, L, d_R)
    sigma, gamma = 0.37, 1.0 / B
    ref = explicit_mlra(q_nope, q_rope, c, kr, W_uk, W_uv, sigma, gamma)
    q_lat = np.concatenate([np.einsum("hkd,hk->hd", W_uk[:, b], q_nope[:, b]) for b in range(B)], 1)
    out, _ = _one_seq(orc, q_lat, q_rope, c, kr, B, sigma, gamma)
    w_cat = np.concatenate([W_uv[:, b] for b in range(B)], axis=2)   # [H, d_h, d_c]
    y = orc.project(out[None], w_cat)[0]                             # step 3
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert err <= 1e-12, f"absorbed vs explicit rel err {err:.3e}"


def pin_summed_equals_explicit_shared_wuv(orc, seed=1, H=5, B=2, d_blk=6, d_R=4, d_h=3, L=29):
    """Summed output mode == explicit form when every branch shares W^UV (section 3.3 sum)."""
    rng = np.random.default_rng(seed)
    W_uk = _rand(rng, H, B, d_h, d_blk)
    W_uv = np.repeat(_rand(rng, H, 1, d_h, d_blk), B, axis=1)
    q_nope, q_rope = _rand(rng, H, B, d_h), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, B * d_blk), _rand(rng, L, d_R)
    sigma, gamma = 0.5, 1.0 / B
    ref = explicit_mlra(q_nope, q_rope, c, kr, W_uk, W_uv, sigma, gamma)
    q_lat = np.concatenate([np.einsum("hkd,hk->hd", W_uk[:, b], q_nope[:, b]) for b in range(B)], 1)
    out, _ = _one_seq(orc, q_lat, q_rope, c, kr, B, sigma, gamma, out_mode="summed")
    y = np.einsum("hkd,hd->hk", W_uv[:, 0], out)
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert err <= 1e-12, f"summed vs explicit rel err {err:.3e}"


def pin_b1_equals_mqa(orc, seed=2, H=8, d_c=16, d_R=8, L=50):
    """B=1 is MLA decode: MQA attention with key [c; k^R] and value c (section 1.3, step 2)."""
    rng = np.random.default_rng(seed)
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    sigma = 1 / math.sqrt(d_c + d_R)
    q = torch.from_numpy(np.concatenate([q_lat, q_rope], 1))[None, :, None]      # [1,H,1,D]
    k = torch.from_numpy(np.concatenate([c, kr], 1))[None, None].expand(1, H, L, -1)
    v = torch.from_numpy(c)[None, None].expand(1, H, L, -1)
    ref = F.scaled_dot_product_attention(q, k, v, scale=sigma)[0, :, 0].numpy()
    out, lse = _one_seq(orc, q_lat, q_rope, c, kr, 1, sigma, 1.0)
    assert np.abs(out - ref).max() <= 1e-12 * np.abs(ref).max(), "B=1 differs from MQA attention"
    scores = sigma * (np.concatenate([q_lat, q_rope], 1) @ np.concatenate([c, kr], 1).T)
    assert np.allclose(lse[:, 0], logsumexp(scores, axis=1), rtol=0, atol=1e-12), "lse"


def brute_force(q_lat, q_rope, c, kr, B, sigma, gamma):
    """Pure-Python loops, unshifted exp: for tiny inputs only."""
    H, d_c = len(q_lat), len(q_lat[0])
    d = d_c // B
    L = len(c)
    out = [[0.0] * d_c for _ in range(H)]
    lse = [[0.0] * B for _ in range(H)]
    for h in range(H):
        for b in range(B):
            w = []
            for j in range(L):
                s = 0.0
                for k in range(d):
                    s += q_lat[h][b * d + k] * c[j][b * d + k]
                for k in range(len(kr[j])):
                    s += q_rope[h][k] * kr[j][k]
                w.append(math.exp(sigma * s))
            z = sum(w)
            lse[h][b] = math.log(z)
            for i in range(d):
                out[h][b * d + i] = gamma * sum(w[j] * c[j][b * d + i] for j in range(L)) / z
    return np.array(out), np.array(lse)


def pin_brute_force(orc, seed=3):
    """Two-pass shifted softmax == unshifted brute force on tiny inputs, B in {1, 2, 4}."""
    rng = np.random.default_rng(seed)
    for B, H, d_c, d_R, L in [(1, 2, 4, 2, 5), (2, 3, 6, 2, 9), (4, 2, 8, 3, 13)]:
        q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
        c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
        ref, ref_lse = brute_force(q_lat.tolist(), q_rope.tolist(), c.tolist(), kr.tolist(), B, 0.7, 0.3)
        out, lse = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.7, 0.3)
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-13), f"brute force out B={B}"
        assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-13), f"brute force lse B={B}"


def pin_probabilities(orc, seed=4, H=7, B=4, d_c=32, d_R=8, L=40):
    """Each branch's weights are >= 0 and sum to 1 over positions (independent softmax, 3.1)."""
    rng = np.random.default_rng(seed)
    q_lat, q_rope = _rand(rng, H, d_c, scale=3), _rand(rng, H, d_R, scale=3)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    p = orc.branch_probabilities(q_lat, q_rope, c, kr, B, 0.9)
    assert p.shape == (B, H, L)
    assert (p >= 0).all()
    assert np.abs(p.sum(-1) - 1).max() <= 1e-13, "weights do not sum to one"
    # different branches see different blocks -> different weights
    assert np.abs(p[0] - p[1]).max() > 1e-3


def pin_closed_forms(orc, seed=5):
    """Special cases with closed-form results."""
    rng = np.random.default_rng(seed)
    H, B, d_c, d_R, gamma = 4, 4, 16, 4, 0.25
    d = d_c // B
    # one position: the output is gamma * c_0
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, 1, d_c), _rand(rng, 1, d_R)
    out, lse = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.8, gamma)
    assert np.allclose(out, gamma * np.broadcast_to(c[0], (H, d_c)), rtol=0, atol=1e-15), "L=1"
    scores0 = [[0.8 * (q_lat[h, b * d:(b + 1) * d] @ c[0, b * d:(b + 1) * d] + q_rope[h] @ kr[0])
                for b in range(B)] for h in range(H)]
    assert np.allclose(lse, scores0, rtol=0, atol=1e-13), "L=1 lse equals the single score"
    # zero queries: uniform weights, the output is gamma * mean_j c_j
    L = 23
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    out, lse = _one_seq(orc, np.zeros((H, d_c)), np.zeros((H, d_R)), c, kr, B, 0.8, gamma)
    assert np.allclose(out, gamma * c.mean(0)[None], rtol=0, atol=1e-14), "q=0 mean"
    assert np.allclose(lse, math.log(L), rtol=0, atol=1e-13), "q=0 lse = log L"
    # constant latent block: weights sum to one, so the output is gamma * const
    c = np.full((L, d_c), 1.5)
    out, _ = _one_seq(orc, _rand(rng, H, d_c), _rand(rng, H, d_R), c, kr, B, 0.8, gamma)
    assert np.allclose(out, gamma * 1.5, rtol=0, atol=1e-14), "constant c"
    # one dominant score (the RoPE term, shared by every branch): output ~ gamma * c_j*
    c = _rand(rng, L, d_c)
    kr = np.zeros((L, d_R))
    kr[11, 0] = 60.0
    q_rope = np.zeros((H, d_R))
    q_rope[:, 0] = 1.0
    out, _ = _one_seq(orc, _rand(rng, H, d_c, scale=0.1), q_rope, c, kr, B, 1.0, gamma)
    assert np.allclose(out, gamma * c[11][None], rtol=0, atol=1e-12), "spike"
    # huge common shift of every score changes nothing (max subtraction)
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    base, lb = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.8, gamma)
    kr2 = np.concatenate([kr, np.full((L, 1), 1000.0)], 1)
    qr2 = np.concatenate([q_rope, np.ones((H, 1))], 1)
    shifted, ls = _one_seq(orc, q_lat, qr2, c, kr2, B, 0.8, gamma)
    assert np.isfinite(shifted).all() and np.allclose(shifted, base, rtol=0, atol=1e-12), "shift"
    assert np.allclose(ls - lb, 800.0, rtol=0, atol=1e-9), "lse shifts by sigma * 1000"


def pin_scale_sign(orc, seed=13, H=4, B=4, d_c=16, d_R=4, L=21):
    """The softmax scale's sign: a negative scale equals the positive one applied to the negated
    query (both parts), output and log-sum-exp; a zero scale gives uniform weights (the mean of
    each branch block, lse = log L) whatever the query."""
    rng = np.random.default_rng(seed)
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    neg, lneg = _one_seq(orc, q_lat, q_rope, c, kr, B, -0.7, 0.5)
    flip, lflip = _one_seq(orc, -q_lat, -q_rope, c, kr, B, 0.7, 0.5)
    assert np.allclose(neg, flip, rtol=0, atol=1e-14), "negative scale = negated query"
    assert np.allclose(lneg, lflip, rtol=0, atol=1e-13), "negative scale lse"
    pos, _ = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.7, 0.5)
    assert not np.allclose(neg, pos, rtol=0, atol=1e-6), "the sign matters"
    zero, lz = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.0, 0.5)
    assert np.allclose(zero, 0.5 * c.mean(0)[None], rtol=0, atol=1e-14), "zero scale: mean"
    assert np.allclose(lz, math.log(L), rtol=0, atol=1e-13), "zero scale: lse = log L"


def pin_branch_independence(orc, seed=6, H=5, B=4, d_c=32, d_R=8, L=31):
    """Changing block b' of the latent leaves every other branch's output bit-identical."""
    rng = np.random.default_rng(seed)
    d = d_c // B
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    base, lb = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.6, 0.25)
    for bp in range(B):
        c2 = c.copy()
        c2[:, bp * d:(bp + 1) * d] = _rand(rng, L, d)
        out, l2 = _one_seq(orc, q_lat, q_rope, c2, kr, B, 0.6, 0.25)
        for b in range(B):
            same = np.array_equal(out[:, b * d:(b + 1) * d], base[:, b * d:(b + 1) * d])
            assert same == (b != bp), f"branch {b} after changing block {bp}"
            assert np.array_equal(l2[:, b], lb[:, b]) == (b != bp)
    # and the shared RoPE key moves every branch
    kr2 = kr.copy()
    kr2[3] += 1.0
    out, _ = _one_seq(orc, q_lat, q_rope, c, kr2, B, 0.6, 0.25)
    for b in range(B):
        assert not np.array_equal(out[:, b * d:(b + 1) * d], base[:, b * d:(b + 1) * d])


def pin_position_permutation(orc, seed=7, H=3, B=2, d_c=12, d_R=4, L=19):
    """Attention is a set function of the cached positions."""
    rng = np.random.default_rng(seed)
    q_lat, q_rope = _rand(rng, H, d_c), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, d_c), _rand(rng, L, d_R)
    perm = rng.permutation(L)
    a, la = _one_seq(orc, q_lat, q_rope, c, kr, B, 0.9, 0.5)
    b, lb = _one_seq(orc, q_lat, q_rope, c[perm], kr[perm], B, 0.9, 0.5)
    assert np.allclose(a, b, rtol=0, atol=1e-13) and np.allclose(la, lb, rtol=0, atol=1e-13)


def pin_batch_rows_and_paging(orc, seed=8):
    """Paged (shuffled pages) and contiguous layouts give identical results; empty sequence."""
    rng = np.random.default_rng(seed)
    N, H, B, d_c, d_R, P = 3, 4, 2, 8, 4, 4
    lens = [10, 0, 7]
    Lmax = 12
    q_lat, q_rope = _rand(rng, N, H, d_c), _rand(rng, N, H, d_R)
    c_cont, kr_cont = _rand(rng, N * Lmax, d_c), _rand(rng, N * Lmax, d_R)
    out_c, lse_c = orc.decode(q_lat, q_rope, c_cont, kr_cont, lens, None, B, 0.7, 0.5, max_seq_len=Lmax)
    # scatter the same rows into shuffled pages
    n_pages = 3 * (Lmax // P)
    perm = rng.permutation(n_pages)
    pt = np.full((N, Lmax // P), -1)
    c_pool, kr_pool = np.full((n_pages * P, d_c), np.nan), np.full((n_pages * P, d_R), np.nan)
    k = 0
    for s in range(N):
        for pg in range((lens[s] + P - 1) // P):
            pt[s, pg] = perm[k]
            k += 1
            for r in range(P):
                j = pg * P + r
                if j < lens[s]:
                    c_pool[pt[s, pg] * P + r] = c_cont[s * Lmax + j]
                    kr_pool[pt[s, pg] * P + r] = kr_cont[s * Lmax + j]
    out_p, lse_p = orc.decode(q_lat, q_rope, c_pool, kr_pool, lens, pt, B, 0.7, 0.5, page_size=P)
    assert np.array_equal(out_p, out_c) and np.array_equal(lse_p, lse_c), "paged != contiguous"
    assert (out_c[1] == 0).all() and np.isneginf(lse_c[1]).all(), "empty sequence"
    # each sequence alone equals its batch entry
    for s in (0, 2):
        o1, l1 = _one_seq(orc, q_lat[s], q_rope[s], c_cont[s * Lmax:s * Lmax + lens[s]],
                          kr_cont[s * Lmax:s * Lmax + lens[s]], B, 0.7, 0.5)
        assert np.array_equal(o1, out_c[s]) and np.array_equal(l1, lse_c[s])


# --------------------------------------------------------------------------- golden fixtures
def read_fixture(name):
    """Parse ``key = expression`` lines (``#`` comments) with math names available."""
    env = {k: getattr(math, k) for k in ("log", "exp", "sqrt", "inf")}
    vals = {}
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, expr = (x.strip() for x in line.split("=", 1))
        vals[key] = eval(expr, {"__builtins__": {}}, env)  # fixture text is ours and tiny
    return vals


def pin_golden_hand_worked(orc):
    """Hand-derived closed-form example (tests/golden/hand_worked_mlra2.txt)."""
    f = read_fixture("hand_worked_mlra2.txt")
    q_lat, q_rope = np.array(f["q_lat"], float), np.array(f["q_rope"], float)
    c, kr = np.array(f["c_kv"], float), np.array(f["k_rope"], float)
    for tag in ("a", "b"):
        sigma, gamma = f[f"sigma_{tag}"], f["gamma"]
        out, lse = _one_seq(orc, q_lat, q_rope, c, kr, 2, sigma, gamma)
        assert np.allclose(out, f[f"out_{tag}"], rtol=0, atol=1e-14), f"golden out {tag}"
        assert np.allclose(lse, f[f"lse_{tag}"], rtol=0, atol=1e-14), f"golden lse {tag}"
        summed, _ = _one_seq(orc, q_lat, q_rope, c, kr, 2, sigma, gamma, out_mode="summed")
        assert np.allclose(summed[:, 0], f[f"summed_{tag}"], rtol=0, atol=1e-14), f"golden sum {tag}"


def pin_golden_multi_token(orc):
    """Hand-derived example of two new tokens attending causally
    (tests/golden/hand_worked_multi_token.txt)."""
    f = read_fixture("hand_worked_multi_token.txt")
    c, kr = np.array(f["c_kv"], float), np.array(f["k_rope"], float)
    q_rope = np.array(f["q_rope"], float)[None, :, None, :]            # [1, q, 1, d_R]
    for tag in ("a", "b"):
        q_lat = np.array(f[f"q_lat_{tag}"], float)[None, :, None, :]    # [1, q, 1, d_c]
        out, lse = orc.decode_multi(q_lat, q_rope, c, kr, [c.shape[0]], None, 1, f["sigma"],
                                    f["gamma"], max_seq_len=c.shape[0])
        assert np.allclose(out[0, :, 0, 0], f[f"out_{tag}"], rtol=0, atol=1e-14), f"golden out {tag}"
        assert np.allclose(lse[0, :, 0, 0], f[f"lse_{tag}"], rtol=0, atol=1e-14), f"golden lse {tag}"


def pin_golden_rows(orc):
    """Hand-written page-resolution example (tests/golden/page_rows.txt)."""
    f = read_fixture("page_rows.txt")
    for s, L in enumerate(f["seq_lens"]):
        paged = orc.resolve_rows(L, s, f["page_table"], f["page_size"], 0).tolist()
        cont = orc.resolve_rows(L, s, None, 0, f["max_seq_len"]).tolist()
        assert paged == f["paged_rows"][s], f"paged rows of sequence {s}"
        assert cont == f["contiguous_rows"][s], f"contiguous rows of sequence {s}"


def pin_project_brute_force(orc, seed=9, N=2, H=3, B=2, d_blk=4, d_h=3):
    """Step 3 by plain loops: y[s,h,k] = sum_b sum_i W^UV_{h,b}[k,i] out[s,h,b*d_blk+i]; and with
    identity blocks (d_h = d_blk) y is the plain sum of the branch outputs (section 3.3)."""
    rng = np.random.default_rng(seed)
    out = _rand(rng, N, H, B * d_blk)
    w = _rand(rng, H, d_h, B * d_blk)
    y = orc.project(out, w)
    for s_ in range(N):
        for h in range(H):
            for k in range(d_h):
                acc = 0.0
                for b in range(B):
                    for i in range(d_blk):
                        acc += w[h, k, b * d_blk + i] * out[s_, h, b * d_blk + i]
                assert abs(y[s_, h, k] - acc) <= 1e-12 * (1 + abs(acc)), "project vs loops"
    eye = np.tile(np.eye(d_blk), (H, 1, B))                           # [H, d_blk, B*d_blk]
    y_eye = orc.project(out, eye)
    assert np.allclose(y_eye, out.reshape(N, H, B, d_blk).sum(axis=2), rtol=0, atol=1e-12), "identity"


def pin_absorb_equals_explicit(orc, seed=10, H=4, B=4, d_blk=8, d_R=4, d_h=6, L=23):
    """Step 1 (``absorb``: one query per head, W^UK of every branch side by side) -> step 2 ->
    step 3 == explicit attention whose branch-b keys are W^UK_{h,b} c_b (sections 1.3, 2, 3)."""
    rng = np.random.default_rng(seed)
    W_uk, W_uv = _rand(rng, H, B, d_h, d_blk), _rand(rng, H, B, d_h, d_blk)
    q_head, q_rope = _rand(rng, H, d_h), _rand(rng, H, d_R)
    c, kr = _rand(rng, L, B * d_blk), _rand(rng, L, d_R)
    sigma, gamma = 0.29, 1.0 / B
    ref = explicit_mlra(np.repeat(q_head[:, None], B, axis=1), q_rope, c, kr, W_uk, W_uv, sigma, gamma)
    w_uk = np.concatenate([W_uk[:, b] for b in range(B)], axis=2)    # [H, d_h, d_c]
    q_lat = orc.absorb(q_head[None], w_uk)[0]                         # step 1
    out, _ = _one_seq(orc, q_lat, q_rope, c, kr, B, sigma, gamma)
    y = orc.project(out[None], np.concatenate([W_uv[:, b] for b in range(B)], axis=2))[0]
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert err <= 1e-12, f"absorb -> decode -> project vs explicit rel err {err:.3e}"


def pin_rope(orc, seed=11):
    """RoPE: the identity at position 0, a rotation (norms kept), scores that depend on the
    relative position only, the closed forms of the first two pairs, and 2x2 rotations by loops."""
    rng = np.random.default_rng(seed)
    d, base = 8, 10000.0
    x = _rand(rng, 5, d)
    assert np.allclose(orc.rope(x, np.zeros(5), base), x, rtol=0, atol=1e-15), "position 0"
    pos = rng.integers(0, 100000, size=5).astype(np.float64)
    y = orc.rope(x, pos, base)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12), "norm"
    q, k = _rand(rng, d), _rand(rng, d)
    for m, n in [(7, 3), (1000, 12), (54321, 54300)]:
        lhs = orc.rope(q[None], [m], base)[0] @ orc.rope(k[None], [n], base)[0]
        rhs = orc.rope(q[None], [m - n], base)[0] @ k
        assert abs(lhs - rhs) <= 1e-9 * (1 + abs(rhs)), "relative position"
    for p_ in (0.5, 2.0, 31.0):
        e0 = orc.rope(np.array([[1.0, 0.0, 0.0, 1.0]]), [p_], base)[0]
        a1 = p_ * base ** -0.5
        want = [math.cos(p_), math.sin(p_), -math.sin(a1), math.cos(a1)]
        assert np.allclose(e0, want, rtol=0, atol=1e-13), "closed form"
    for r in range(5):
        for i in range(d // 2):
            a = pos[r] * base ** (-2.0 * i / d)
            rot = [x[r, 2 * i] * math.cos(a) - x[r, 2 * i + 1] * math.sin(a),
                   x[r, 2 * i] * math.sin(a) + x[r, 2 * i + 1] * math.cos(a)]
            assert abs(y[r, 2 * i] - rot[0]) + abs(y[r, 2 * i + 1] - rot[1]) <= 1e-9, "loops"


def pin_append_token(orc, seed=12):
    """The new token lands at position seq_lens[s] (the decode's row addressing), nothing else
    changes, and the decode then sees exactly one more position."""
    rng = np.random.default_rng(seed)
    N, d_c, d_R, P = 3, 8, 4, 64
    lens = np.array([5, 64, 0])
    pt = np.array([[3, 1], [0, 2], [4, 5]])                # pages of 64 rows
    rows = 6 * P
    c_kv, k_rope = _rand(rng, rows, d_c), _rand(rng, rows, d_R)
    c_new, kr_new = _rand(rng, N, d_c), _rand(rng, N, d_R)
    c2, k2, lens2 = orc.append_token(c_kv, k_rope, lens, pt, P, 0, c_new, kr_new)
    assert list(lens2) == [6, 65, 1]
    want_rows = [3 * P + 5, 2 * P + 0, 4 * P + 0]
    changed = sorted(set(np.nonzero((c2 != c_kv).any(1))[0]) | set(np.nonzero((k2 != k_rope).any(1))[0]))
    assert changed == sorted(want_rows), (changed, want_rows)
    for s_, r in enumerate(want_rows):
        assert np.array_equal(c2[r], c_new[s_]) and np.array_equal(k2[r], kr_new[s_])
    # contiguous layout: row s * max_seq_len + L
    c3, _, _ = orc.append_token(c_kv, k_rope, [2, 0, 7], None, 0, 10, c_new, kr_new)
    assert [r for r in range(rows) if (c3[r] != c_kv[r]).any()] == [2, 10, 27]


def explicit_mlra_causal(q_nope, q_rope, c, kr, W_uk, W_uv, sigma, gamma):
    """Like ``explicit_mlra`` for the q newest tokens of one sequence with a causal mask: query t
    (q_nope [q, H, B, d_h], q_rope [q, H, d_R]) sees keys 0 .. L - q + t.  The mask is built as a
    boolean matrix (the decode alignment is bottom-right, not SDPA's is_causal top-left)."""
    q_len = q_nope.shape[0]
    H, B, d_h, d_blk = W_uk.shape
    L = c.shape[0]
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    mask = torch.arange(L)[None, :] <= (L - q_len + torch.arange(q_len))[:, None]   # [q, L]
    y = torch.zeros(q_len, H, d_h, dtype=torch.float64)
    for b in range(B):
        cb = t(c[:, b * d_blk:(b + 1) * d_blk])
        k_nope = torch.einsum("hkd,ld->hlk", t(W_uk[:, b]), cb)            # [H, L, d_h]
        v = torch.einsum("hkd,ld->hlk", t(W_uv[:, b]), cb)
        k = torch.cat([k_nope, t(kr)[None].expand(H, -1, -1)], dim=-1)     # [H, L, d_h + d_R]
        qq = torch.cat([t(q_nope[:, :, b]), t(q_rope)], dim=-1).transpose(0, 1)  # [H, q, d_h+d_R]
        o = F.scaled_dot_product_attention(qq[None], k[None], v[None], attn_mask=mask, scale=sigma)[0]
        y += o.transpose(0, 1)                                               # [q, H, d_h]
    return (gamma * y).numpy()


def pin_multi_token_equals_explicit_causal(orc, seed=12, H=3, B=4, d_blk=8, d_R=4, d_h=5, L=29, q=3):
    """The q newest tokens (``decode_multi``) -> step 3 == explicit decompressed attention with a
    bottom-right causal mask; q = 1 is the single-token decode; a token ignores later positions."""
    rng = np.random.default_rng(seed)
    W_uk, W_uv = _rand(rng, H, B, d_h, d_blk), _rand(rng, H, B, d_h, d_blk)
    q_nope, q_rope = _rand(rng, q, H, B, d_h), _rand(rng, q, H, d_R)
    c, kr = _rand(rng, L, B * d_blk), _rand(rng, L, d_R)
    sigma, gamma = 0.31, 1.0 / B
    ref = explicit_mlra_causal(q_nope, q_rope, c, kr, W_uk, W_uv, sigma, gamma)
    q_lat = np.stack([np.concatenate([np.einsum("hkd,hk->hd", W_uk[:, b], q_nope[t, :, b])
                                      for b in range(B)], 1) for t in range(q)])  # [q, H, d_c]
    w_uv = np.concatenate([W_uv[:, b] for b in range(B)], axis=2)
    out, lse = orc.decode_multi(q_lat[None], q_rope[None], c, kr, [L], None, B, sigma, gamma,
                                max_seq_len=L)
    assert out.shape == (1, q, H, B * d_blk) and lse.shape == (1, q, H, B)
    y = orc.project(out[0], w_uv)
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert err <= 1e-12, f"multi-token vs explicit causal rel err {err:.3e}"
    one, _ = orc.decode_multi(q_lat[None, -1:], q_rope[None, -1:], c, kr, [L], None, B, sigma,
                              gamma, max_seq_len=L)
    single, _ = _one_seq(orc, q_lat[-1], q_rope[-1], c, kr, B, sigma, gamma)
    assert np.array_equal(one[0, 0], single), "q = 1 is the single-token decode"
    c2 = c.copy()
    c2[L - 1] += 5.0  # the last position: seen by the last token only
    out2, _ = orc.decode_multi(q_lat[None], q_rope[None], c2, kr, [L], None, B, sigma, gamma,
                               max_seq_len=L)
    assert np.array_equal(out2[0, :-1], out[0, :-1]), "earlier tokens ignore later positions"
    assert not np.allclose(out2[0, -1], out[0, -1]), "the last token sees its own position"


ALL_PINS = [
    pin_multi_token_equals_explicit_causal,
    pin_absorb_equals_explicit,
    pin_rope,
    pin_append_token,
    pin_project_brute_force,
    pin_absorbed_equals_explicit,
    pin_summed_equals_explicit_shared_wuv,
    pin_b1_equals_mqa,
    pin_brute_force,
    pin_probabilities,
    pin_closed_forms,
    pin_scale_sign,
    pin_branch_independence,
    pin_position_permutation,
    pin_batch_rows_and_paging,
    pin_golden_hand_worked,
    pin_golden_multi_token,
    pin_golden_rows,
]
