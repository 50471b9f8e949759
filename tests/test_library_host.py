"""The C-ABI library on the host: it loads, exports what include/mlra.h declares, and its
host-side logic (argument checks, workspace sizing, split plan) behaves.  No GPU needed; no
compute call is made."""
import ctypes
import pathlib
import random
import re

import pytest

from latent_kv_cache_mlra_b200 import mlra

HEADER = pathlib.Path(__file__).parents[1] / "include" / "mlra.h"


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(mlra_[a-z_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = mlra.lib()
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), f"{n} declared in mlra.h but not exported"
    assert set(names) == set(mlra.EXPORTS)
    assert lib.mlra_version() == 0x000100


def test_status_strings():
    for code in range(9):
        s = mlra.status_string(code)
        assert s.startswith("MLRA_")
    assert "unknown" in mlra.status_string(99)


def dims(**kw):
    base = dict(batch=8, heads=64, num_branches=4, d_latent=512, d_rope=64, max_seq_len=32768,
                cache_rows=8 * 32768, num_ranges=74)
    base.update(kw)
    return mlra.make_dims(**base)


def test_workspace_size_layout():
    # status 256 + plan scratch (5 N + 2 ints) + plan (a range record per range, a segment
    # descriptor per slot, a sequence record per sequence) + a status slot per CTA and one for
    # the prep kernel + (R + N - 1) slots of (m, l) and partial outputs
    n = mlra.workspace_size(dims())
    slots, H, B, dck, R, N = 74 + 8 - 1, 64, 4, 512, 74, 8
    plan = 4 * (5 * N + 2) + 8 * R + 16 * slots + 8 * N + 4 * (R * B + 1)
    expect_min = 256 + plan + slots * H * B * 2 * 4 + slots * H * dck * 4
    assert expect_min <= n <= expect_min + 8 * 256 + 64
    # fp32 input adds padded bf16 copies of queries and cache
    n32 = mlra.workspace_size(dims(dtype="f32"))
    assert n32 - n >= 8 * 32768 * (512 + 64) * 2
    # odd branch width -> padded copy too
    assert mlra.workspace_size(dims(batch=1, heads=8, d_latent=128, d_rope=16, max_seq_len=256,
                                    cache_rows=256)) > 256 * 64 * 4 * 2


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), mlra.MLRA_ERR_INVALID_ARG),
    (dict(heads=0), mlra.MLRA_ERR_INVALID_ARG),
    (dict(num_branches=3), mlra.MLRA_ERR_INVALID_ARG),          # 3 does not divide 512
    (dict(cache_rows=100), mlra.MLRA_ERR_INVALID_ARG),          # contiguous rows too few
    (dict(c_row_stride=100), mlra.MLRA_ERR_INVALID_ARG),        # stride below the width
    (dict(heads=129), mlra.MLRA_ERR_UNSUPPORTED),
    (dict(d_latent=1024, num_branches=8), mlra.MLRA_ERR_UNSUPPORTED),
    (dict(d_rope=128, kr_row_stride=128), mlra.MLRA_ERR_UNSUPPORTED),
    (dict(page_size=32, max_pages_per_seq=1024), mlra.MLRA_ERR_UNSUPPORTED),
    (dict(c_row_stride=516), mlra.MLRA_ERR_UNSUPPORTED),        # bf16 rows not 16-byte aligned
])
def test_workspace_size_rejects(kw, code):
    with pytest.raises(mlra.MlraError) as e:
        mlra.workspace_size(dims(**kw))
    assert e.value.status == code


def test_decode_argument_errors_before_any_launch():
    lib = mlra.lib()
    d = dims()
    sc = mlra.Scales(0.1, 0.25)
    fake = ctypes.c_void_p(256)
    args = [fake] * 5 + [None, 4, ctypes.byref(sc), fake, None, ctypes.byref(d), fake, 1 << 30, None]
    bad = list(args)
    bad[0] = None                                   # null q_lat
    assert lib.mlra_decode(*bad) == mlra.MLRA_ERR_INVALID_ARG
    bad = list(args)
    bad[6] = 2                                      # B != dims.num_branches
    assert lib.mlra_decode(*bad) == mlra.MLRA_ERR_INVALID_ARG
    nan = mlra.Scales(float("nan"), 0.25)
    bad = list(args)
    bad[7] = ctypes.byref(nan)
    assert lib.mlra_decode(*bad) == mlra.MLRA_ERR_INVALID_ARG
    bad = list(args)
    bad[12] = 16                                    # workspace too small
    assert lib.mlra_decode(*bad) == mlra.MLRA_ERR_WORKSPACE
    bad = list(args)
    bad[11] = ctypes.c_void_p(256 + 8)              # misaligned workspace
    assert lib.mlra_decode(*bad) == mlra.MLRA_ERR_WORKSPACE


def ranges_by_definition(tiles, R):
    """Per sequence, the set of ranges [floor(rT/R), floor((r+1)T/R)) it intersects, with R cut
    to the tile count T when T < R (no range may be empty)."""
    prefix = [0]
    for t in tiles:
        prefix.append(prefix[-1] + t)
    T = prefix[-1]
    R = min(R, max(T, 1))
    assert all((r + 1) * T // R > r * T // R for r in range(R))
    out = []
    for s in range(len(tiles)):
        a, b = prefix[s], prefix[s + 1]
        rs = [r for r in range(R) if max(a, r * T // R) < min(b, (r + 1) * T // R)]
        out.append(rs)
    return out


def cost_boundaries(tiles, R, cost):
    """Range starts of the cost-balanced plan, written from its definition: every non-empty
    sequence is `cost` virtual tiles followed by its real tiles; range r starts at virtual
    position floor(r V / R), mapped back to the real tile it falls on (a position among a
    sequence's leading cost tiles maps to the sequence's first tile)."""
    T = sum(tiles)
    R = min(R, max(T, 1))
    virtual = []  # real tile (or first tile of the sequence) of every virtual position
    g = 0
    for t in tiles:
        if t == 0:
            continue
        virtual += [g] * cost + list(range(g, g + t))
        g += t
    V = len(virtual)
    return [virtual[r * V // R] if r * V // R < V else T for r in range(R)] + [T]


@pytest.mark.parametrize("seed", range(12))
def test_plan_host_matches_definition(seed):
    rnd = random.Random(seed)
    n = rnd.randint(1, 40) if seed % 2 else rnd.randint(1, 4)
    tiles = [rnd.choice([0, 1, 2, 5, 17, 64, 513] if seed % 2 else [0, 1, 2, 5]) for _ in range(n)]
    if sum(tiles) == 0:
        tiles[0] = 3
    R = rnd.randint(1, 160)
    first, parts = mlra.plan_host(tiles, R)
    ref = ranges_by_definition(tiles, R)
    for s in range(n):
        assert parts[s] == len(ref[s]), (s, tiles, R)
        if ref[s]:
            assert ref[s] == list(range(first[s], first[s] + parts[s]))
    # partial slots r + s are unique and below R + N - 1
    slots = [r + s for s in range(n) for r in ref[s]]
    assert len(slots) == len(set(slots)) and max(slots) < R + n - 1
    # ranges are balanced to one tile and none is empty
    T = sum(tiles)
    Re = min(R, T)
    sizes = [(r + 1) * T // Re - r * T // Re for r in range(Re)]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_plan_fewer_tiles_than_ranges():
    # 2 tiles, 5 ranges: the old plan left range 3 empty between the two parts
    first, parts = mlra.plan_host([2], 5)
    assert (first, parts) == ([0], [2])
    first, parts = mlra.plan_host([0, 1, 0, 1], 100)
    assert parts == [0, 1, 0, 1] and first[1] != first[3]


@pytest.mark.parametrize("seed", range(12))
def test_segment_walk_covers_every_tile_once(seed):
    """The kernel's per-CTA walk (host replica): every tile of every sequence is visited by
    exactly one CTA, segments agree with the partial counts, CTAs past the effective number of
    ranges walk nothing."""
    rnd = random.Random(100 + seed)
    n = rnd.randint(1, 30)
    tiles = [rnd.choice([0, 0, 1, 2, 3, 9, 40, 300]) for _ in range(n)]
    R = rnd.choice([1, 2, 3, 7, 74, 148, 1000])
    segs = mlra.plan_segments_host(tiles, R)
    seen = {}
    for r, s, t0, nt in segs:
        assert nt >= 1 and 0 <= s < n and 0 <= t0 and t0 + nt <= tiles[s]
        for t in range(t0, t0 + nt):
            assert (s, t) not in seen
            seen[(s, t)] = r
    assert len(seen) == sum(tiles)
    T = sum(tiles)
    assert all(r < max(1, min(R, T)) for r, *_ in segs)
    if T:
        first, parts = mlra.plan_host(tiles, R)
        for s in range(n):
            rs = sorted({r for r, ss, *_ in segs if ss == s})
            assert len(rs) == parts[s] and (not rs or rs[0] == first[s])


@pytest.mark.parametrize("seed", range(16))
def test_cost_balanced_plan_matches_definition(seed):
    """The plan the kernels use (a cost of c tiles per sequence start) against its definition
    written out position by position; every tile is covered once, the ranges of a sequence are
    consecutive and non-empty, partial slots are unique."""
    rnd = random.Random(500 + seed)
    n = rnd.randint(1, 40)
    tiles = [rnd.choice([0, 1, 2, 3, 5, 9, 40, 256, 300]) for _ in range(n)]
    if sum(tiles) == 0:
        tiles[-1] = 7
    R = rnd.choice([1, 2, 3, 7, 37, 74, 148, 400])
    cost = rnd.choice([0, 1, 3, 8])
    bounds = cost_boundaries(tiles, R, cost)
    segs = mlra.plan_segments_host(tiles, R, cost)
    prefix = [0]
    for t in tiles:
        prefix.append(prefix[-1] + t)
    # every segment is the overlap of its range with its sequence
    expect = []
    for r in range(len(bounds) - 1):
        a, b = bounds[r], bounds[r + 1]
        for s in range(n):
            lo, hi = max(a, prefix[s]), min(b, prefix[s + 1])
            if lo < hi:
                expect.append((r, s, lo - prefix[s], hi - lo))
    assert segs == expect
    covered = sorted((s, t) for _, s, t0, nt in segs for t in range(t0, t0 + nt))
    assert covered == [(s, t) for s in range(n) for t in range(tiles[s])]
    first, parts = mlra.plan_host(tiles, R, cost)
    for s in range(n):
        rs = [r for r, ss, *_ in segs if ss == s]
        assert len(rs) == parts[s] and rs == list(range(first[s], first[s] + parts[s])) if rs else parts[s] == 0
    slots = [r + s for r, s, *_ in segs]
    assert len(slots) == len(set(slots)) and max(slots) < R + n - 1
    if cost == 0:
        assert bounds == [r * sum(tiles) // min(R, sum(tiles)) for r in range(min(R, sum(tiles)))] + [sum(tiles)]


def test_cost_balanced_plan_moves_work_off_sequence_starts():
    # 8 sequences of 256 tiles over 37 ranges: a range in which a sequence starts gets fewer tiles
    tiles, R, cost = [256] * 8, 37, 3
    segs = mlra.plan_segments_host(tiles, R, cost)
    per_range = {}
    for r, s, t0, nt in segs:
        per_range.setdefault(r, []).append((s, t0, nt))
    sizes = {r: sum(nt for _, _, nt in v) for r, v in per_range.items()}
    starts = {r: sum(1 for i, (s, t0, nt) in enumerate(v) if i > 0 and t0 == 0) for r, v in per_range.items()}
    plain = [r for r in sizes if starts[r] == 0 and r > 0]
    split = [r for r in sizes if starts[r] == 1]
    assert split and plain
    assert max(sizes[r] for r in split) <= min(sizes[r] for r in plain) - cost + 1


def test_plan_host_rejects():
    with pytest.raises(mlra.MlraError):
        mlra.plan_host([1, -1], 4)
    with pytest.raises(mlra.MlraError):
        mlra.plan_host([1, 2], 0)
    with pytest.raises(mlra.MlraError):
        mlra.plan_host([1, 2], 4, -1)


def test_project_argument_errors_without_a_gpu():
    """mlra_project checks its sizes and alignment before touching the device."""
    lib = mlra.lib()
    fake = ctypes.c_void_p(4096)
    ok = [fake, fake, fake, 8, 64, 512, 128, None, None]
    for i, v, want in [(0, None, mlra.MLRA_ERR_INVALID_ARG), (3, 0, mlra.MLRA_ERR_INVALID_ARG),
                       (4, 0, mlra.MLRA_ERR_INVALID_ARG), (5, 96, mlra.MLRA_ERR_UNSUPPORTED),
                       (5, 576, mlra.MLRA_ERR_UNSUPPORTED), (6, 100, mlra.MLRA_ERR_UNSUPPORTED),
                       (2, ctypes.c_void_p(4100), mlra.MLRA_ERR_UNSUPPORTED)]:
        args = list(ok)
        args[i] = v
        assert lib.mlra_project(*args) == want, (i, v)


def test_pack_wuv_argument_errors_without_a_gpu():
    lib = mlra.lib()
    fake = ctypes.c_void_p(4096)
    assert lib.mlra_pack_wuv(None, fake, 2, 512, 128, None) == mlra.MLRA_ERR_INVALID_ARG
    assert lib.mlra_pack_wuv(fake, fake, 2, 96, 128, None) == mlra.MLRA_ERR_UNSUPPORTED
    assert lib.mlra_pack_wuv(fake, fake, 2, 512, 100, None) == mlra.MLRA_ERR_UNSUPPORTED
    assert lib.mlra_pack_wuv(ctypes.c_void_p(4100), fake, 2, 512, 128, None) == mlra.MLRA_ERR_UNSUPPORTED


def test_rope_append_argument_errors_without_a_gpu():
    """mlra_rope_append checks its arguments (base, dims, dtype, alignment) before any launch."""
    lib = mlra.lib()
    fake = ctypes.c_void_p(4096)

    def call(dims, base=10000.0, **ptrs):
        a = dict(q_in=fake, kr=fake, c=fake, lens=fake, pt=None, ckv=fake, krc=fake, q_out=fake)
        a.update(ptrs)
        return lib.mlra_rope_append(a["q_in"], a["kr"], a["c"], a["lens"], a["pt"], ctypes.byref(dims),
                                    a["ckv"], a["krc"], a["q_out"], ctypes.c_double(base), None, None)

    good = dict(batch=2, heads=4, num_branches=1, d_latent=128, d_rope=64, max_seq_len=64,
                cache_rows=128)
    assert call(mlra.make_dims(**good), base=0.0) == mlra.MLRA_ERR_INVALID_ARG
    assert call(mlra.make_dims(**good), base=float("nan")) == mlra.MLRA_ERR_INVALID_ARG
    assert call(mlra.make_dims(**good), q_in=None) == mlra.MLRA_ERR_INVALID_ARG
    assert call(mlra.make_dims(**dict(good, d_rope=63))) == mlra.MLRA_ERR_UNSUPPORTED
    assert call(mlra.make_dims(**dict(good, dtype="f32"))) == mlra.MLRA_ERR_UNSUPPORTED
    assert call(mlra.make_dims(**dict(good, kr_row_stride=65))) == mlra.MLRA_ERR_UNSUPPORTED
    assert call(mlra.make_dims(**dict(good, d_latent=127))) == mlra.MLRA_ERR_UNSUPPORTED
    assert call(mlra.make_dims(**dict(good, c_row_stride=129))) == mlra.MLRA_ERR_UNSUPPORTED
    for name in ("q_in", "kr", "c", "q_out", "krc", "ckv"):
        assert call(mlra.make_dims(**good), **{name: ctypes.c_void_p(4104)}) == mlra.MLRA_ERR_UNSUPPORTED, name
    assert call(mlra.make_dims(**dict(good, cache_rows=100))) == mlra.MLRA_ERR_INVALID_ARG  # 2 x 64 rows


def test_head_groups_in_the_plan():
    """More than 64 heads: one CTA per (range, branch, 64-head group)."""
    info = mlra.query_plan(dims(heads=128, num_branches=1))
    assert info.ctas == info.num_ranges * 2
    info4 = mlra.query_plan(dims(heads=96, num_branches=4))
    assert info4.ctas == info4.num_ranges * 8
    assert mlra.query_plan(dims(heads=64, num_branches=4)).ctas == 74 * 4


def test_workspace_size_multi_covers_the_virtual_sequences():
    """q query tokens per sequence plan N * q virtual sequences of H rows (odd q, or shapes the
    two-token kernel does not take): the workspace equals that of a single-token call with N * q
    sequences.  An even q with 64 heads and 128-wide branches plans N * q / 2 units of two tokens
    (128 rows each): the workspace holds their partial results, R + N q / 2 - 1 slots of
    128 rows x d_c fp32 plus (m, l) per branch."""
    kw = dict(heads=64, num_branches=4, d_latent=512, d_rope=64, max_seq_len=4096,
              cache_rows=64 * 1024, page_size=64, max_pages_per_seq=64, num_ranges=37)
    d = mlra.make_dims(batch=8, **kw)
    for q in (1, 3):
        assert mlra.workspace_size_multi(d, q) == mlra.workspace_size(mlra.make_dims(batch=8 * q, **kw))
    kw2 = {**kw, "num_branches": 2}   # 256-wide branches: one token per CTA for any q
    d2 = mlra.make_dims(batch=8, **kw2)
    assert mlra.workspace_size_multi(d2, 2) == mlra.workspace_size(mlra.make_dims(batch=16, **kw2))
    for q in (2, 4):
        units = 8 * q // 2
        slots = 37 + units - 1
        need = slots * 128 * 512 * 4 + slots * 128 * 4 * 2 * 4
        got = mlra.workspace_size_multi(d, q)
        assert need <= got <= need + 64 * 1024
    with pytest.raises(mlra.MlraError):
        mlra.workspace_size_multi(d, 0)
