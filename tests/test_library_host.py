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
    # status 256 + lens + prefix + plan (a range record per range, a segment descriptor per
    # slot, a sequence record per sequence) + (R + N - 1) slots of (m, l) and partial outputs
    n = mlra.workspace_size(dims())
    slots, H, B, dck, R, N = 74 + 8 - 1, 64, 4, 512, 74, 8
    plan = 8 * R + 16 * slots + 8 * N
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
    (dict(heads=65), mlra.MLRA_ERR_UNSUPPORTED),
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


def test_plan_host_rejects():
    with pytest.raises(mlra.MlraError):
        mlra.plan_host([1, -1], 4)
    with pytest.raises(mlra.MlraError):
        mlra.plan_host([1, 2], 0)
