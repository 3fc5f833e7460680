"""The work decomposition of the attention launches, decoded by the kernels'
own index code compiled for the host (test hooks of include/moga_testing.h),
against the oracle's groups (CPU only).

MoGA: tiles follow the groups largest first (ties by index), then head, then
pairs of 128-row query tiles, each tile's keys being its whole group; every
(head, row) is a query of exactly one tile.  Frames: every (head, token) once,
keys the token's frame.  Windows: mapped from the window-major index space to
tokens, each tile's queries lie in one oracle window group and its keys are
exactly that group's keys (borrowed frames included); every (head, token)
once.
"""
import ctypes

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import stga as ostga
from sparse_attention_long_moga_b200 import _lib
from sparse_attention_long_moga_b200.build import build

PAIR = 256
I32P = ctypes.POINTER(ctypes.c_int32)


@pytest.fixture(scope="module")
def hooks():
    build()
    lib = _lib.load()
    tiles = lib.moga_test_attn_tiles
    tiles.restype = ctypes.c_int32
    tiles.argtypes = [ctypes.c_int32, I32P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                      ctypes.POINTER(_lib.StgaGeom), I32P, ctypes.c_int32]
    wtok = lib.moga_test_window_tokens
    wtok.restype = ctypes.c_int32
    wtok.argtypes = [ctypes.POINTER(_lib.StgaGeom), ctypes.c_int32, ctypes.c_int32, I32P]
    return tiles, wtok


def _geom(d):
    shots = (ctypes.c_int32 * len(d["shots"]))(*d["shots"])
    g = _lib.StgaGeom(d["T"], d["h"], d["w"], d["win_h"], d["win_w"], len(d["shots"]), ctypes.cast(shots, I32P),
                      d["tg_max"], d["aug"])
    return g, shots


def _tiles(fn, mode, H, cu=None, N=0, geom=None):
    cu_arr = None if cu is None else (ctypes.c_int32 * len(cu))(*[int(c) for c in cu])
    g = keep = None
    if geom is not None:
        g, keep = _geom(geom)
    args = (mode, cu_arr, 0 if cu is None else len(cu) - 1, N, H, None if g is None else ctypes.byref(g))
    n = fn(*args, None, 0)
    assert n >= 0
    out = (ctypes.c_int32 * (5 * max(n, 1)))()
    assert fn(*args, out, n) == n
    del keep
    return np.frombuffer(out, dtype=np.int32)[:5 * n].reshape(n, 5)


def _window_tokens(fn, geom, N):
    g, keep = _geom(geom)
    out = (ctypes.c_int32 * N)()
    assert fn(ctypes.byref(g), 0, N, out) == N
    del keep
    return np.frombuffer(out, dtype=np.int32).copy()


@settings(max_examples=120, deadline=None)
@given(st.lists(st.integers(0, 900), min_size=1, max_size=32), st.integers(1, 4))
def test_moga_tiles_follow_groups_largest_first(hooks, sizes, H):
    fn, _ = hooks
    N = sum(sizes)
    if N == 0:
        return
    cu = np.concatenate([[0], np.cumsum(sizes)])
    got = _tiles(fn, 0, H, cu=cu, N=N)
    want = []
    for gi in sorted(range(len(sizes)), key=lambda i: (-sizes[i], i)):
        s, e = cu[gi], cu[gi + 1]
        for h in range(H):
            for q0 in range(s, e, PAIR):
                want.append((h, q0, min(e, q0 + PAIR), s, e))
    assert [tuple(r) for r in got] == want
    cover = np.zeros((H, N), dtype=np.int64)
    for h, q0, q1, _, _ in got:
        cover[h, q0:q1] += 1
    assert np.all(cover == 1)


@st.composite
def geometries(draw):
    shots = draw(st.lists(st.integers(1, 7), min_size=1, max_size=4))
    win_h, win_w = draw(st.integers(1, 4)), draw(st.integers(1, 6))
    return dict(T=sum(shots), h=win_h * draw(st.integers(1, 3)), w=win_w * draw(st.integers(1, 3)), win_h=win_h,
                win_w=win_w, shots=shots, tg_max=draw(st.integers(0, 4)), aug=draw(st.integers(0, 3)))


@settings(max_examples=120, deadline=None)
@given(geometries(), st.integers(1, 3))
def test_static_tiles_match_oracle_groups(hooks, geom, H):
    fn, wtok = hooks
    hw = geom["h"] * geom["w"]
    N = geom["T"] * hw
    # frames: every (head, token) once, keys = the token's frame
    cover = np.zeros((H, N), dtype=np.int64)
    for h, q0, q1, k0, k1 in _tiles(fn, 2, H, geom=geom):
        assert k0 % hw == 0 and k1 == k0 + hw and k0 <= q0 < q1 <= k1 and q1 - q0 <= PAIR
        cover[h, q0:q1] += 1
    assert np.all(cover == 1)
    # windows: the window-major order is a permutation of the tokens
    order = _window_tokens(wtok, geom, N)
    assert np.array_equal(np.sort(order), np.arange(N))
    groups = ostga.window_groups(geom)
    group_of = np.empty(N, dtype=np.int64)
    for i, (q, _) in enumerate(groups):
        group_of[q] = i
    cover[:] = 0
    for h, q0, q1, k0, k1 in _tiles(fn, 1, H, geom=geom):
        assert 0 < q1 - q0 <= PAIR
        qt, kt = order[q0:q1], order[k0:k1]
        gi = group_of[qt]
        assert np.all(gi == gi[0])
        assert np.array_equal(kt, groups[gi[0]][1])
        cover[h, qt] += 1
    assert np.all(cover == 1)


def test_suite_geometries(hooks):
    fn, wtok = hooks
    for geom, H in ((dict(T=21, h=30, w=52, win_h=15, win_w=26, shots=[21], tg_max=7, aug=2), 2),
                    (dict(T=41, h=30, w=52, win_h=15, win_w=26, shots=[14, 14, 13], tg_max=7, aug=2), 1)):
        N = geom["T"] * geom["h"] * geom["w"]
        order = _window_tokens(wtok, geom, N)
        groups = ostga.window_groups(geom)
        got = {(int(r[1]), int(r[2]), int(r[3]), int(r[4])) for r in _tiles(fn, 1, H, geom=geom) if r[0] == 0}
        ranges = {}
        for q0, q1, k0, k1 in got:
            ranges.setdefault((k0, k1), []).append((q0, q1))
        assert len(ranges) == len(groups)
        for (k0, k1), qs in ranges.items():
            kt = order[k0:k1]
            match = [g for g in groups if np.array_equal(g[1], kt)]
            assert len(match) == 1
            q_all = np.concatenate([order[a:b] for a, b in sorted(qs)])
            assert np.array_equal(q_all, match[0][0])


def test_hook_rejections(hooks):
    fn, wtok = hooks
    assert fn(7, None, 0, 0, 1, None, None, 0) == -1
    assert fn(0, None, 4, 100, 1, None, None, 0) == -1
    g, keep = _geom(dict(T=2, h=2, w=2, win_h=1, win_w=1, shots=[2], tg_max=0, aug=2))
    out = (ctypes.c_int32 * 8)()
    assert wtok(ctypes.byref(g), 0, 9, out) == -1
    assert wtok(ctypes.byref(g), 0, 8, out) == 8


@pytest.fixture(scope="module")
def bwd_hook(hooks):
    lib = _lib.load()
    fn = lib.moga_test_bwd_units
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_int32, ctypes.c_int32, I32P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                   ctypes.POINTER(_lib.StgaGeom), I32P, I32P, ctypes.c_int32]
    return fn, hooks[1]


def _units(fn, mode, keys, H, cu=None, N=0, geom=None):
    cu_arr = None if cu is None else (ctypes.c_int32 * len(cu))(*[int(c) for c in cu])
    g = keep = None
    if geom is not None:
        g, keep = _geom(geom)
    grid = ctypes.c_int32(0)
    args = (mode, keys, cu_arr, 0 if cu is None else len(cu) - 1, N, H, None if g is None else ctypes.byref(g),
            ctypes.byref(grid))
    n = fn(*args, None, 0)
    assert n >= 0
    out = (ctypes.c_int32 * (7 * max(n, 1)))()
    assert fn(*args, out, n) == n
    del keep
    return grid.value, np.frombuffer(out, dtype=np.int32)[:7 * n].reshape(n, 7)


@settings(max_examples=100, deadline=None)
@given(st.lists(st.integers(0, 700), min_size=1, max_size=32), st.integers(1, 3), st.booleans())
def test_moga_backward_units_cover_every_row_once(bwd_hook, sizes, H, keys):
    fn, _ = bwd_hook
    N = sum(sizes)
    if N == 0:
        return
    cu = np.concatenate([[0], np.cumsum(sizes)])
    grid, units = _units(fn, 0, int(keys), H, cu=cu, N=N)
    assert len(units) <= grid       # the launch's upper-bound grid reaches every tile
    cover = np.zeros((H, N), dtype=np.int64)
    seg = {(int(cu[i]), int(cu[i + 1])) for i in range(len(sizes)) if sizes[i]}
    for h, q0, q1, k0, k1, t0, t1 in units:
        assert (q0, q1) == (k0, k1) and (q0, q1) in seg
        assert q0 <= t0 < t1 <= q1 and t1 - t0 <= 128 and (t0 - q0) % 128 == 0
        cover[h, t0:t1] += 1
    assert np.all(cover == 1)


@settings(max_examples=80, deadline=None)
@given(geometries(), st.integers(1, 3))
def test_static_backward_units_match_oracle_groups(bwd_hook, geom, H):
    fn, wtok = bwd_hook
    hw = geom["h"] * geom["w"]
    N = geom["T"] * hw
    for keys in (0, 1):
        grid, units = _units(fn, 2, keys, H, geom=geom)
        assert len(units) == grid
        cover = np.zeros((H, N), dtype=np.int64)
        for h, q0, q1, k0, k1, t0, t1 in units:
            assert (q0, q1) == (k0, k1) and q0 % hw == 0 and q1 == q0 + hw and t1 - t0 <= 128
            cover[h, t0:t1] += 1
        assert np.all(cover == 1)
    order = _window_tokens(wtok, geom, N)
    groups = ostga.window_groups(geom)
    group_of = np.empty(N, dtype=np.int64)      # two groups may share their keys, never a query
    for i, (q, _) in enumerate(groups):
        group_of[q] = i
    # dQ: every (head, token) is a query of exactly one unit
    grid, units = _units(fn, 1, 0, H, geom=geom)
    assert len(units) == grid
    cover = np.zeros((H, N), dtype=np.int64)
    for h, q0, q1, k0, k1, t0, t1 in units:
        gi = group_of[order[q0]]
        assert np.array_equal(order[q0:q1], groups[gi][0]) and np.array_equal(order[k0:k1], groups[gi][1])
        assert q0 <= t0 < t1 <= q1 and t1 - t0 <= 128
        cover[h, order[t0:t1]] += 1
    assert np.all(cover == 1)
    # dK/dV: every key of every (group, head) in exactly one unit
    grid, units = _units(fn, 1, 1, H, geom=geom)
    assert len(units) == grid
    seen = {}
    for h, q0, q1, k0, k1, t0, t1 in units:
        gi = group_of[order[q0]]
        assert np.array_equal(order[q0:q1], groups[gi][0]) and np.array_equal(order[k0:k1], groups[gi][1])
        assert k0 <= t0 < t1 <= k1 and t1 - t0 <= 128
        seen.setdefault((gi, int(h)), []).append((int(t0 - k0), int(t1 - k0)))
    assert len(seen) == len(groups) * H
    for (gi, h), parts in seen.items():
        n_kv = len(groups[gi][1])
        c = np.zeros(n_kv, dtype=np.int64)
        for a, b in parts:
            c[a:b] += 1
        assert np.all(c == 1)
