"""The static-group geometry the CUDA path's host code builds (temporal
groups and borrowed frames, passed to the window launches) against the
oracle's groups, over random geometries.  Host code only: the test hook
validates the geometry as stga_attn does and launches nothing (CPU only).
"""
import ctypes
import os
import re

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import stga as ostga
from sparse_attention_long_moga_b200 import _lib
from sparse_attention_long_moga_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def groups_fn():
    build()
    lib = _lib.load()
    fn = lib.moga_test_stga_groups
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.POINTER(_lib.StgaGeom), ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
    return lib, fn


def _geom(d):
    shots = (ctypes.c_int32 * len(d["shots"]))(*d["shots"])
    g = _lib.StgaGeom(d["T"], d["h"], d["w"], d["win_h"], d["win_w"], len(d["shots"]),
                      ctypes.cast(shots, ctypes.POINTER(ctypes.c_int32)), d["tg_max"], d["aug"])
    return g, shots


def _cuda_groups(fn, d):
    g, keep = _geom(d)
    cap = 512
    out = (ctypes.c_int32 * (4 * cap))()
    n = fn(ctypes.byref(g), out, cap)
    del keep
    return n, [tuple(out[4 * i:4 * i + 4]) for i in range(max(n, 0))]


def _oracle_groups(d):
    res = []
    for grp in ostga.temporal_groups(d["shots"], d["tg_max"]):
        kvf = ostga.kv_frames(grp, d["shots"], d["aug"])
        before = sum(1 for f in kvf if f < grp["t0"])
        after = sum(1 for f in kvf if f >= grp["t1"])
        res.append((grp["t0"], grp["t1"], before, after))
    return res


@st.composite
def geometries(draw):
    shots = draw(st.lists(st.integers(1, 40), min_size=1, max_size=12))
    return dict(T=sum(shots), h=draw(st.sampled_from([2, 4, 6])), w=draw(st.sampled_from([2, 3, 6])), win_h=2,
                win_w=1, shots=shots, tg_max=draw(st.integers(0, 9)),
                aug=draw(st.integers(0, 4)))


@settings(max_examples=300, deadline=None)
@given(geometries())
def test_host_temporal_groups_equal_oracle(groups_fn, d):
    _, fn = groups_fn
    n, got = _cuda_groups(fn, d)
    want = _oracle_groups(d)
    if len(want) > 256:          # more temporal groups than one launch takes: rejected
        assert n == -1
    else:
        assert n == len(want) and got == want


@pytest.mark.parametrize("shots,tg_max,aug", [((21,), 7, 2), ((14, 14, 13), 7, 2), ((37, 36, 36, 36, 36), 7, 2),
                                              ((37,) + (36,) * 9, 7, 2), ((4, 4), 0, 2), ((2, 1, 2), 2, 2)])
def test_host_temporal_groups_of_the_suite(groups_fn, shots, tg_max, aug):
    _, fn = groups_fn
    d = dict(T=sum(shots), h=30, w=52, win_h=15, win_w=26, shots=list(shots), tg_max=tg_max, aug=aug)
    n, got = _cuda_groups(fn, d)
    assert got == _oracle_groups(d)


def test_host_geometry_rejections(groups_fn):
    lib, fn = groups_fn
    base = dict(T=4, h=4, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=0, aug=2)
    assert _cuda_groups(fn, base)[0] == 2
    for bad in (dict(base, T=5), dict(base, win_h=3), dict(base, shots=[4, 0], T=4), dict(base, aug=-1),
                dict(base, tg_max=-1)):
        assert _cuda_groups(fn, bad)[0] == -1
    assert b"geometry" in lib.moga_last_error() or b"shot" in lib.moga_last_error()


def test_testing_header_symbols_are_exported(groups_fn):
    lib, _ = groups_fn
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moga_testing.h")).read(), flags=re.S)
    names = re.findall(r"^\s*(?:void|int32_t)\s+(\w+)\s*\(", text, flags=re.M)
    assert set(names) == {"moga_test_set_attn_debug", "moga_test_set_attn_events", "moga_test_stga_groups",
                          "moga_test_attn_tiles", "moga_test_window_tokens", "moga_test_bwd_units"}
    for name in names:
        assert hasattr(lib, name)
