"""Properties of the oracle's static groups over random geometries.

The readings of the pages (windows tile each frame without overlap; temporal
groups never cross a shot cut and split a shot into ceil(len / tg_max) runs
as equal as possible; a group touching a cut borrows, per side, the
min(aug, len) frames of the neighbouring shot nearest the cut, in the same
window, as keys/values only) imply invariants that any geometry must
satisfy.  Each is checked here from the token lists the oracle returns.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import stga as ostga


@st.composite
def geometries(draw):
    shots = draw(st.lists(st.integers(1, 6), min_size=1, max_size=4))
    win_h = draw(st.integers(1, 3))
    win_w = draw(st.integers(1, 3))
    return dict(T=sum(shots), h=win_h * draw(st.integers(1, 3)), w=win_w * draw(st.integers(1, 3)), win_h=win_h,
                win_w=win_w, shots=shots, tg_max=draw(st.integers(0, 4)), aug=draw(st.integers(0, 3)))


@settings(max_examples=150, deadline=None)
@given(geometries())
def test_window_groups_partition_queries_and_borrow_only_at_cuts(geom):
    T, h, w = geom["T"], geom["h"], geom["w"]
    hw = h * w
    shots = geom["shots"]
    starts = np.concatenate([[0], np.cumsum(shots)])
    shot_of = np.repeat(np.arange(len(shots)), shots)
    groups = ostga.window_groups(geom)
    n_win = (h // geom["win_h"]) * (w // geom["win_w"])
    runs = sum(1 if geom["tg_max"] == 0 else -(-L // geom["tg_max"]) for L in shots)
    assert len(groups) == n_win * runs
    seen = np.zeros(T * hw, dtype=np.int64)
    for q, kv in groups:
        seen[q] += 1
        qf, kf = q // hw, kv // hw
        # queries: one window, consecutive frames of one shot, at most tg_max of them
        assert len(set(shot_of[qf])) == 1
        frames = np.unique(qf)
        assert np.array_equal(frames, np.arange(frames[0], frames[-1] + 1))
        if geom["tg_max"]:
            assert len(frames) <= geom["tg_max"]
        pos = q % hw
        rows, cols = pos // w, pos % w
        assert len(set(rows // geom["win_h"])) == 1 and len(set(cols // geom["win_w"])) == 1
        # keys/values: the queries plus whole borrowed frames of the same window
        assert set(q).issubset(set(kv))
        extra = np.setdiff1d(np.unique(kf), frames)
        s = shot_of[frames[0]]
        before = [f for f in extra if f < frames[0]]
        after = [f for f in extra if f > frames[-1]]
        first, last = frames[0] == starts[s], frames[-1] + 1 == starts[s + 1]
        want_before = list(range(starts[s] - min(geom["aug"], shots[s - 1]), starts[s])) if first and s > 0 else []
        want_after = (list(range(starts[s + 1], starts[s + 1] + min(geom["aug"], shots[s + 1])))
                      if last and s + 1 < len(shots) else [])
        assert before == want_before and after == want_after
        assert len(kv) == (len(frames) + len(extra)) * geom["win_h"] * geom["win_w"]
        kpos = kv % hw
        assert set(kpos) == set(pos)
    # every token is a query of exactly one window group
    assert np.all(seen == 1)
    # run lengths of each shot differ by at most one, longer runs first
    for L in shots:
        r = ostga.split_runs(L, geom["tg_max"])
        assert sum(r) == L and max(r) - min(r) <= 1 and r == sorted(r, reverse=True)


@settings(max_examples=50, deadline=None)
@given(geometries())
def test_frame_groups_cover_each_frame_once(geom):
    hw = geom["h"] * geom["w"]
    groups = ostga.frame_groups(geom)
    assert len(groups) == geom["T"]
    allq = np.concatenate([q for q, _ in groups])
    assert np.array_equal(np.sort(allq), np.arange(geom["T"] * hw))
    for t, (q, kv) in enumerate(groups):
        assert np.array_equal(q, kv) and np.all(q // hw == t)
