"""CPU checks of the stratified row sampler and of the sampled branch rows.

The sampled-row form must give exactly the rows of the oracle's whole-layer
branches (it only restricts which rows are computed), and the sample must hit
every stratum it promises: every MoGA group with its first and last member,
every window group, one token per window in each frame within `aug` frames of
a cut, and every frame.
"""
import numpy as np

from oracle import attention as oatt
from oracle import sample as osample
from oracle import stga as ostga
from synth import workloads as W

GEOMS = [
    dict(T=6, h=6, w=10, win_h=3, win_w=5, shots=[2, 3, 1], tg_max=2, aug=2),
    dict(T=9, h=4, w=8, win_h=2, win_w=4, shots=[4, 5], tg_max=3, aug=1),
    dict(T=5, h=4, w=4, win_h=4, win_w=4, shots=[5], tg_max=0, aug=2),
]


def test_sample_heads_spread():
    assert osample.sample_heads(40, 8) == [0, 6, 11, 17, 22, 28, 33, 39]
    assert osample.sample_heads(12, 8)[0] == 0 and osample.sample_heads(12, 8)[-1] == 11
    assert osample.sample_heads(2, 8) == [0, 1]
    assert osample.sample_heads(1, 8) == [0]


def test_strata_covered():
    rs = np.random.default_rng(3)
    for geom in GEOMS:
        N = geom["T"] * geom["h"] * geom["w"]
        hw = geom["h"] * geom["w"]
        M = 5
        g = rs.integers(0, M, N)
        g[:7] = 4        # one small group
        for per_head in (16, 200):
            toks = osample.stratified_tokens(geom, g, M, np.random.default_rng(per_head), per_head=per_head)
            assert np.all(np.diff(toks) > 0)
            s = set(toks.tolist())
            for i in range(M):
                mem = np.nonzero(g == i)[0]
                if len(mem):
                    assert mem[0] in s and mem[-1] in s
            for qt, _ in ostga.window_groups(geom):
                assert s & set(qt.tolist())
            assert set(t // hw for t in s) == set(range(geom["T"]))
            cuts = np.cumsum(geom["shots"])[:-1]
            for c in cuts.tolist():
                for f in range(max(c - geom["aug"], 0), min(c + geom["aug"], geom["T"])):
                    for y0 in range(0, geom["h"], geom["win_h"]):
                        for x0 in range(0, geom["w"], geom["win_w"]):
                            win = ostga.window_tokens([f], y0, x0, geom["win_h"], geom["win_w"], geom["h"],
                                                      geom["w"])
                            assert s & set(win.tolist())
            if per_head == 200:
                assert len(toks) >= min(200, N)


def test_branch_rows_equal_whole_branches():
    rs = np.random.default_rng(7)
    for geom in GEOMS:
        N = geom["T"] * geom["h"] * geom["w"]
        M, H, hd = 4, 2, 8
        q, k, v = (rs.standard_normal((N, H, hd)) for _ in range(3))
        g = rs.integers(0, M, N)
        p_g = rs.uniform(0.3, 1.0, N)
        scale = 1.0 / np.sqrt(hd)
        whole = dict(moga=oatt.moga(q, k, v, g, p_g, M, scale),
                     win=oatt.grouped(q, k, v, ostga.window_groups(geom), scale),
                     frame=oatt.grouped(q, k, v, ostga.frame_groups(geom), scale))
        rows = osample.stratified_rows(geom, g, M, H, n_heads=2, per_head=40)
        for h, toks in rows.items():
            om, ow, of = osample.branch_rows(q[:, h], k[:, h], v[:, h], toks, g, p_g, M, geom, scale)
            np.testing.assert_allclose(om, whole["moga"][toks, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(ow, whole["win"][toks, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(of, whole["frame"][toks, h], rtol=1e-12, atol=1e-13)


def test_suite_samples_reach_4096_rows():
    for wl in (W.WAN13B_5S, W.LONG_60S):
        g = np.random.default_rng(0).integers(0, wl.M, wl.N)
        rows = osample.stratified_rows(W.stga_shape(wl), g, wl.M, wl.H, n_heads=8, per_head=512)
        assert len(rows) == 8 and sum(len(t) for t in rows.values()) >= 4096
