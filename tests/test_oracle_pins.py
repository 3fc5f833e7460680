"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test below would fail under a plausible mistake in the oracle: a missing
softmax scale, a transposed operand, a wrong gate, a group-membership slip,
an off-by-one in the shot-cut augmentation, a dropped term in the loss.
"""
import json
import math
import os
import random

import numpy as np
import pytest

from oracle import attention, layer, permute, route, stga

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


# ----------------------------------------------------------------------------- route

def test_route_closed_form():
    c = GOLDEN["route_two_groups"]
    g, p_g, p = route.route(np.array(c["x"]), np.array(c["w_r"]))
    np.testing.assert_allclose(p, c["p"], rtol=0, atol=1e-15)
    assert g.tolist() == c["g"]
    np.testing.assert_allclose(p_g, c["p_g"], rtol=0, atol=1e-15)
    g, p_g, p = route.route(np.array(c["x"]), np.array(c["w_r"]), np.array(c["bias"]))
    np.testing.assert_allclose(p, c["p_with_bias"], rtol=0, atol=1e-15)
    assert g.tolist() == c["g_with_bias"]
    np.testing.assert_allclose(p_g, c["p_g_with_bias"], rtol=0, atol=1e-15)


def _route_brute(x, w, b):
    out_g, out_pg, out_p = [], [], []
    for row in x:
        r = [sum(row[k] * w[k][i] for k in range(len(row))) + (b[i] if b is not None else 0.0)
             for i in range(len(w[0]))]
        e = [math.exp(v) for v in r]
        s = sum(e)
        p = [v / s for v in e]
        best = 0
        for i in range(1, len(p)):
            if p[i] > p[best]:
                best = i
        out_g.append(best)
        out_pg.append(p[best])
        out_p.append(p)
    return out_g, out_pg, out_p


@pytest.mark.parametrize("M", [1, 2, 5, 7])
def test_route_brute_force(M):
    rs = np.random.default_rng(M)
    x = rs.standard_normal((40, 9))
    w = rs.standard_normal((9, M)) / 3
    b = rs.standard_normal(M) * 0.1
    g, p_g, p = route.route(x, w, b)
    bg, bpg, bp = _route_brute(x.tolist(), w.tolist(), b.tolist())
    assert g.tolist() == bg
    np.testing.assert_allclose(p_g, bpg, rtol=1e-13)
    np.testing.assert_allclose(p, bp, rtol=1e-13)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_route_single_group_and_ties():
    x = np.random.default_rng(0).standard_normal((10, 4))
    g, p_g, p = route.route(x, np.ones((4, 1)))
    assert (g == 0).all() and (p_g == 1.0).all()
    # exact tie between groups 1 and 2 (identical columns): lowest index wins
    w = np.array([[0.0, 1.0, 1.0]] * 4)
    g, _, _ = route.route(np.ones((3, 4)), w)
    assert (g == 1).all()


def test_route_margin():
    p = np.array([[0.5, 0.3, 0.2], [0.34, 0.33, 0.33]])
    np.testing.assert_allclose(route.top2_margin(p), [0.2, 0.01])


# ----------------------------------------------------------------------------- permute

@pytest.mark.parametrize("N,M", [(0, 3), (1, 1), (37, 4), (300, 32), (129, 5)])
def test_permute_matches_stable_sort(N, M):
    rs = random.Random(N * 31 + M)
    g = [rs.randrange(M) for _ in range(N)]
    if N > 3:
        g = [x if x != 1 else 0 for x in g]          # leave group 1 empty
    perm, cu, counts, mx = permute.permute(np.array(g, dtype=np.int64), M)
    expect = sorted(range(N), key=lambda t: (g[t], t))
    assert perm.tolist() == expect
    assert counts.sum() == N and cu[0] == 0 and cu[-1] == N
    assert (np.diff(cu) == counts).all() and (np.diff(cu) >= 0).all()
    assert mx == (max(counts) if N else 0)
    inv = np.empty(N, dtype=np.int64)
    inv[perm] = np.arange(N)
    assert (perm[inv] == np.arange(N)).all()
    for i in range(M):
        seg = perm[cu[i]:cu[i + 1]]
        assert all(g[t] == i for t in seg)
        assert (np.diff(seg) > 0).all()


# ----------------------------------------------------------------------------- attention

def test_attention_closed_form():
    c = GOLDEN["attention_two_keys"]
    q, k, v = (np.array(c[n]) for n in ("q", "k", "v"))
    sa = attention.attend(q, k, v, attention.default_scale(2))
    np.testing.assert_allclose(sa, c["sa"], rtol=0, atol=1e-13)
    o = attention.rows_of_group(q, k, v, attention.default_scale(2), gate=[c["gate"]])
    np.testing.assert_allclose(o, c["moga"], rtol=0, atol=1e-13)


def _dense_masked(q, k, v, allowed, scale, gate=None):
    """Pure-Python dense attention: row t attends to every u with allowed(t, u)."""
    N, H, hd, dv = len(q), len(q[0]), len(q[0][0]), len(v[0][0])
    out = [[[0.0] * dv for _ in range(H)] for _ in range(N)]
    for t in range(N):
        keys = [u for u in range(len(k)) if allowed(t, u)]
        if not keys:
            continue
        for h in range(H):
            sc = [scale * sum(q[t][h][c] * k[u][h][c] for c in range(hd)) for u in keys]
            m = max(sc)
            e = [math.exp(s - m) for s in sc]
            z = sum(e)
            for c in range(dv):
                val = sum(e[j] * v[u][h][c] for j, u in enumerate(keys)) / z
                out[t][h][c] = val * (gate[t] if gate is not None else 1.0)
    return np.array(out)


def test_moga_dense_brute_force():
    rs = np.random.default_rng(3)
    N, H, hd, M = 14, 2, 4, 3
    q, k, v = (rs.standard_normal((N, H, hd)) for _ in range(3))
    g = np.array([0, 2, 2, 0, 1, 0, 2, 2, 1, 0, 0, 2, 1, 2])
    p_g = rs.uniform(0.3, 1.0, N)
    o = attention.moga(q, k, v, g, p_g, M, 0.5)
    ref = _dense_masked(q.tolist(), k.tolist(), v.tolist(), lambda t, u: g[t] == g[u], 0.5, p_g.tolist())
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_moga_single_group_is_full_attention():
    rs = np.random.default_rng(4)
    N, H, hd = 9, 1, 3
    q = rs.standard_normal((N, H, hd))
    k = rs.standard_normal((N + 0, H, hd))
    v = rs.standard_normal((N, H, hd))
    o = attention.moga(q, k, v, np.zeros(N, dtype=np.int64), np.ones(N), 1, 1 / math.sqrt(hd))
    ref = _dense_masked(q.tolist(), k.tolist(), v.tolist(), lambda t, u: True, 1 / math.sqrt(hd))
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_attend_rectangular_operands():
    rs = np.random.default_rng(5)
    q, k, v = rs.standard_normal((3, 4)), rs.standard_normal((7, 4)), rs.standard_normal((7, 2))
    ref = _dense_masked(q[:, None].tolist(), k[:, None].tolist(), v[:, None].tolist(), lambda t, u: True, 0.7)
    np.testing.assert_allclose(attention.attend(q, k, v, 0.7), ref[:, 0], rtol=1e-12)


def test_moga_zero_query_and_constant_value():
    rs = np.random.default_rng(6)
    N, H, hd, M = 40, 3, 8, 4
    g = rs.integers(0, M, N)
    p_g = rs.uniform(0.3, 1, N)
    k, v = rs.standard_normal((N, H, hd)), rs.standard_normal((N, H, hd))
    o = attention.moga(np.zeros((N, H, hd)), k, v, g, p_g, M, 0.3)
    for t in range(N):
        mean = v[g == g[t]].mean(axis=0)
        np.testing.assert_allclose(o[t], p_g[t] * mean, rtol=1e-12, atol=1e-14)
    o = attention.moga(rs.standard_normal((N, H, hd)), k, np.full((N, H, hd), 2.5), g, p_g, M, 0.3)
    np.testing.assert_allclose(o, 2.5 * p_g[:, None, None] * np.ones((N, H, hd)), rtol=1e-12)


# ----------------------------------------------------------------------------- STGA

def test_temporal_splits_golden():
    for case in GOLDEN["temporal_splits"]["cases"]:
        assert stga.split_runs(case["len"], case["tg_max"]) == case["runs"]


@pytest.mark.parametrize("aug", [1, 2])
def test_stga_small_geometry_golden(aug):
    c = GOLDEN["stga_small_geometry"]
    groups = stga.temporal_groups(c["shots"], c["tg_max"])
    assert [[gp["t0"], gp["t1"]] for gp in groups] == c["groups"]
    assert [stga.kv_frames(gp, c["shots"], aug) for gp in groups] == c["kv_frames_aug%d" % aug]


def _visible_window(geom):
    """Independent visibility predicate for the window branch, token by token."""
    T, h, w, wh, ww = geom["T"], geom["h"], geom["w"], geom["win_h"], geom["win_w"]
    shots, tg, aug = geom["shots"], geom["tg_max"], geom["aug"]
    frame_shot, frame_grp, bounds = [], [], []
    gid = 0
    for s, L in enumerate(shots):
        n = 1 if tg == 0 else math.ceil(L / tg)
        base, extra = L // n, L % n
        for j in range(n):
            size = base + (1 if j < extra else 0)
            for _ in range(size):
                frame_shot.append(s)
                frame_grp.append(gid)
            gid += 1
    shot_start = [sum(shots[:s]) for s in range(len(shots))]

    def info(tok):
        f = tok // (h * w)
        y, x = (tok % (h * w)) // w, tok % w
        return f, y // wh, x // ww

    def visible(t, u):
        ft, wyt, wxt = info(t)
        fu, wyu, wxu = info(u)
        if (wyt, wxt) != (wyu, wxu):
            return False
        if frame_grp[fu] == frame_grp[ft]:
            return True
        s = frame_shot[ft]
        grp_frames = [f for f in range(T) if frame_grp[f] == frame_grp[ft]]
        first, last = grp_frames[0], grp_frames[-1]
        if first == shot_start[s] and s > 0 and frame_shot[fu] == s - 1 and fu >= shot_start[s] - aug:
            return True
        if last == shot_start[s] + shots[s] - 1 and s + 1 < len(shots) and frame_shot[fu] == s + 1 \
                and fu < shot_start[s + 1] + aug:
            return True
        return False
    return visible


@pytest.mark.parametrize("geom", [
    dict(T=6, h=4, w=4, win_h=2, win_w=2, shots=[3, 1, 2], tg_max=2, aug=2),
    dict(T=5, h=2, w=6, win_h=2, win_w=3, shots=[5], tg_max=2, aug=2),
    dict(T=4, h=2, w=2, win_h=1, win_w=2, shots=[2, 2], tg_max=0, aug=2),
    dict(T=7, h=2, w=2, win_h=2, win_w=1, shots=[1, 4, 2], tg_max=3, aug=1),
])
def test_stga_window_dense_brute_force(geom):
    rs = np.random.default_rng(7)
    N = geom["T"] * geom["h"] * geom["w"]
    H, hd = 2, 3
    q, k, v = (rs.standard_normal((N, H, hd)) for _ in range(3))
    o = attention.grouped(q, k, v, stga.window_groups(geom), 0.6)
    vis = _visible_window(geom)
    ref = _dense_masked(q.tolist(), k.tolist(), v.tolist(), vis, 0.6)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    # every token is the query of exactly one window group
    qs = np.concatenate([qt for qt, _ in stga.window_groups(geom)])
    assert sorted(qs.tolist()) == list(range(N))


def test_stga_zero_query_mean_of_augmented_set():
    geom = dict(T=6, h=4, w=4, win_h=2, win_w=4, shots=[2, 4], tg_max=2, aug=2)
    rs = np.random.default_rng(8)
    N, H, hd = 96, 1, 2
    v = rs.standard_normal((N, H, hd))
    o = attention.grouped(np.zeros((N, H, hd)), rs.standard_normal((N, H, hd)), v, stga.window_groups(geom), 1.0)
    vis = _visible_window(geom)
    for t in range(N):
        mem = [u for u in range(N) if vis(t, u)]
        np.testing.assert_allclose(o[t], v[mem].mean(axis=0), rtol=1e-12)


def test_stga_single_shot_has_no_augmentation():
    geom = dict(T=21, h=30, w=52, win_h=15, win_w=26, shots=[21], tg_max=7, aug=2)
    for qt, kvt in stga.window_groups(geom):
        assert np.array_equal(qt, kvt) and len(qt) == 7 * 15 * 26


def test_frame_groups_are_varlen_segments():
    geom = dict(T=3, h=2, w=3, win_h=1, win_w=3, shots=[3], tg_max=0, aug=2)
    rs = np.random.default_rng(9)
    q, k, v = (rs.standard_normal((18, 2, 4)) for _ in range(3))
    o = attention.grouped(q, k, v, stga.frame_groups(geom), 0.5)
    ref = _dense_masked(q.tolist(), k.tolist(), v.tolist(), lambda t, u: t // 6 == u // 6, 0.5)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- mean, loss, layer

def test_balance_loss_closed_forms():
    c = GOLDEN["balance_loss"]
    M, alpha, N = c["M"], c["alpha"], 1000
    counts = np.full(M, N // M)
    assert layer.balance_loss(counts, np.full((N, M), 1.0 / M), alpha) == pytest.approx(c["uniform"], rel=1e-14)
    p = np.zeros((N, M))
    p[:, 0] = 1
    assert layer.balance_loss(np.array([N] + [0] * (M - 1)), p, alpha) == pytest.approx(c["collapsed"], rel=1e-14)


def test_balance_loss_minimal_at_uniform():
    rs = np.random.default_rng(10)
    M, N, alpha = 5, 500, 0.1
    for _ in range(20):
        g = rs.integers(0, M, N)
        counts = np.bincount(g, minlength=M)
        # P equal to F: the assignment's own share; L = alpha*M*sum F^2 >= alpha
        p = np.tile(counts / N, (N, 1))
        assert layer.balance_loss(counts, p, alpha) >= alpha - 1e-15


def test_balance_loss_terms():
    # two groups, hand numbers: F = (0.75, 0.25), P = (0.6, 0.4): L = 0.1*2*(0.45+0.1) = 0.11
    p = np.array([[0.9, 0.1], [0.7, 0.3], [0.5, 0.5], [0.3, 0.7]])
    assert layer.balance_loss(np.array([3, 1]), p, 0.1) == pytest.approx(0.11, rel=1e-14)


def test_mean_linearity():
    rs = np.random.default_rng(11)
    a, b, c = (rs.standard_normal((5, 2, 3)) for _ in range(3))
    z = np.zeros_like(a)
    np.testing.assert_allclose(layer.mean3(a, z, z) + layer.mean3(z, b, z) + layer.mean3(z, z, c),
                               layer.mean3(a, b, c), rtol=1e-15)
    np.testing.assert_allclose(layer.mean3(a, b, c), (a + b + c) / 3, rtol=1e-15)


def test_layer_forward_tiny_brute_force():
    rs = np.random.default_rng(12)
    geom = dict(T=4, h=2, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=1, aug=1)
    N, d, M, H, hd = 32, 6, 3, 1, 4
    x, w_r = rs.standard_normal((N, d)), rs.standard_normal((d, M))
    q, k, v = (rs.standard_normal((N, H, hd)) for _ in range(3))
    res = layer.forward(x, w_r, None, q, k, v, M, geom, alpha=0.1)
    bg, bpg, bp = _route_brute(x.tolist(), w_r.tolist(), None)
    scale = 1 / math.sqrt(hd)
    o1 = _dense_masked(q.tolist(), k.tolist(), v.tolist(), lambda t, u: bg[t] == bg[u], scale, bpg)
    o2 = _dense_masked(q.tolist(), k.tolist(), v.tolist(), _visible_window(geom), scale)
    o3 = _dense_masked(q.tolist(), k.tolist(), v.tolist(), lambda t, u: t // 8 == u // 8, scale)
    np.testing.assert_allclose(res["out"], (o1 + o2 + o3) / 3, rtol=1e-12, atol=1e-13)
    F = [bg.count(i) / N for i in range(M)]
    P = [sum(row[i] for row in bp) / N for i in range(M)]
    assert res["loss"] == pytest.approx(0.1 * M * sum(f * p for f, p in zip(F, P)), rel=1e-13)
