"""Pins of the batched oracle (CPU): the per-video groups of a batch of B
videos against independent formulations (Python's stable sort on the key,
dense masked attention over the whole flattened batch, brute-force routing)
and the reductions to the single-video forward."""
import math

import numpy as np
import pytest

from oracle import batch, layer
from test_oracle_pins import _dense_masked, _route_brute, _visible_window

GEOM = dict(T=4, h=2, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=1, aug=1)
N = 32


@pytest.mark.parametrize("B,M", [(1, 3), (3, 4), (2, 20), (5, 7)])
def test_permute_batched_matches_stable_sort(B, M):
    rs = np.random.default_rng(B * 100 + M)
    n = 37
    g = rs.integers(0, M, B * n)
    perm, cu, counts, mx = batch.permute_batched(g, B, M)
    key = [(t // n) * M + int(g[t]) for t in range(B * n)]
    want = sorted(range(B * n), key=lambda t: (key[t], t))
    assert perm.tolist() == want
    assert counts.tolist() == [key.count(kk) for kk in range(B * M)]
    assert cu[0] == 0 and cu[-1] == B * n and np.all(np.diff(cu) == counts)
    assert mx == max(counts)
    for s in range(B * M):
        seg = perm[cu[s]:cu[s + 1]]
        assert all(key[t] == s for t in seg)


def _inputs(B, M, seed):
    rs = np.random.default_rng(seed)
    d, H, hd = 6, 1, 4
    x = rs.standard_normal((B, N, d))
    w_r = rs.standard_normal((d, M))
    q, k, v = (rs.standard_normal((B, N, H, hd)) for _ in range(3))
    return x, w_r, q, k, v


def test_batched_forward_dense_brute_force():
    """Every branch against dense masked attention over the flattened batch:
    a token sees the tokens of its own video only, and, for MoGA, of its group."""
    B, M = 3, 3
    x, w_r, q, k, v = _inputs(B, M, 7)
    res = batch.forward_batched(x, w_r, None, q, k, v, M, GEOM, alpha=0.1)
    xf = x.reshape(B * N, -1)
    bg, bpg, bp = _route_brute(xf.tolist(), w_r.tolist(), None)
    qf, kf, vf = (a.reshape(B * N, *a.shape[2:]).tolist() for a in (q, k, v))
    scale = 1 / math.sqrt(q.shape[3])
    vis = _visible_window(GEOM)
    o1 = _dense_masked(qf, kf, vf, lambda t, u: t // N == u // N and bg[t] == bg[u], scale, bpg)
    o2 = _dense_masked(qf, kf, vf, lambda t, u: t // N == u // N and vis(t % N, u % N), scale)
    o3 = _dense_masked(qf, kf, vf, lambda t, u: t // 8 == u // 8, scale)
    want = ((o1 + o2 + o3) / 3).reshape(res["out"].shape)
    np.testing.assert_allclose(res["out"], want, rtol=1e-12, atol=1e-13)
    F = [bg.count(i) / (B * N) for i in range(M)]
    P = [sum(row[i] for row in bp) / (B * N) for i in range(M)]
    assert res["loss"] == pytest.approx(0.1 * M * sum(f * p for f, p in zip(F, P)), rel=1e-13)


def test_single_video_batch_is_the_layer_forward():
    x, w_r, q, k, v = _inputs(1, 4, 8)
    a = batch.forward_batched(x, w_r, None, q, k, v, 4, GEOM, alpha=0.1)
    b = layer.forward(x[0], w_r, None, q[0], k[0], v[0], 4, GEOM, alpha=0.1)
    np.testing.assert_array_equal(a["out"][0], b["out"])
    assert a["perm"].tolist() == b["perm"].tolist()
    assert a["cu_seqlens"].tolist() == b["cu_seqlens"].tolist()
    assert a["loss"] == b["loss"]


def test_duplicated_video_gives_its_outputs_twice():
    """Two copies of one video: each copy's output is the single-video output
    (no attention across videos), and F, P (so the loss) are unchanged."""
    x, w_r, q, k, v = _inputs(1, 4, 9)
    two = [np.concatenate([a, a]) for a in (x, q, k, v)]
    a = batch.forward_batched(two[0], w_r, None, two[1], two[2], two[3], 4, GEOM, alpha=0.1)
    b = layer.forward(x[0], w_r, None, q[0], k[0], v[0], 4, GEOM, alpha=0.1)
    np.testing.assert_allclose(a["out"][0], b["out"], rtol=1e-15, atol=0)
    np.testing.assert_allclose(a["out"][1], b["out"], rtol=1e-15, atol=0)
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-14)
    assert a["cu_seqlens"][-1] == 2 * N and len(a["cu_seqlens"]) == 2 * 4 + 1
