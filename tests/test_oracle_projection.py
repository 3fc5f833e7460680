"""Pins of the projection oracle (CPU)."""
import numpy as np

from oracle import projection
from synth import workloads as W


def test_matches_the_generators_projection():
    """The tiny workload's Q/K/V are generated as bf16(x . W) from the same weight
    draws: the oracle's projection with those weights (fp64) must round to the same
    bf16 values, up to fp64 rounding ties."""
    wl = W.TINY
    x = W.x_stored(wl, W.redraw_map(wl)).astype(np.float64)
    rows = np.arange(0, wl.N, 7)
    import math
    from synth import rng
    ws = []
    for which, stream in (("q", W.S_WQ), ("k", W.S_WK), ("v", W.S_WV)):
        ws.append(rng.normal_block(wl.seed, stream, np.arange(wl.d), wl.H * wl.hd) / math.sqrt(wl.d))
    w_qkv = np.concatenate(ws, axis=1).T          # [3 H hd, d]
    q, k, v = projection.qkv(x[rows], w_qkv, wl.H, wl.hd)
    for got, which in ((q, "q"), (k, "k"), (v, "v")):
        want = W.qkv_rows_bits(wl, which, rows, W.redraw_map(wl))
        same = np.mean(W.to_bf16_bits(got) == want)
        assert same > 0.9999, (which, same)


def test_unit_rows_copy_columns():
    rs = np.random.default_rng(0)
    N, d, H, hd = 9, 8, 2, 2
    x = rs.standard_normal((N, d))
    w = np.zeros((3 * H * hd, d))
    cols = rs.integers(0, d, 3 * H * hd)
    w[np.arange(3 * H * hd), cols] = 1.0
    q, k, v = projection.qkv(x, w, H, hd)
    got = np.concatenate([a.reshape(N, -1) for a in (q, k, v)], axis=1)
    np.testing.assert_array_equal(got, x[:, cols])
