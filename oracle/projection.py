"""Oracle: the attention layer's Q/K/V projection (test infrastructure only).

The step just before the path (MoGA note, flowchart: the visual-attention
block projects its input tokens to queries, keys and values; key design 1:
the router reads the same tokens).  With the projection weight in the layout
of a linear layer's weight, W_qkv [3 H hd, d] (rows [0, H hd) for Q, then K,
then V):

    q[t, h, e] = sum_k x[t, k] * W_qkv[h hd + e, k]          (likewise k, v)

in float64; the router is `route.route` on the same x.  Pinned by
(tests/test_oracle_projection.py): the input generator's own projection of
the projected workload (computed there from the same weight draws), and a
weight made of unit rows that copies columns of x.
"""
from __future__ import annotations

import numpy as np


def qkv(x: np.ndarray, w_qkv: np.ndarray, H: int, hd: int):
    """x [N, d], w_qkv [3*H*hd, d] -> (q, k, v), each [N, H, hd] float64."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w_qkv, dtype=np.float64).T
    n = y.shape[0]
    w = H * hd
    return tuple(y[:, i * w:(i + 1) * w].reshape(n, H, hd) for i in range(3))
