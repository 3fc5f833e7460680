"""Oracle: linear top-1 token router.

Definition (note, key design 1; translation, 混合分组注意力; blog 2.3): for a
token x in R^d and M groups, r = Router(x) = x . W_r with W_r in R^{d x M}
and no bias (the blog's sketch uses a bias-free linear layer);
p(i|x) = softmax(r)_i; g(x) = argmax_i p(i|x); the gate is p(g(x)|x).

The optional bias exists only to build a skewed workload (one group holding
about 40 % of the tokens); None means the pages' bias-free router.

Ties in the argmax go to the lowest index (numpy's argmax returns the first
maximum).  The workloads redraw inputs whose top-2 probability gap is below
1e-3, so ties never decide a parity result.

Pinned by: brute-force pure-Python routing on tiny inputs, sum_i p = 1,
M = 1 giving g = 0 and p = 1, and a hand-computed two-group example.
"""
from __future__ import annotations

import numpy as np


def logits(x: np.ndarray, w_r: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """r = x . W_r (+ bias), float64, shape [N, M]."""
    r = np.asarray(x, dtype=np.float64) @ np.asarray(w_r, dtype=np.float64)
    if bias is not None:
        r = r + np.asarray(bias, dtype=np.float64)[None, :]
    return r


def probabilities(r: np.ndarray) -> np.ndarray:
    """p(i|x) = softmax(r)_i = exp(r_i) / sum_j exp(r_j) (shifted by max r for range)."""
    e = np.exp(r - r.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def route(x: np.ndarray, w_r: np.ndarray, bias: np.ndarray | None = None):
    """Returns (g [N] int64, p_g [N] float64, p [N, M] float64)."""
    p = probabilities(logits(x, w_r, bias))
    g = np.argmax(p, axis=1)
    p_g = p[np.arange(p.shape[0]), g]
    return g, p_g, p


def top2_margin(p: np.ndarray) -> np.ndarray:
    """p_(1) - p_(2): gap between the largest and second-largest probability (inf at M=1)."""
    if p.shape[1] == 1:
        return np.full(p.shape[0], np.inf)
    s = np.sort(p, axis=1)
    return s[:, -1] - s[:, -2]
