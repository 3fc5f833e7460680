"""Oracle: full softmax attention inside groups (MoGA, STGA windows, frames).

Self-attention inside one group is the textbook non-causal scaled dot-product
attention SA(q, K, V) = softmax(q K^T / sqrt(hd)) V, with no mask, no dropout
and no bias (note, key design 1: "SA(q, K_g(x), V_g(x))").  The MoGA branch
multiplies each token's output by its gate p(g(x)|x), which is what makes the
router differentiable (note, key design 1), and writes it back at the token's
own position (the repermute of note, key design 2).

All arithmetic is float64.  Output rows are independent by definition, so
rows may be computed in chunks to bound memory; nothing else is reordered.

Pinned by: dense N x N masked attention written out in pure Python on tiny
inputs, M = 1 equal to textbook full attention, Q = 0 giving the gate times
the group mean of V, constant V giving gate * c, and a hand-computed
two-key example.
"""
from __future__ import annotations

import numpy as np

ROW_CHUNK = 2048


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q k^T * scale) v for q [nq, hd], k [nk, hd], v [nk, dv]; float64."""
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    for s in range(0, q.shape[0], ROW_CHUNK):
        S = (q[s:s + ROW_CHUNK] @ k.T) * scale
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[s:s + ROW_CHUNK] = P @ v
    return out


def default_scale(hd: int) -> float:
    return 1.0 / np.sqrt(hd)


def moga(q, k, v, g, p_g, M: int, scale: float) -> np.ndarray:
    """o[t, h] = p_g[t] * SA(q[t, h], K of group g_t, V of group g_t); q,k,v [N, H, hd]."""
    N, H, _ = q.shape
    o = np.zeros_like(q, dtype=np.float64)
    for i in range(M):
        mem = np.nonzero(np.asarray(g) == i)[0]
        if len(mem) == 0:
            continue
        for h in range(H):
            o[mem, h] = p_g[mem, None] * attend(q[mem, h], k[mem, h], v[mem, h], scale)
    return o


def grouped(q, k, v, groups, scale: float) -> np.ndarray:
    """o[t, h] = SA(q[t, h], K[kv, h], V[kv, h]) for each (q tokens, kv tokens) group.

    Used for the STGA window groups and the per-frame groups; a token that is
    a query of no group keeps a zero row.
    """
    N, H, _ = q.shape
    o = np.zeros_like(q, dtype=np.float64)
    for qt, kvt in groups:
        for h in range(H):
            o[qt, h] = attend(q[qt, h], k[kvt, h], v[kvt, h], scale)
    return o


def rows_of_group(q_rows, k_rows, v_rows, scale: float, gate=None) -> np.ndarray:
    """One head's attention for the listed query rows against a whole group's K/V.

    q_rows [n, hd], k_rows/v_rows [m, hd]; gate [n] or None.  This is the
    sampled form used at sizes where the full output is too large: each row
    is computed from its full definition.
    """
    o = attend(q_rows, k_rows, v_rows, scale)
    return o if gate is None else np.asarray(gate)[:, None] * o
