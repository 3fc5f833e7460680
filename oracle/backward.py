"""Oracle: backward of the visual-attention layer (test infrastructure only).

The pages train the layer end to end (MoGA note, key designs 1 and 3: the
gate p(g(x)|x) multiplies the MoGA output so that the router receives a
gradient, and the balancing loss is added to the training objective).  This
module writes out the gradients of the forward in `layer.forward` by hand,
in float64, for the objective

    J = sum(dout * out) + dloss * L_gb

with upstream gradients dout [N, H, hd] and dloss (scalar).  Readings:

* g(x) = argmax and the counts F_i are piecewise constant: zero gradient.
  The gate p_g = p(g(x)|x) and the mean probabilities P_i carry the router's
  gradient.
* Q, K, V are inputs of the layer (their projection from x is outside it),
  so x receives gradient through the router only.

Attention (per group and head, S = q k^T * scale, P = softmax(S), O = P v):
    dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
    dQ = dS K * scale,  dK = dS^T Q * scale.
MoGA: o = p_g * O, so the attention sees dO = p_g * do and
    dgate[t] = sum_{h, d} do[t, h, d] * O[t, h, d].
Mean: each branch receives dout / 3.
Router: with p = softmax(r) per token and
    u[t, i] = dgate[t] * [i == g_t] + dloss * alpha * M * F_i / N,
    dr = p * (u - sum_i u_i p_i),  dW_r = x^T dr,  dx = dr W_r^T,  dbias = sum_t dr.

Pinned by central finite differences of `layer.forward` in float64 (see
tests/test_oracle_backward.py) along random directions for every input, and
by the closed forms of the uniform-attention and single-key cases.
"""
from __future__ import annotations

import numpy as np

from . import attention, layer, route, stga


def attend_bwd(q, k, v, do, scale: float):
    """Gradients of O = softmax(q k^T * scale) v for one group and head.

    q [nq, hd], k [nk, hd], v [nk, dv], do [nq, dv] -> (dq, dk, dv)."""
    S = (q @ k.T) * scale
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    O = P @ v
    dv = P.T @ do
    dP = do @ v.T
    D = np.sum(do * O, axis=1, keepdims=True)
    dS = P * (dP - D)
    dq = (dS @ k) * scale
    dk = (dS.T @ q) * scale
    return dq, dk, dv


def grouped_bwd(q, k, v, do, groups, scale: float):
    """Gradients of `attention.grouped` for upstream do [N, H, hd]; keys that
    belong to several groups (frames borrowed across a shot cut) accumulate."""
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    H = q.shape[1]
    for qt, kvt in groups:
        for h in range(H):
            a, b, c = attend_bwd(q[qt, h], k[kvt, h], v[kvt, h], do[qt, h], scale)
            dq[qt, h] += a
            dk[kvt, h] += b
            dv[kvt, h] += c
    return dq, dk, dv


def moga_bwd(q, k, v, g, p_g, M: int, scale: float, do):
    """Gradients of `attention.moga` for upstream do: (dq, dk, dv, dgate [N])."""
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    dgate = np.zeros(q.shape[0], dtype=np.float64)
    H = q.shape[1]
    g = np.asarray(g)
    for i in range(M):
        mem = np.nonzero(g == i)[0]
        if len(mem) == 0:
            continue
        for h in range(H):
            O = attention.attend(q[mem, h], k[mem, h], v[mem, h], scale)
            dgate[mem] += np.sum(do[mem, h] * O, axis=1)
            a, b, c = attend_bwd(q[mem, h], k[mem, h], v[mem, h], p_g[mem, None] * do[mem, h], scale)
            dq[mem, h] += a
            dk[mem, h] += b
            dv[mem, h] += c
    return dq, dk, dv, dgate


def route_bwd(x, w_r, bias, g, p, dgate, counts, alpha: float, dloss: float):
    """Gradients of the router through the gate and the balancing loss:
    (dx [N, d], dw_r [d, M], dbias [M] or None, dr [N, M])."""
    N, M = p.shape
    u = np.zeros((N, M), dtype=np.float64)
    u[np.arange(N), np.asarray(g)] = dgate
    F = np.asarray(counts, dtype=np.float64) / N
    u += dloss * alpha * M * F[None, :] / N
    dr = p * (u - np.sum(u * p, axis=1, keepdims=True))
    x = np.asarray(x, dtype=np.float64)
    dw_r = x.T @ dr
    dx = dr @ np.asarray(w_r, dtype=np.float64).T
    dbias = None if bias is None else dr.sum(axis=0)
    return dx, dw_r, dbias, dr


def layer_backward(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float, dout, dloss: float,
                   scale: float | None = None) -> dict:
    """All gradients of J = sum(dout * out) + dloss * L_gb; every tensor float64."""
    hd = q.shape[2]
    scale = attention.default_scale(hd) if scale is None else scale
    g, p_g, p = route.route(x, w_r, bias)
    counts = np.bincount(np.asarray(g), minlength=M)
    do = np.asarray(dout, dtype=np.float64) / 3.0
    dq, dk, dv, dgate = moga_bwd(q, k, v, g, p_g, M, scale, do)
    for groups in (stga.window_groups(geom), stga.frame_groups(geom)):
        a, b, c = grouped_bwd(q, k, v, do, groups, scale)
        dq += a
        dk += b
        dv += c
    dx, dw_r, dbias, dr = route_bwd(x, w_r, bias, g, p, dgate, counts, alpha, dloss)
    return dict(dq=dq, dk=dk, dv=dv, dx=dx, dw_r=dw_r, dbias=dbias, dgate=dgate, dr=dr)


def objective(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float, dout, dloss: float,
              scale: float | None = None) -> float:
    """J = sum(dout * out) + dloss * L_gb from the forward oracle (for finite differences)."""
    fw = layer.forward(x, w_r, bias, q, k, v, M, geom, alpha, scale)
    return float(np.sum(np.asarray(dout, dtype=np.float64) * fw["out"]) + dloss * fw["loss"])
