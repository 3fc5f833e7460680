"""Oracle: three-way mean and group-balancing loss; the whole layer forward.

Mean: every token receives one dynamic output (MoGA) and two static outputs
(the STGA window group and its frame), and the layer output is their average
(note, flowchart and key design 4; translation, 时空分组注意力).  Equal weights
of 1/3; the MoGA output already carries the gate.

Loss (note, key design 3; translation, 组平衡损失, whose formula did not
survive extraction): L_gb = alpha * M * sum_i F_i * P_i with
F_i = (1/N) sum_x 1(g(x) = i), the share of tokens routed to group i, and P_i
the mean routing probability of group i.  P_i is read as the mean of p(i|x)
over all N tokens (the MoE load-balancing form the note says it borrows).

Pinned by: uniform F = P = 1/M gives L = alpha; full collapse (all tokens in
group 0 with p = 1) gives L = alpha * M; random perturbations of a uniform
assignment never go below alpha; linearity of the mean.
"""
from __future__ import annotations

import numpy as np

from . import attention, permute, route, stga


def mean3(o_moga: np.ndarray, o_win: np.ndarray, o_frame: np.ndarray) -> np.ndarray:
    return (o_moga + o_win + o_frame) / 3.0


def balance_loss(counts: np.ndarray, p: np.ndarray, alpha: float) -> float:
    """L_gb from group counts [M] and routing probabilities p [N, M]."""
    N, M = p.shape
    F = np.asarray(counts, dtype=np.float64) / N
    P = p.mean(axis=0)
    return float(alpha * M * np.sum(F * P))


def forward(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float, scale: float | None = None) -> dict:
    """The whole visual-attention layer forward; every tensor float64.

    x [N, d], w_r [d, M], q/k/v [N, H, hd].  Returns every intermediate.
    """
    hd = q.shape[2]
    scale = attention.default_scale(hd) if scale is None else scale
    g, p_g, p = route.route(x, w_r, bias)
    perm, cu, counts, max_seqlen = permute.permute(g, M)
    o_moga = attention.moga(q, k, v, g, p_g, M, scale)
    o_win = attention.grouped(q, k, v, stga.window_groups(geom), scale)
    o_frame = attention.grouped(q, k, v, stga.frame_groups(geom), scale)
    return dict(g=g, p_g=p_g, p=p, perm=perm, cu_seqlens=cu, counts=counts, max_seqlen=max_seqlen,
                o_moga=o_moga, o_win=o_win, o_frame=o_frame, out=mean3(o_moga, o_win, o_frame),
                loss=balance_loss(counts, p, alpha))
