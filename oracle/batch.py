"""Oracle: the layer forward over a batch of B videos (test infrastructure only).

The pages fine-tune on many multi-shot videos and scale the method to an
MMDiT-based model at M = 20 with a context of about 578k tokens (note,
training setup).  They are silent on how a batch of videos meets the
router's groups.  Readings taken
here (each is the plainest one the rest supports):

* Groups are per video: a token attends only to tokens of its own video in
  its group (attention between different videos has no meaning), so the
  permute sorts by the key b * M + g(x), b the video of the token, giving
  B * M segments with cu_seqlens of B * M + 1 entries.  Inside a segment the
  order is ascending token index (the unique stable order).
* The router is shared and acts per token (key design 1), so routing the
  batch is routing its B * N tokens.
* The static STGA groups are per video, each with the same geometry.
* L_gb takes F_i and P_i over all B * N tokens of the batch (the MoE
  load-balancing form the note says it borrows is computed over the batch).
* Text tokens do not enter the visual-attention layer: the pages condition
  each shot on its text through the separate cross-modal block.

Tokens are flattened video-major: token t of video b is row b * N + t.

Pinned by (tests/test_oracle_batch.py): the batched permute against Python's
stable sort on (b * M + g, t); MoGA against dense masked attention over the
whole batch with mask [same video and same group]; B = 1 reducing to
`layer.forward`; a batch of two copies of one video giving that video's
outputs twice and its loss.
"""
from __future__ import annotations

import numpy as np

from . import attention, layer, route, stga


def permute_batched(g: np.ndarray, B: int, M: int):
    """Stable sort of B * N tokens by b * M + g.  Returns (perm [B*N] int64 of
    flattened token indices, cu_seqlens [B*M+1], counts [B*M], max_seqlen)."""
    g = np.asarray(g).reshape(B, -1)
    N = g.shape[1]
    members = []
    for b in range(B):
        for i in range(M):
            members.append(b * N + np.nonzero(g[b] == i)[0])
    counts = np.array([len(m) for m in members], dtype=np.int64)
    cu = np.zeros(B * M + 1, dtype=np.int64)
    cu[1:] = np.cumsum(counts)
    perm = np.concatenate(members).astype(np.int64)
    return perm, cu, counts, int(counts.max())


def forward_batched(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float, scale: float | None = None) -> dict:
    """x [B, N, d], q/k/v [B, N, H, hd]; every tensor float64.  Returns the
    flattened routing results, the batched permute, per-video branch outputs
    stacked to [B, N, H, hd], out and the batch loss."""
    B, N = x.shape[0], x.shape[1]
    hd = q.shape[3]
    scale = attention.default_scale(hd) if scale is None else scale
    g, p_g, p = route.route(np.asarray(x).reshape(B * N, -1), w_r, bias)
    perm, cu, counts, max_seqlen = permute_batched(g, B, M)
    gb, pgb = g.reshape(B, N), p_g.reshape(B, N)
    o_moga = np.stack([attention.moga(q[b], k[b], v[b], gb[b], pgb[b], M, scale) for b in range(B)])
    wg, fg = stga.window_groups(geom), stga.frame_groups(geom)
    o_win = np.stack([attention.grouped(q[b], k[b], v[b], wg, scale) for b in range(B)])
    o_frame = np.stack([attention.grouped(q[b], k[b], v[b], fg, scale) for b in range(B)])
    group_counts = counts.reshape(B, M).sum(axis=0)
    return dict(g=g, p_g=p_g, p=p, perm=perm, cu_seqlens=cu, counts=counts, max_seqlen=max_seqlen,
                o_moga=o_moga, o_win=o_win, o_frame=o_frame, out=layer.mean3(o_moga, o_win, o_frame),
                loss=layer.balance_loss(group_counts, p, alpha))
