"""Stratified (token, head) rows for sampled checks at sizes where the whole
output is too large for the oracle, and for the timed CPU baseline.

TEST INFRASTRUCTURE ONLY, like the rest of this package.  This module picks
rows; it computes none of the layer's outputs.  Each picked row is then
computed by the oracle from its full definition (a query row against its whole
group's keys and values), so sampling changes which rows are checked, never
how a row is computed.

Coverage, per sampled head:
  * every MoGA group: its first and last member (in token order) and random
    members, at least `per_group` of them (all members of a small group);
  * every static window group (spatial window x temporal group): at least
    one query token;
  * both sides of every shot cut: for each window, one token in each of the
    `aug` frames before the cut and the `aug` frames after it (the frames that
    the groups at the cut borrow as keys/values, and the queries of those
    groups);
  * every latent frame: at least one token (the per-frame branch);
  * uniform random tokens up to `per_head` rows.

The sampled heads are spread evenly over [0, H) and always include the first
and the last head.
"""
from __future__ import annotations

import numpy as np

from . import stga as ostga


def sample_heads(H: int, n_heads: int) -> list:
    """n_heads heads spread evenly over [0, H), including 0 and H - 1."""
    n = min(n_heads, H)
    if n <= 1:
        return [0]
    return sorted(set(int(round(i * (H - 1) / (n - 1))) for i in range(n)))


def stratified_tokens(geom: dict, g: np.ndarray, M: int, rs: np.random.Generator, per_group: int = 8,
                      per_head: int = 512) -> np.ndarray:
    """Sorted unique token indices covering every group, window group, cut side and frame."""
    g = np.asarray(g)
    N = len(g)
    hw = geom["h"] * geom["w"]
    toks = []
    order = np.argsort(g, kind="stable")
    counts = np.bincount(g, minlength=M)
    starts = np.concatenate([[0], np.cumsum(counts)])
    for i in range(M):
        mem = order[starts[i]:starts[i + 1]]
        if len(mem) == 0:
            continue
        toks.append(mem[[0, -1]])
        toks.append(rs.choice(mem, size=min(per_group, len(mem)), replace=False))
    for qt, _ in ostga.window_groups(geom):
        toks.append(rs.choice(qt, size=1))
    shots = list(geom["shots"])
    cuts = np.cumsum(shots)[:-1]
    aug = max(int(geom["aug"]), 1)
    wh, ww = geom["win_h"], geom["win_w"]
    for c in cuts.tolist():
        for f in range(max(c - aug, 0), min(c + aug, geom["T"])):
            for y0 in range(0, geom["h"], wh):
                for x0 in range(0, geom["w"], ww):
                    win = ostga.window_tokens([f], y0, x0, wh, ww, geom["h"], geom["w"])
                    toks.append(rs.choice(win, size=1))
    toks.append(np.arange(geom["T"]) * hw + rs.integers(0, hw, geom["T"]))
    got = np.unique(np.concatenate(toks))
    if len(got) < per_head:
        extra = rs.choice(N, size=min(N, 2 * (per_head - len(got))), replace=False)
        got = np.unique(np.concatenate([got, extra]))
        if len(got) > per_head:
            keep = np.isin(got, np.unique(np.concatenate(toks)))
            rest = np.nonzero(~keep)[0]
            drop = rs.choice(rest, size=len(got) - per_head, replace=False)
            got = np.delete(got, drop)
    return got


def stratified_rows(geom: dict, g: np.ndarray, M: int, H: int, n_heads: int = 8, per_head: int = 512,
                    seed: int = 1) -> dict:
    """{head: sorted token indices}; every head gets its own draw of the strata."""
    rs = np.random.default_rng(seed)
    return {h: stratified_tokens(geom, g, M, rs, per_head=per_head) for h in sample_heads(H, n_heads)}


def branch_rows(qh, kh, vh, toks, g, p_g, M: int, geom: dict, scale: float):
    """The three branch outputs of one head at the listed tokens, each row from its definition.

    qh, kh, vh: [N, hd] float64 of one head; toks: token indices; g, p_g: the
    routing of all N tokens.  Returns (o_moga, o_win, o_frame), each
    [len(toks), hd]: the gated attention over the token's MoGA group, the
    attention over its window group's (augmented) keys, and over its frame.
    """
    from . import attention as oatt
    toks = np.asarray(toks)
    g = np.asarray(g)
    hd = qh.shape[1]
    o_m = np.zeros((len(toks), hd))
    o_w = np.zeros_like(o_m)
    o_f = np.zeros_like(o_m)
    order = np.argsort(g, kind="stable")
    counts = np.bincount(g, minlength=M)
    starts = np.concatenate([[0], np.cumsum(counts)])
    gt = g[toks]
    for i in range(M):
        sel = np.nonzero(gt == i)[0]
        if len(sel):
            mem = order[starts[i]:starts[i + 1]]
            o_m[sel] = oatt.rows_of_group(qh[toks[sel]], kh[mem], vh[mem], scale, np.asarray(p_g)[toks[sel]])
    owner = np.full(len(g), -1, dtype=np.int64)
    wgroups = ostga.window_groups(geom)
    for gi, (qt, _) in enumerate(wgroups):
        owner[qt] = gi
    ow = owner[toks]
    for gi in np.unique(ow).tolist():
        sel = np.nonzero(ow == gi)[0]
        kvt = wgroups[gi][1]
        o_w[sel] = oatt.attend(qh[toks[sel]], kh[kvt], vh[kvt], scale)
    hw = geom["h"] * geom["w"]
    fr = toks // hw
    for f in np.unique(fr).tolist():
        sel = np.nonzero(fr == f)[0]
        o_f[sel] = oatt.attend(qh[toks[sel]], kh[f * hw:(f + 1) * hw], vh[f * hw:(f + 1) * hw], scale)
    return o_m, o_w, o_f
