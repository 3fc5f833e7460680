"""Oracle: the static spatial-temporal groups (STGA) and per-frame groups.

Pages: the latent video is cut into fixed spatial windows, then frames are
grouped along time, frames of different shots never sharing a temporal group;
the keys and values (not the queries) of a group gain two latent frames of the
adjacent shot to keep continuity at the cut; a per-frame attention groups the
tokens of each latent frame (note, key design 4; translation, 时空分组注意力;
blog 3.2 and the augment_kv=2 row of its section-9 table).  The training setup
uses a 2 x 2 spatial grouping (note, 训练设置).

Readings taken where the pages are silent:
  * windows: a non-overlapping, unshifted win_h x win_w tiling of the frame;
  * temporal groups: each shot is cut into ceil(len / tg_max) runs of frames,
    as equal as possible, longer runs first (tg_max = 0: the whole shot);
  * K/V augmentation: only a group touching a shot cut is augmented, with the
    min(aug, len) frames of the adjacent shot nearest the cut, on each side
    that has a neighbouring shot, in the same spatial window;
  * per-frame attention: all h*w tokens of the frame, no augmentation.

Tokens are in raster order: token = frame*h*w + row*w + col.

Pinned by: a dense visibility mask built from an independently written
predicate (tests), the Q = 0 closed form (mean of V over the augmented set),
a single shot giving no augmentation, and hand-listed groups for small shapes.
"""
from __future__ import annotations

import numpy as np


def split_runs(length: int, tg_max: int) -> list:
    """Run lengths of one shot's temporal groups (longer runs first)."""
    n = 1 if tg_max == 0 else -(-length // tg_max)
    q, r = divmod(length, n)
    return [q + 1] * r + [q] * (n - r)


def temporal_groups(shots, tg_max: int) -> list:
    """List of dicts {shot, t0, t1} (frames [t0, t1)) in time order."""
    out, t = [], 0
    for s, L in enumerate(shots):
        for run in split_runs(L, tg_max):
            out.append(dict(shot=s, t0=t, t1=t + run))
            t += run
    return out


def kv_frames(group: dict, shots, aug: int) -> list:
    """Frames whose window tokens form the group's keys/values."""
    starts = np.concatenate([[0], np.cumsum(shots)]).astype(int)
    s = group["shot"]
    frames = list(range(group["t0"], group["t1"]))
    if group["t0"] == starts[s] and s > 0:             # first group of a shot after a cut
        a = min(aug, shots[s - 1])
        frames = list(range(starts[s] - a, starts[s])) + frames
    if group["t1"] == starts[s + 1] and s + 1 < len(shots):   # last group before a cut
        a = min(aug, shots[s + 1])
        frames = frames + list(range(starts[s + 1], starts[s + 1] + a))
    return frames


def window_tokens(frames, y0: int, x0: int, win_h: int, win_w: int, h: int, w: int) -> np.ndarray:
    """Tokens of the window with top-left (y0, x0) in the listed frames (frame-major)."""
    ys = np.arange(y0, y0 + win_h)
    xs = np.arange(x0, x0 + win_w)
    f = np.asarray(list(frames), dtype=np.int64)
    tok = f[:, None, None] * (h * w) + ys[None, :, None] * w + xs[None, None, :]
    return tok.reshape(-1)


def window_groups(geom: dict) -> list:
    """All static window groups as (query tokens, key/value tokens)."""
    T, h, w = geom["T"], geom["h"], geom["w"]
    wh, ww = geom["win_h"], geom["win_w"]
    assert h % wh == 0 and w % ww == 0 and sum(geom["shots"]) == T
    out = []
    for grp in temporal_groups(geom["shots"], geom["tg_max"]):
        kvf = kv_frames(grp, geom["shots"], geom["aug"])
        for y0 in range(0, h, wh):
            for x0 in range(0, w, ww):
                q = window_tokens(range(grp["t0"], grp["t1"]), y0, x0, wh, ww, h, w)
                kv = window_tokens(kvf, y0, x0, wh, ww, h, w)
                out.append((q, kv))
    return out


def frame_groups(geom: dict) -> list:
    """Per-frame groups: (tokens of frame t, same tokens)."""
    hw = geom["h"] * geom["w"]
    return [(np.arange(t * hw, (t + 1) * hw), np.arange(t * hw, (t + 1) * hw)) for t in range(geom["T"])]
