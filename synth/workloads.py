"""Synthetic Wan-shaped workloads for the MoGA visual-attention layer.

The shapes follow the pages' setting: a (4,8,8) VAE and a (1,2,2) patchify
turn a 480p video into latent frames of 30 x 52 tokens (MoGA paper, page
"papernotes.org ICLR2026", flowchart; page "xugj520.cn" section 3.1), with
tokens in raster order (frame, row, column).  There is no public dataset for
this layer; the recipe below stands in for Wan latents:

* Q, K, V: i.i.d. N(0, 1) rounded to bf16 (separate counter streams), except
  the tiny case, whose Q/K/V are bf16(x . W) with W ~ N(0, 1/d) (fp64 product).
* x (router input): N(0, 1), fp32 for the tiny case and bf16 otherwise;
  W_r ~ N(0, 1/d) in the same dtype.  The clustered case draws
  x = sqrt(0.75) mu_c + sqrt(0.25) eps with 20 centres mu_c ~ N(0, I), c given
  by a 4 x 5 spatial region map whose region->cluster assignment is permuted
  per shot.
* Margin redraws: a row of x whose exact top-2 routing margin is too small is
  replaced by the next `draw` of that row's counters.  Which rows to redraw is
  decided by the caller (the tests use the CPU oracle); this module only
  regenerates the listed rows.

This module performs none of the attention layer's arithmetic.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field, replace

import numpy as np

from . import rng

# counter streams
S_X, S_WR, S_Q, S_K, S_V, S_WQ, S_WK, S_WV, S_MU, S_EPS, S_REGION, S_DOUT = range(1, 13)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # latent frames
    h: int                 # token rows per frame
    w: int                 # token columns per frame
    d: int                 # hidden size seen by the router
    H: int                 # heads
    hd: int                # head dim
    M: int                 # routing groups
    shots: tuple           # latent frames per shot (sums to T)
    tg_max: int            # max frames per temporal group (0 = whole shot)
    win_h: int
    win_w: int
    aug: int = 2           # adjacent-shot frames added to K/V at a shot cut (per side)
    x_dtype: str = "bf16"  # "f32" | "bf16"
    qkv: str = "iid"       # "iid" | "proj"
    bias0: float | None = None   # fp32 bias on group 0 (skewed router), None = no bias
    clusters: int = 0      # >0: clustered router input with this many centres
    alpha: float = 0.1
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T * self.h * self.w

    @property
    def hw(self) -> int:
        return self.h * self.w

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the benchmark suite.  tg_max=7 and the shot split of
# the long videos are readings of the pages (they give neither number).
TINY = Workload("tiny_2k", T=8, h=16, w=16, d=128, H=2, hd=64, M=4, shots=(4, 4), tg_max=0,
                win_h=8, win_w=8, x_dtype="f32", qkv="proj")
WAN13B_5S = Workload("wan1.3b_5s_1shot_32k", T=21, h=30, w=52, d=1536, H=12, hd=128, M=5,
                     shots=(21,), tg_max=7, win_h=15, win_w=26)
MULTISHOT_10S = Workload("multishot_10s_3shot_64k_skewed", T=41, h=30, w=52, d=1536, H=12, hd=128,
                         M=5, shots=(14, 14, 13), tg_max=7, win_h=15, win_w=26,
                         bias0=float("nan"))  # value filled from tests/golden/skew_bias.json
WAN14B_30S_M5 = Workload("wan14b_30s_5shot_282k_M5", T=181, h=30, w=52, d=5120, H=40, hd=128, M=5,
                         shots=(37, 36, 36, 36, 36), tg_max=7, win_h=15, win_w=26)
WAN14B_30S_M20 = WAN14B_30S_M5.with_(name="wan14b_30s_5shot_282k_M20", M=20)
LONG_60S = Workload("long_60s_10shot_563k_M20_clustered", T=361, h=30, w=52, d=5120, H=40, hd=128,
                    M=20, shots=(37,) + (36,) * 9, tg_max=7, win_h=15, win_w=26, clusters=20)

SUITE = {wl.name: wl for wl in (TINY, WAN13B_5S, MULTISHOT_10S, WAN14B_30S_M5, WAN14B_30S_M20, LONG_60S)}


def even_split(total: int, parts: int) -> list:
    """Split `total` into `parts` integers as equal as possible, larger first."""
    q, r = divmod(total, parts)
    return [q + 1] * r + [q] * (parts - r)


def shots_for(T: int, n_shots: int) -> tuple:
    """Shot lengths for a T-frame video of n_shots shots, earlier shots longer."""
    return tuple(even_split(T, n_shots))


# ----------------------------------------------------------------------------- bf16 bits

def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round to bf16 (round-to-nearest-even from fp32) and return the raw uint16 bits."""
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (f >> np.uint32(16)) & np.uint32(1)
    rounded = (f + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to float64."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- router inputs

def _region_of_token(wl: Workload, tok: np.ndarray) -> np.ndarray:
    """4 x 5 spatial region index (0..19) of each token."""
    rem = tok % wl.hw
    y, xcol = rem // wl.w, rem % wl.w
    ry = np.minimum((y * 4) // wl.h, 3)
    rx = np.minimum((xcol * 5) // wl.w, 4)
    return ry * 5 + rx


def _shot_of_frame(wl: Workload) -> np.ndarray:
    return np.repeat(np.arange(len(wl.shots)), wl.shots)


def cluster_of_token(wl: Workload, tok: np.ndarray) -> np.ndarray:
    """Cluster id c(t) of each token for the clustered router input."""
    assert wl.clusters == 20, "the region map has 4 x 5 = 20 regions"
    shot = _shot_of_frame(wl)[tok // wl.hw]
    region = _region_of_token(wl, tok)
    perms = np.stack([rng.permutation(wl.seed, S_REGION, 20, draw=s) for s in range(len(wl.shots))])
    return perms[shot, region]


def x_rows_f64(wl: Workload, rows: np.ndarray, redraw: dict | None = None) -> np.ndarray:
    """Router input rows as exact float64 values of the stored dtype."""
    rows = np.asarray(rows, dtype=np.int64)
    draws = np.zeros(len(rows), dtype=np.int64)
    if redraw:
        draws = np.array([redraw.get(int(r), 0) for r in rows], dtype=np.int64)
    out = np.empty((len(rows), wl.d), dtype=np.float64)
    for dv in np.unique(draws):
        sel = np.nonzero(draws == dv)[0]
        eps = rng.normal_block(wl.seed, S_EPS if wl.clusters else S_X, rows[sel], wl.d, draw=int(dv))
        if wl.clusters:
            c = cluster_of_token(wl, rows[sel])
            mu = rng.normal_block(wl.seed, S_MU, np.arange(wl.clusters), wl.d)
            eps = math.sqrt(0.75) * mu[c] + math.sqrt(0.25) * eps
        out[sel] = eps
    return _round_like(wl, out)


def _round_like(wl: Workload, a: np.ndarray) -> np.ndarray:
    if wl.x_dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    return bf16_bits_to_f64(to_bf16_bits(a))


def _parallel_chunks(n: int, chunk: int, fn) -> None:
    """Run fn(start, stop) over [0, n) in chunks on a thread pool (numpy releases the GIL)."""
    starts = list(range(0, n, chunk))
    if len(starts) <= 2:
        for s0 in starts:
            fn(s0, min(s0 + chunk, n))
        return
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda s0: fn(s0, min(s0 + chunk, n)), starts))


def x_stored(wl: Workload, redraw: dict | None = None, rows: np.ndarray | None = None,
             chunk: int = 8192) -> np.ndarray:
    """Router input in its stored form: float32 array or bf16 bits (uint16), [len(rows), d]."""
    rows = np.arange(wl.N) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), wl.d), dtype=np.float32 if wl.x_dtype == "f32" else np.uint16)

    def fill(a, b):
        v = x_rows_f64(wl, rows[a:b], redraw)
        out[a:b] = v.astype(np.float32) if wl.x_dtype == "f32" else to_bf16_bits(v)
    _parallel_chunks(len(rows), chunk, fill)
    return out


def w_r_f64(wl: Workload) -> np.ndarray:
    """Router weight W_r [d, M] ~ N(0, 1/d), exact values of the stored dtype."""
    w = rng.normal_block(wl.seed, S_WR, np.arange(wl.d), wl.M) / math.sqrt(wl.d)
    return _round_like(wl, w)


def w_r_stored(wl: Workload) -> np.ndarray:
    w = w_r_f64(wl)
    return w.astype(np.float32) if wl.x_dtype == "f32" else to_bf16_bits(w)


def bias_f64(wl: Workload) -> np.ndarray | None:
    """Optional fp32 router bias (beta on group 0, zeros elsewhere)."""
    if wl.bias0 is None:
        return None
    b = np.zeros(wl.M, dtype=np.float32)
    b[0] = np.float32(wl.bias0)
    return b.astype(np.float64)


# ----------------------------------------------------------------------------- Q, K, V

def qkv_rows_bits(wl: Workload, which: str, rows: np.ndarray, redraw: dict | None = None,
                  head: int | None = None) -> np.ndarray:
    """bf16 bits of Q, K or V for the listed tokens: [len(rows), H, hd], or [len(rows), hd] for one head.

    For the projected (tiny) workload, `redraw` must be the router input's
    redraw map so the projections see the same x rows as the router.
    """
    rows = np.asarray(rows, dtype=np.int64)
    width = wl.H * wl.hd
    cols = np.arange(width) if head is None else np.arange(head * wl.hd, (head + 1) * wl.hd)
    if wl.qkv == "iid":
        stream = {"q": S_Q, "k": S_K, "v": S_V}[which]
        idx = rows[:, None].astype(np.uint64) * np.uint64(width) + cols[None, :].astype(np.uint64)
        a = rng.normal(wl.seed, stream, idx)
    else:
        stream = {"q": S_WQ, "k": S_WK, "v": S_WV}[which]
        W = rng.normal_block(wl.seed, stream, np.arange(wl.d), width) / math.sqrt(wl.d)
        a = x_rows_f64(wl, rows, redraw) @ W[:, cols]
    bits = to_bf16_bits(a)
    return bits if head is not None else bits.reshape(len(rows), wl.H, wl.hd)


def proj_weight_bits(wl: Workload, which: str) -> np.ndarray:
    """bf16 bits of a Q, K or V projection weight [d, H*hd] ~ N(0, 1/d) (the draws of the
    projected workload's weights, rounded to bf16 as a model's weights would be)."""
    stream = {"q": S_WQ, "k": S_WK, "v": S_WV}[which]
    W = rng.normal_block(wl.seed, stream, np.arange(wl.d), wl.H * wl.hd) / math.sqrt(wl.d)
    return to_bf16_bits(W)


def qkv_stored(wl: Workload, which: str, redraw: dict | None = None, chunk: int = 4096) -> np.ndarray:
    out = np.empty((wl.N, wl.H, wl.hd), dtype=np.uint16)

    def fill(a, b):
        out[a:b] = qkv_rows_bits(wl, which, np.arange(a, b), redraw)
    _parallel_chunks(wl.N, chunk, fill)
    return out


def dout_bits(wl: Workload) -> np.ndarray:
    """bf16 bits of an upstream gradient of the layer output, i.i.d. N(0, 1): [N, H, hd]."""
    width = wl.H * wl.hd
    idx = np.arange(wl.N, dtype=np.uint64)[:, None] * np.uint64(width) + np.arange(width, dtype=np.uint64)[None, :]
    return to_bf16_bits(rng.normal(wl.seed, S_DOUT, idx)).reshape(wl.N, wl.H, wl.hd)


def stga_shape(wl: Workload) -> dict:
    """The static-group geometry as plain numbers (shot lengths, windows, aug)."""
    return dict(T=wl.T, h=wl.h, w=wl.w, win_h=wl.win_h, win_w=wl.win_w,
                shots=list(wl.shots), tg_max=wl.tg_max, aug=wl.aug)


# ----------------------------------------------------------------------------- fix-ups

_GOLDEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden")


def resolved(wl: Workload) -> Workload:
    """The workload with its stored skew bias filled in (if it has one)."""
    if wl.bias0 is not None and math.isnan(wl.bias0):
        with open(os.path.join(_GOLDEN, "skew_bias.json")) as f:
            return wl.with_(bias0=float(json.load(f)["bias0"]))
    return wl


def redraw_map(wl: Workload) -> dict:
    """Stored margin redraws {row: draw} of a suite workload ({} if none stored)."""
    path = os.path.join(_GOLDEN, "redraw_%s.json" % wl.name)
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        return {int(k): int(v) for k, v in json.load(f)["redraw"].items()}
