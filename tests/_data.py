"""Shared test inputs: one seeded synthetic case, as numpy (for the oracle) and torch CUDA tensors.

Both sides consume the same stored values (fp32 or bf16 bits from `synth`);
the oracle widens them exactly to float64.
"""
from __future__ import annotations

import functools
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import route as oroute  # noqa: E402
from synth import workloads as W  # noqa: E402

MARGIN = 1e-3


def margin_redraws(wl, rows=None) -> dict:
    """Rows of x to redraw until every exact top-2 probability gap is >= MARGIN (oracle routing)."""
    w = W.w_r_f64(wl)
    b = W.bias_f64(wl)
    redraw = {}
    rows = np.arange(wl.N) if rows is None else rows
    while len(rows):
        x = W.x_rows_f64(wl, rows, redraw)
        p = oroute.probabilities(oroute.logits(x, w, b))
        rows = rows[oroute.top2_margin(p) < MARGIN]
        for r in rows.tolist():
            redraw[r] = redraw.get(r, 0) + 1
    return redraw


class Case:
    def __init__(self, wl: W.Workload, redraw: dict | None = None, with_qkv: bool = True):
        wl = W.resolved(wl)
        self.wl = wl
        if redraw is None:
            redraw = W.redraw_map(wl) if wl.name in W.SUITE else margin_redraws(wl)
        self.redraw = redraw
        self.x_st = W.x_stored(wl, redraw)
        self.w_st = W.w_r_stored(wl)
        self.bias = W.bias_f64(wl)
        if with_qkv:
            self.q_bits = W.qkv_stored(wl, "q", redraw)
            self.k_bits = W.qkv_stored(wl, "k", redraw)
            self.v_bits = W.qkv_stored(wl, "v", redraw)
        self.geom = W.stga_shape(wl)

    # ----------------------------------------------------------------- oracle side
    def x64(self):
        return self.x_st.astype(np.float64) if self.x_st.dtype == np.float32 else W.bf16_bits_to_f64(self.x_st)

    def w64(self):
        return self.w_st.astype(np.float64) if self.w_st.dtype == np.float32 else W.bf16_bits_to_f64(self.w_st)

    @functools.lru_cache(maxsize=None)
    def route64(self):
        return oroute.route(self.x64(), self.w64(), self.bias)

    def head64(self, which: str, h: int) -> np.ndarray:
        bits = {"q": self.q_bits, "k": self.k_bits, "v": self.v_bits}[which]
        return W.bf16_bits_to_f64(bits[:, h, :])

    def qkv64(self):
        return tuple(W.bf16_bits_to_f64(b) for b in (self.q_bits, self.k_bits, self.v_bits))

    # ----------------------------------------------------------------- device side
    def gpu(self, device="cuda:0"):
        import torch
        if self.x_st.dtype == np.float32:
            x = torch.from_numpy(self.x_st).to(device)
            w = torch.from_numpy(self.w_st).to(device)
        else:
            x = torch.from_numpy(self.x_st.view(np.int16)).to(device).view(torch.bfloat16)
            w = torch.from_numpy(self.w_st.view(np.int16)).to(device).view(torch.bfloat16)
        bias = None if self.bias is None else torch.from_numpy(self.bias.astype(np.float32)).to(device)
        out = dict(x=x, w_r=w, bias=bias)
        if hasattr(self, "q_bits"):
            for n in ("q", "k", "v"):
                out[n] = torch.from_numpy(getattr(self, n + "_bits").view(np.int16)).to(device).view(torch.bfloat16)
        return out


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# tolerances for attention outputs computed from bf16 inputs (fp32 accumulate,
# bf16 probabilities in the P.V product)
REL_L2 = 1e-2
MAX_ABS = 3e-2
LOSS_REL = 1e-5
GATE_REL = 1e-5


def assert_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert r <= REL_L2 and m <= MAX_ABS, "%s: rel-L2 %.3e (<= %.0e), max-abs %.3e (<= %.0e)" % (what, r, REL_L2, m,
                                                                                             MAX_ABS)
    return r, m
