"""Counter-based random numbers for the synthetic workloads.

Every random value is a pure function of (seed, stream, draw, element index),
so any subset of a tensor can be regenerated without generating the rest:
the CPU oracle can rebuild only the rows it samples, and a row whose inputs
must be replaced is regenerated from the next `draw` of its own counters.

Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; constants as published with
S. Vigna's reference version).  Normals: the Box-Muller transform (G. Box,
M. Muller, 1958), cosine branch only, one normal per 64-bit output.

This module holds input generation only; it performs none of the attention
layer's arithmetic.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied elementwise (uint64, wrapping)."""
    z = (z ^ (z >> np.uint64(30))) * _MIX1
    z = (z ^ (z >> np.uint64(27))) * _MIX2
    return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, stream: int, draw: int) -> np.uint64:
    """64-bit starting state of one (seed, stream, draw) counter sequence."""
    with np.errstate(over="ignore"):
        s = np.array([seed], dtype=np.uint64)
        s = _mix64(s + _GAMMA * np.uint64(stream + 1))
        s = _mix64(s + _GAMMA * np.uint64(draw + 0x51))
    return s[0]


def uint64(seed: int, stream: int, index: np.ndarray, draw: int = 0) -> np.ndarray:
    """SplitMix64 outputs number `index` (0-based) of the given sequence."""
    idx = np.asarray(index, dtype=np.uint64)
    base = _stream_base(seed, stream, draw)
    with np.errstate(over="ignore"):
        return _mix64(base + (idx + np.uint64(1)) * _GAMMA)


def uniform01(seed: int, stream: int, index: np.ndarray, draw: int = 0) -> np.ndarray:
    """Uniform doubles in [0, 1) from the top 53 bits."""
    u = uint64(seed, stream, index, draw)
    return (u >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(seed: int, stream: int, index: np.ndarray, draw: int = 0) -> np.ndarray:
    """Standard normals, one per counter (Box-Muller, cosine branch)."""
    u = uint64(seed, stream, index, draw)
    hi = (u >> np.uint64(32)).astype(np.float64)
    lo = (u & np.uint64(0xFFFFFFFF)).astype(np.float64)
    u1 = (hi + 1.0) * (1.0 / 4294967296.0)  # (0, 1]
    u2 = lo * (1.0 / 4294967296.0)  # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def normal_block(seed: int, stream: int, rows: np.ndarray, ncols: int,
                 draw: int = 0, row_stride: int | None = None) -> np.ndarray:
    """Normals for the listed rows of a row-major [*, ncols] tensor.

    Element (r, c) uses counter r * row_stride + c (row_stride defaults to
    ncols), so a row's values do not depend on which other rows are asked for.
    """
    rows = np.asarray(rows, dtype=np.int64)
    stride = ncols if row_stride is None else row_stride
    idx = rows[:, None].astype(np.uint64) * np.uint64(stride) + np.arange(ncols, dtype=np.uint64)[None, :]
    return normal(seed, stream, idx, draw)


def permutation(seed: int, stream: int, n: int, draw: int = 0) -> np.ndarray:
    """A permutation of range(n): indices sorted by their 64-bit counter output."""
    keys = uint64(seed, stream, np.arange(n, dtype=np.uint64), draw)
    return np.argsort(keys, kind="stable")
