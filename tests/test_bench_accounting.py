"""The work the benchmark divides by (its roofline `achieved` and the layer
TFLOP/s) against a count made independently from the oracle's own groups.

Attention FLOPs are 4 * H * hd per visible (query, key) pair.  The benchmark
counts the static branches from the geometry in closed form (run lengths,
borrowed frames per side, windows per frame) and MoGA from the group counts;
here the same totals come from enumerating every window group, frame group
and routed group the oracle builds and summing n_q * n_kv, or, for MoGA on a
small case, from the dense same-group mask.
"""
import numpy as np
import pytest

import bench
from oracle import permute as opermute
from oracle import stga as ostga
from synth import workloads as W

CASES = [
    W.TINY,
    W.WAN13B_5S,
    W.MULTISHOT_10S,
    W.WAN14B_30S_M5,
    W.LONG_60S,   # the benchmark's headline workload: ten shots, borrowed frames at nine cuts
    # a middle shot shorter than the borrowed-frame count, temporal groups of 2
    W.Workload("acct_short_shot", T=5, h=6, w=10, d=64, H=3, hd=128, M=7, shots=(2, 1, 2), tg_max=2, win_h=3,
               win_w=5),
    # several runs per shot, ragged run lengths, four shots
    W.Workload("acct_runs", T=23, h=8, w=8, d=64, H=2, hd=64, M=4, shots=(7, 5, 9, 2), tg_max=3, win_h=4,
               win_w=4, aug=3),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_stga_flops_equal_enumerated_groups(wl):
    geom = W.stga_shape(wl)
    pairs = sum(len(q) * len(kv) for q, kv in ostga.window_groups(geom))
    pairs += sum(len(q) * len(kv) for q, kv in ostga.frame_groups(geom))
    assert bench.stga_flops(wl) == 4.0 * wl.H * wl.hd * pairs


def test_stga_flops_of_the_bench_workload():
    # window groups: 4 windows x 3 runs of 7 frames x (7 * 390)^2; frames: 21 x 1560^2
    wl = W.WAN13B_5S
    assert bench.stga_flops(wl) == 4.0 * 12 * 128 * (4 * 3 * (7 * 390) ** 2 + 21 * 1560 ** 2)


@pytest.mark.parametrize("N,M", [(1, 1), (300, 7), (2000, 5)])
def test_moga_flops_equal_dense_mask(N, M):
    rs = np.random.default_rng(N * 31 + M)
    g = rs.integers(0, M, N)
    g[rs.random(N) < 0.3] = 0
    counts = opermute.permute(g, M)[2]
    pairs = int(np.count_nonzero(g[:, None] == g[None, :]))
    assert bench.moga_flops(counts, 3, 64) == 4.0 * 3 * 64 * pairs


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_cpu_baseline_row_costs_match_flop_count(wl):
    """The CPU baseline scales its sampled attention rows to the whole layer by
    the keys each (token, head) row attends over in the three branches; summed
    over all rows (times 4 hd) that must be exactly the benchmark's FLOP count
    of the three branches."""
    rs = np.random.default_rng(5)
    g = rs.integers(0, wl.M, wl.N)
    counts = np.bincount(g, minlength=wl.M)
    kv_win = np.zeros(wl.N, dtype=np.int64)
    for qt, kvt in ostga.window_groups(W.stga_shape(wl)):
        kv_win[qt] = len(kvt)
    cost_tok = counts[g] + kv_win + wl.hw
    flops_from_rows = 4.0 * wl.hd * float(cost_tok.sum()) * wl.H
    assert flops_from_rows == bench.moga_flops(counts, wl.H, wl.hd) + bench.stga_flops(wl)


def test_traffic_figures_scale_with_the_elements_moved():
    """`roofline.traffic` is the attention launch's captured DRAM bytes, the
    call's figure adds its gather copy; both are per launch on the captured
    workload and proportional to N * H * hd elsewhere."""
    wl = W.resolved(W.WAN13B_5S)
    kern, src = bench.scaled_traffic(wl, bench.KERNEL_TRAFFIC_BYTES, "kernel")
    call, _ = bench.scaled_traffic(wl, bench.CALL_TRAFFIC_BYTES, "call")
    assert "captured on this workload" in src
    assert (kern, call) == (bench.KERNEL_TRAFFIC_BYTES, bench.CALL_TRAFFIC_BYTES)
    # the gather copy reads and writes Q, K, V once: it sits between the
    # algorithmic bytes of one read + one write of Q, K, V (2 x 302 MB) and
    # the copy's written bytes alone
    gather = call - kern
    qkv = 3 * wl.N * wl.H * wl.hd * 2
    assert qkv < gather <= 2 * qkv
    # the attention launch reads Q, K, V once and writes the fp32 output at
    # most once: its traffic stays within the algorithmic bytes' band
    alg = 4 * wl.N * wl.H * wl.hd * 2 + 4 * wl.N
    assert 1.0 <= kern / alg < 1.5
    big = W.resolved(W.LONG_60S)
    k2, src2 = bench.scaled_traffic(big, bench.KERNEL_TRAFFIC_BYTES, "kernel")
    assert "scaled by N*H*hd" in src2
    assert k2 == pytest.approx(kern * (big.N * big.H * big.hd) / (wl.N * wl.H * wl.hd), rel=1e-12)
