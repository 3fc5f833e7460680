"""GPU parity: router, permute and balance loss against the fp64 oracle.

Group ids, perm, cu_seqlens, counts and max_seqlen must be bit-exact (inputs
carry a top-2 routing margin of at least 1e-3); gate probabilities agree to a
relative 1e-5 (fp32 softmax of M values); L_gb to a relative 1e-5.
"""
import numpy as np
import pytest

from _data import GATE_REL, LOSS_REL, Case
from oracle import layer as olayer
from oracle import permute as opermute
from synth import workloads as W

pytestmark = pytest.mark.gpu

EDGE = W.Workload("edge_300", T=5, h=6, w=10, d=64, H=3, hd=128, M=7, shots=(2, 1, 2), tg_max=2,
                  win_h=3, win_w=5)

CASES = {
    "tiny": W.TINY,
    "wan13b_5s": W.WAN13B_5S,
    "multishot_skewed": W.MULTISHOT_10S,
    "edge_M7_N300": EDGE,
    "edge_M1": EDGE.with_(name="edge_M1", M=1),
    "edge_M32": EDGE.with_(name="edge_M32", M=32, T=7, shots=(3, 4)),
    "edge_N1": W.Workload("edge_N1", T=1, h=1, w=1, d=16, H=1, hd=64, M=3, shots=(1,), tg_max=0,
                          win_h=1, win_w=1),
    "edge_f32_ragged": W.Workload("edge_f32", T=3, h=7, w=9, d=24, H=1, hd=64, M=5, shots=(3,), tg_max=0,
                                  win_h=7, win_w=9, x_dtype="f32"),
    # fp32 path over many 128-token blocks, ragged last block, d not a multiple of 64, M > 16
    "f32_blocks_M20": W.Workload("f32_blocks", T=4, h=17, w=19, d=136, H=1, hd=64, M=20, shots=(4,), tg_max=0,
                                 win_h=17, win_w=19, x_dtype="f32"),
    # bf16 tensor-core path: 151 chunks of 32 tokens (more chunks than SMs, so
    # some CTAs take two), ragged last chunk, ragged last k slice, 32-column MMA
    "bf16_chunks_M17": W.Workload("bf16_chunks", T=5, h=31, w=31, d=200, H=1, hd=64, M=17, shots=(5,),
                                  tg_max=0, win_h=31, win_w=31),
    # bf16, M = 16 (largest 16-column MMA), fewer chunks than SMs
    "bf16_M16": W.Workload("bf16_M16", T=2, h=9, w=11, d=1024, H=1, hd=64, M=16, shots=(2,), tg_max=0,
                           win_h=9, win_w=11),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def routed(request, cuda_device):
    import sparse_attention_long_moga_b200 as moga
    case = Case(CASES[request.param], with_qkv=False)
    t = case.gpu()
    g, gate, ws = moga.moga_route(t["x"], t["w_r"], t["bias"])
    M = case.wl.M
    perm, cu, counts, mx = moga.moga_permute(g, M)
    loss = moga.moga_balance_loss(counts, ws, case.wl.N, M, case.wl.alpha)
    moga.device_status()
    return case, dict(g=g.cpu().numpy(), gate=gate.cpu().numpy(), perm=perm.cpu().numpy(), cu=cu.cpu().numpy(),
                      counts=counts.cpu().numpy(), mx=int(mx.item()), loss=float(loss.item()))


def test_group_ids_bit_exact(routed):
    case, got = routed
    g, p_g, p = case.route64()
    assert np.array_equal(got["g"], g.astype(np.int32))


def test_gate_prob(routed):
    case, got = routed
    g, p_g, p = case.route64()
    np.testing.assert_allclose(got["gate"], p_g, rtol=GATE_REL, atol=0)


def test_permute_bit_exact(routed):
    case, got = routed
    g, _, _ = case.route64()
    perm, cu, counts, mx = opermute.permute(g, case.wl.M)
    assert np.array_equal(got["perm"], perm.astype(np.int32))
    assert np.array_equal(got["cu"], cu.astype(np.int32))
    assert np.array_equal(got["counts"], counts.astype(np.int32))
    assert got["mx"] == mx


def test_balance_loss(routed):
    case, got = routed
    g, _, p = case.route64()
    counts = np.bincount(g, minlength=case.wl.M)
    ref = olayer.balance_loss(counts, p, case.wl.alpha)
    assert got["loss"] == pytest.approx(ref, rel=LOSS_REL)


def test_skewed_router_fraction(cuda_device):
    case = Case(W.MULTISHOT_10S, with_qkv=False)
    g, _, _ = case.route64()
    assert 0.395 <= np.mean(g == 0) <= 0.405


@pytest.mark.parametrize("N,M,skew", [(1, 1, 0.0), (31, 5, 0.0), (33, 32, 0.0), (1024, 5, 0.9), (32760, 32, 0.0),
                                      (65535, 5, 0.6), (65536, 32, 0.0), (65537, 5, 0.0), (100000, 32, 0.99),
                                      (65536, 1, 0.0)])
def test_permute_sizes_bit_exact(N, M, skew, cuda_device):
    """The permute on random ids, a share `skew` of them in group 0, from one
    token to several 2048-token tiles with ragged tails and up to 32 groups:
    bit-exact against the oracle."""
    import torch
    import sparse_attention_long_moga_b200 as moga
    rs = np.random.default_rng(N + M)
    g = rs.integers(0, M, N).astype(np.int32)
    g[rs.random(N) < skew] = 0
    perm, cu, counts, mx = moga.moga_permute(torch.from_numpy(g).to(cuda_device), M)
    moga.device_status()
    rp, rcu, rcounts, rmx = opermute.permute(g, M)
    assert np.array_equal(perm.cpu().numpy(), rp.astype(np.int32))
    assert np.array_equal(cu.cpu().numpy(), rcu.astype(np.int32))
    assert np.array_equal(counts.cpu().numpy(), rcounts.astype(np.int32))
    assert int(mx.item()) == rmx
