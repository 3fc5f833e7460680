"""GPU parity of the router fused into the Q/K/V projection against the oracle.

Q, K, V: the kernel accumulates in fp32 (the tensor core's accumulation
truncates: up to one unit in the last place per K = 16 step) and rounds to
bf16.  Every element must lie within one bf16 unit of the fp64 product plus
the accumulation bound (d / 16) * 2^-23 * sum_k |x_k w_k| (which also covers
results that cancel to near zero); the elements whose bf16 value differs from
the rounded fp64 product are those near a rounding boundary, a share that
grows with d (2.8e-3 at d = 5120), checked to stay below 1e-2.  Routing: group ids
bit-exact (inputs pass the 1e-3 router-margin filter), the gate within 1e-5
relative, and the per-32-token sums it leaves in the workspace give the
balance loss within 1e-5 of the oracle's.
"""
import numpy as np
import pytest

from _data import GATE_REL, LOSS_REL, Case
from oracle import layer as olayer
from oracle import permute as opermute
from oracle import projection
from synth import workloads as W

pytestmark = pytest.mark.gpu

CASES = {
    # ragged N (not a multiple of 128) and d (not a multiple of 64): both tails
    "ragged_1000_d136_m4": W.Workload("qkv_ragged", T=5, h=8, w=25, d=136, H=3, hd=64, M=4, shots=(5,), tg_max=0,
                                      win_h=8, win_w=25, seed=11),
    "tiny_bf16_m20": W.Workload("qkv_tiny_m20", T=8, h=16, w=16, d=128, H=2, hd=128, M=20, shots=(8,), tg_max=0,
                                win_h=8, win_w=8, seed=12),
    # the widest router input of the suite: 80 k stages, 20 per router slot
    "d5120_m5": W.Workload("qkv_d5120", T=4, h=16, w=16, d=5120, H=2, hd=128, M=5, shots=(4,), tg_max=0, win_h=8,
                           win_w=8, seed=13),
    "wan1.3b_32k": W.WAN13B_5S,
}


def _weights(wl):
    ws = [W.proj_weight_bits(wl, which) for which in "qkv"]      # [d, H*hd] each
    return np.ascontiguousarray(np.concatenate(ws, axis=1).T)     # [3*H*hd, d]


@pytest.mark.parametrize("name", sorted(CASES))
def test_qkv_route_matches_oracle(name, cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    wl = CASES[name]
    case = Case(wl, with_qkv=False)
    t = case.gpu(cuda_device)
    wbits = _weights(wl)
    w_qkv = torch.from_numpy(wbits.view(np.int16)).to(cuda_device).view(torch.bfloat16)
    q, k, v, g, gate, ws = moga.moga_qkv_route(t["x"], w_qkv, t["w_r"], t["bias"], wl.H, wl.hd)
    perm, cu, cnt, mx = moga.moga_permute(g, wl.M)
    loss = moga.moga_balance_loss(cnt, ws, wl.N, wl.M, wl.alpha)
    moga.device_status()
    x64 = case.x64()
    w64 = W.bf16_bits_to_f64(wbits)
    rq, rk, rv = projection.qkv(x64, w64, wl.H, wl.hd)
    mags = projection.qkv(np.abs(x64), np.abs(w64), wl.H, wl.hd)   # sum_k |x_k w_k|
    for got, ref, mag, which in ((q, rq, mags[0], "q"), (k, rk, mags[1], "k"), (v, rv, mags[2], "v")):
        gb = got.view(torch.int16).cpu().numpy().view(np.uint16)
        diff = gb != W.to_bf16_bits(ref)
        assert diff.mean() <= 1e-2, "%s %s: %.2e of the elements differ" % (name, which, diff.mean())
        err = np.abs(W.bf16_bits_to_f64(gb) - ref)
        bound = 2.0 ** -8 * np.abs(ref) + (wl.d / 16) * 2.0 ** -23 * mag
        assert np.all(err <= bound), "%s %s: worst error / bound %.3f" % (name, which, float(np.max(err / bound)))
    rg, rpg, rp = case.route64()
    assert np.array_equal(g.cpu().numpy(), rg)
    gr = gate.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(gr - rpg) / rpg) <= GATE_REL
    counts = opermute.permute(rg, wl.M)[2]
    ref_loss = olayer.balance_loss(counts, rp, wl.alpha)
    assert abs(float(loss.item()) - ref_loss) <= LOSS_REL * abs(ref_loss)
