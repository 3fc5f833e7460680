"""GPU parity of the batched layer (B videos, per-video groups) against the
batched oracle.

The batched permute is integer work: perm, cu_seqlens, counts and
max_seqlen must match the oracle bit for bit, for B * M keys from 12 up to
the 1024 the call supports (many videos per 2048-token tile included).  The
whole batched layer is compared on small videos: routing bit-exact, out
within the forward's rel-L2 1e-2 / max-abs 3e-2, the loss within 1e-5
relative.  Each case draws its B videos as consecutive frames of one seeded
workload (so every token passes the router-margin filter against the one
shared W_r), then splits them into videos.
"""
import numpy as np
import pytest

from _data import LOSS_REL, Case, assert_close
from oracle import batch as obatch
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,M,n", [(1, 5, 32760), (3, 4, 3001), (2, 20, 5000), (64, 16, 300), (8, 20, 70000),
                                   (5, 7, 2048)])
def test_permute_batched_bit_exact(B, M, n, cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    rs = np.random.default_rng(B * 1000 + M)
    g = rs.integers(0, M, B * n).astype(np.int32)
    gt = torch.from_numpy(g).to(cuda_device)
    perm, cu, counts, mx = moga.moga_permute_batched(gt, B, M)
    moga.device_status()
    rp, rcu, rcounts, rmx = obatch.permute_batched(g, B, M)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(cu.cpu().numpy(), rcu)
    assert np.array_equal(counts.cpu().numpy(), rcounts)
    assert int(mx.item()) == rmx
    if B == 1:
        p1, c1, n1, m1 = moga.moga_permute(gt, M)
        for a, b in ((perm, p1), (cu, c1), (counts, n1), (mx, m1)):
            assert torch.equal(a, b)


def test_permute_batched_rejects_too_many_keys(cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    g = torch.zeros(65 * 16, dtype=torch.int32, device=cuda_device)
    with pytest.raises(ValueError):
        moga.moga_permute_batched(g, 65, 16)   # 1040 keys > 1024


def _video_batch(B, per_video: W.Workload):
    """B videos of per_video's geometry drawn as consecutive frames of one workload."""
    big = per_video.with_(name="%s_x%d" % (per_video.name, B), T=per_video.T * B, shots=tuple(per_video.shots) * B)
    return Case(big), W.stga_shape(per_video)


CASES = {
    "tiny_b3_m4": (3, W.Workload("batch_video_2k", T=8, h=16, w=16, d=128, H=2, hd=64, M=4, shots=(4, 4), tg_max=0,
                                 win_h=8, win_w=8, aug=2, x_dtype="bf16", qkv="iid", seed=3)),
    "b2_m20_hd128": (2, W.Workload("batch_video_1k_m20", T=4, h=16, w=16, d=128, H=2, hd=128, M=20, shots=(2, 2),
                                   tg_max=0, win_h=8, win_w=8, aug=1, x_dtype="bf16", qkv="iid", seed=5)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_batched_layer_matches_oracle(name, cuda_device):
    import sparse_attention_long_moga_b200 as moga
    B, per = CASES[name]
    case, geom = _video_batch(B, per)
    n = per.T * per.h * per.w
    t = case.gpu(cuda_device)
    H, hd = per.H, per.hd
    res = moga.visual_attention_forward_batched(t["x"].view(B, n, -1), t["w_r"], t["bias"], t["q"].view(B, n, H, hd),
                                                t["k"].view(B, n, H, hd), t["v"].view(B, n, H, hd), per.M, geom,
                                                per.alpha)
    moga.device_status()
    q, k, v = (a.reshape(B, n, H, hd) for a in case.qkv64())
    ref = obatch.forward_batched(case.x64().reshape(B, n, -1), case.w64(), case.bias, q, k, v, per.M, geom,
                                 per.alpha)
    assert np.array_equal(res["g"].cpu().numpy(), ref["g"])
    assert np.array_equal(res["perm"].cpu().numpy(), ref["perm"])
    assert np.array_equal(res["cu_seqlens"].cpu().numpy(), ref["cu_seqlens"])
    assert np.array_equal(res["counts"].cpu().numpy(), ref["counts"])
    assert_close(res["out"].float().cpu().numpy(), ref["out"], "batched out " + name)
    assert abs(float(res["loss"].item()) - ref["loss"]) <= LOSS_REL * abs(ref["loss"])
