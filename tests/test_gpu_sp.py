"""GPU side of the sequence-parallel path.

The head pack / unpack kernels are pure data movement: bit-exact against the
layout they are defined by (numpy reshape and transpose).  With one rank
(an NCCL group of one GPU) the whole sequence-parallel forward must equal the
single-GPU forward bit for bit (same kernels on the same data; the
collectives are copies), and, on the tiny workload, match the fp64 oracle's
layer forward directly (routing and perm bit-exact, output within the
attention tolerance, loss to 1e-5).  The multi-rank exchange is covered on
CPU by tests/test_sp_cpu.py.
"""
import datetime
import socket

import numpy as np
import pytest

from _data import LOSS_REL, Case, assert_close
from oracle import layer as olayer
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,H,hd,P", [(1000, 12, 128, 2), (777, 12, 128, 3), (512, 40, 128, 8), (300, 2, 64, 2),
                                      (64, 4, 64, 4), (33, 12, 64, 1)])
def test_pack_unpack_heads_bit_exact(n, H, hd, P, cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    from sparse_attention_long_moga_b200.sp import CudaOps
    rs = np.random.default_rng(n + H + P)
    bits = rs.integers(0, 1 << 16, (n, H, hd), dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).to(cuda_device).view(torch.bfloat16)
    ops = CudaOps()
    packed = ops.pack_heads(t, P)
    want = bits.reshape(n, P, H // P, hd).transpose(1, 0, 2, 3).reshape(P * n, H // P, hd)
    assert np.array_equal(packed.view(torch.int16).cpu().numpy().view(np.uint16), want)
    back = ops.unpack_heads(packed, n, H, hd, P)
    moga.device_status()
    assert np.array_equal(back.view(torch.int16).cpu().numpy().view(np.uint16), bits)


def test_pack_rejects_heads_not_divisible(cuda_device):
    import torch
    from sparse_attention_long_moga_b200 import MogaError
    from sparse_attention_long_moga_b200.sp import CudaOps
    t = torch.zeros((16, 12, 64), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(MogaError):
        CudaOps().pack_heads(t, 5)


@pytest.fixture(scope="module")
def nccl_world_of_one(cuda_device):
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny_2k", "wan1.3b_5s_1shot_32k"])
def test_sp_one_rank_equals_single_gpu(name, nccl_world_of_one, cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    from sparse_attention_long_moga_b200.sp import sp_visual_attention_forward
    case = Case(W.SUITE[name], with_qkv=True)
    wl = case.wl
    t = case.gpu(cuda_device)
    ref = moga.visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], wl.M, case.geom,
                                        wl.alpha, fused_mean=False)
    got = sp_visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], wl.M, case.geom, wl.alpha)
    moga.device_status()
    assert torch.equal(got["out"], ref["out"])
    assert torch.equal(got["perm"], ref["perm"])
    assert float(got["loss"].item()) == float(ref["loss"].item())


def test_sp_one_rank_against_oracle(nccl_world_of_one, cuda_device):
    """The sequence-parallel forward checked against the oracle itself, not only
    against the single-GPU CUDA path."""
    import sparse_attention_long_moga_b200 as moga
    from sparse_attention_long_moga_b200.sp import sp_visual_attention_forward
    case = Case(W.TINY, with_qkv=True)
    wl = case.wl
    t = case.gpu(cuda_device)
    got = sp_visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], wl.M, case.geom, wl.alpha)
    moga.device_status()
    q, k, v = case.qkv64()
    ref = olayer.forward(case.x64(), case.w64(), case.bias, q, k, v, wl.M, case.geom, wl.alpha)
    assert np.array_equal(got["perm"].cpu().numpy(), ref["perm"].astype(np.int32))
    assert_close(got["out"].float().cpu().numpy(), ref["out"], "sp layer output")
    assert abs(float(got["loss"].item()) - ref["loss"]) <= LOSS_REL * abs(ref["loss"])
