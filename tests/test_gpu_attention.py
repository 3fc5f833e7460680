"""GPU parity: MoGA group attention, the STGA window and frame branches (each on
its own) and the layer output vs the fp64 oracle.

Attention outputs from bf16 inputs must reach rel-L2 <= 1e-2 and max-abs
<= 3e-2, on every branch separately and on the output.  The branches come
from the training forward, which writes each to its own buffer with the same
kernels; the production call that adds both into the accumulator is checked
to equal their fp32 sum bit for bit.  Small cases are compared element by
element over every token and head; the 32k and 64k workloads are compared on
a stratified sample of >= 4096 (token, head) rows over 8 heads covering every
MoGA group, every window group, both sides of every shot cut and every frame,
each sampled row computed by the oracle from its full definition.
"""
import numpy as np
import pytest

from _data import Case, assert_close
from oracle import attention as oatt
from oracle import layer as olayer
from oracle import sample as osample
from oracle import stga as ostga
from synth import workloads as W

pytestmark = pytest.mark.gpu

EDGE = W.Workload("edge_300", T=5, h=6, w=10, d=64, H=3, hd=128, M=7, shots=(2, 1, 2), tg_max=2,
                  win_h=3, win_w=5)

SMALL = {
    "tiny_hd64": W.TINY,
    "edge_M7_hd128": EDGE,
    "edge_M1_full_attention": EDGE.with_(name="edge_M1", M=1),
    "edge_M32_many_small_groups": EDGE.with_(name="edge_M32", M=32, T=7, shots=(3, 4)),
    "edge_one_frame_shots": EDGE.with_(name="edge_1f", T=4, shots=(1, 1, 1, 1), tg_max=1, aug=2),
    "edge_ragged_hd64": W.Workload("edge_rag", T=3, h=7, w=9, d=24, H=2, hd=64, M=3, shots=(2, 1),
                                   tg_max=0, win_h=7, win_w=3, aug=1),
    "mid_2shot": W.Workload("mid_2shot", T=6, h=10, w=20, d=64, H=2, hd=128, M=3, shots=(4, 2), tg_max=3,
                            win_h=5, win_w=10),
    # more work tiles than SMs, so every persistent CTA runs several tiles and
    # crosses tile boundaries (single key tiles; then tiles of one or two
    # query tiles over two to four key tiles)
    "many_tiles_M32_H40": EDGE.with_(name="edge_M32_H40", M=32, H=40),
    "many_tiles_M3_H64": W.Workload("mid_H64", T=6, h=10, w=20, d=64, H=64, hd=128, M=3, shots=(4, 2), tg_max=3,
                                    win_h=5, win_w=10),
}


def _run_gpu(case, q_scale=1.0):
    """Returns dict(moga, win, frame, static, out) as numpy fp32 and keeps the bf16 bit
    patterns of the fused and the two-call layer output in _run_gpu.last_bits."""
    import torch
    import sparse_attention_long_moga_b200 as moga
    t = case.gpu()
    if q_scale != 1.0:
        t["q"] = (t["q"].float() * q_scale).to(torch.bfloat16)
    g, gate, ws = moga.moga_route(t["x"], t["w_r"], t["bias"])
    perm, cu, counts, mx = moga.moga_permute(g, case.wl.M)
    o_moga = moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, case.wl.M)
    o_moga_cpu = o_moga.cpu().numpy().copy()
    o_static = moga.stga_attn(t["q"], t["k"], t["v"], case.geom)          # zero-initialised accumulator
    o_win, _, o_frame, _ = moga.stga_attn_train(t["q"], t["k"], t["v"], case.geom)
    # the accumulating call adds exactly the values the split call writes
    assert torch.equal(o_static, (torch.zeros_like(o_win) + o_win) + o_frame), case.wl.name
    # the three branches with one gather pass: the same bits as the two calls
    o_two = moga.stga_attn(t["q"], t["k"], t["v"], case.geom, o_acc=o_moga.clone())
    o_one = moga.visual_attn_branches(t["q"], t["k"], t["v"], perm, cu, gate, case.wl.M, case.geom)
    assert torch.equal(o_one, o_two), case.wl.name
    res = moga.visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], case.wl.M,
                                        case.geom, case.wl.alpha)
    res_unfused = moga.visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], case.wl.M,
                                                case.geom, case.wl.alpha, fused_mean=False)
    moga.device_status()
    # bf16 bit patterns of the fused and the two-call output
    _run_gpu.last_bits = (res["out"].view(torch.int16).cpu().numpy(),
                          res_unfused["out"].view(torch.int16).cpu().numpy())
    return dict(moga=o_moga_cpu, win=o_win.cpu().numpy(), frame=o_frame.cpu().numpy(),
                static=o_static.cpu().numpy(), out=res["out"].float().cpu().numpy())


@pytest.fixture(scope="module", params=sorted(SMALL))
def small(request, cuda_device):
    case = Case(SMALL[request.param])
    q, k, v = case.qkv64()
    g, p_g, p = case.route64()
    scale = 1.0 / np.sqrt(case.wl.hd)
    ref = dict(
        moga=oatt.moga(q, k, v, g, p_g, case.wl.M, scale),
        win=oatt.grouped(q, k, v, ostga.window_groups(case.geom), scale),
        frame=oatt.grouped(q, k, v, ostga.frame_groups(case.geom), scale),
    )
    ref["out"] = olayer.mean3(ref["moga"], ref["win"], ref["frame"])
    res = _run_gpu(case)
    return case, ref, res, _run_gpu.last_bits


def test_moga_attention_small(small):
    case, ref, res, _ = small
    assert_close(res["moga"], ref["moga"], "moga " + case.wl.name)


def test_stga_window_small(small):
    case, ref, res, _ = small
    assert_close(res["win"], ref["win"], "window " + case.wl.name)


def test_stga_frame_small(small):
    case, ref, res, _ = small
    assert_close(res["frame"], ref["frame"], "frame " + case.wl.name)


def test_stga_attention_small(small):
    case, ref, res, _ = small
    assert_close(res["static"], ref["win"] + ref["frame"], "stga " + case.wl.name)


def test_layer_output_small(small):
    case, ref, res, _ = small
    # the output is bf16: add its half-ulp rounding to the budget through the same tolerance
    assert_close(res["out"], ref["out"], "layer " + case.wl.name)


def test_fused_mean_equals_two_calls(small):
    """stga_attn_mean adds the frame term and divides by 3 in the same fp32 order as
    stga_attn + visual_attn_mean, so the bf16 outputs agree bit for bit."""
    case, _, _, (fused, unfused) = small
    assert np.array_equal(fused, unfused), case.wl.name


def test_peaky_queries(cuda_device):
    """Q scaled by 4 (exact in bf16) makes softmax far from flat, so rel-L2 is not passed trivially."""
    case = Case(EDGE.with_(name="edge_peaky"))
    q, k, v = case.qkv64()
    q = q * 4.0
    g, p_g, _ = case.route64()
    scale = 1.0 / np.sqrt(case.wl.hd)
    res = _run_gpu(case, q_scale=4.0)
    assert_close(res["moga"], oatt.moga(q, k, v, g, p_g, case.wl.M, scale), "peaky moga")
    assert_close(res["win"], oatt.grouped(q, k, v, ostga.window_groups(case.geom), scale), "peaky window")
    assert_close(res["frame"], oatt.grouped(q, k, v, ostga.frame_groups(case.geom), scale), "peaky frame")


@pytest.mark.parametrize("wl", [W.WAN13B_5S, W.MULTISHOT_10S], ids=lambda w: w.name)
def test_sampled_rows_full_size(wl, cuda_device):
    """Full-size workload in the benchmark's launch configuration; oracle on >= 4096
    stratified (token, head) rows, every branch on its own."""
    case = Case(wl)
    res = _run_gpu(case)
    g, p_g, _ = case.route64()
    rows = osample.stratified_rows(case.geom, g, wl.M, wl.H, n_heads=8, per_head=512)
    assert sum(len(t) for t in rows.values()) >= 4096
    scale = 1.0 / np.sqrt(wl.hd)
    got = {n: [] for n in ("moga", "win", "frame", "out")}
    ref = {n: [] for n in got}
    for h, toks in rows.items():
        qh, kh, vh = (case.head64(n, h) for n in ("q", "k", "v"))
        om, ow, of = osample.branch_rows(qh, kh, vh, toks, g, p_g, wl.M, case.geom, scale)
        for n, r in (("moga", om), ("win", ow), ("frame", of), ("out", olayer.mean3(om, ow, of))):
            ref[n].append(r)
            got[n].append(res[n][toks, h])
    for n in got:
        assert_close(np.concatenate(got[n]), np.concatenate(ref[n]), "%s sampled %s" % (n, wl.name))


def test_attention_timing_hook(cuda_device):
    """moga_test_set_attn_events brackets the attention launch of one call (not
    its gather copy), changes no result, and records nothing once switched off."""
    import ctypes
    import torch
    import sparse_attention_long_moga_b200 as moga
    case = Case(SMALL["many_tiles_M3_H64"])
    t = case.gpu()
    g, gate, _ = moga.moga_route(t["x"], t["w_r"], t["bias"])
    perm, cu, _, _ = moga.moga_permute(g, case.wl.M)
    hook = moga._lib.lib().moga_test_set_attn_events
    hook.restype = None
    hook.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    ref = moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, case.wl.M)
    a, b, c0, c1 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
    a.record()
    b.record()
    c0.record()
    hook(a, b)
    got = moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, case.wl.M)
    hook(None, None)
    c1.record()
    c1.synchronize()
    moga.device_status()
    assert torch.equal(got, ref)
    k_ms, c_ms = a.elapsed_time(b), c0.elapsed_time(c1)
    assert 0.0 < k_ms <= c_ms
    moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, case.wl.M)
    torch.cuda.synchronize()
    assert a.elapsed_time(b) == k_ms
