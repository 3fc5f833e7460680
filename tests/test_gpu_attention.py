"""GPU parity: MoGA group attention, STGA window + frame attention and the layer output vs the fp64 oracle.

Attention outputs from bf16 inputs must reach rel-L2 <= 1e-2 and max-abs
<= 3e-2.  Small cases are compared element by element over every token and
head; the 32k-token Wan-1.3B-shaped workload (the one the benchmark times) is
compared on a stratified sample of tokens over every head, each sampled row
computed by the oracle from its full definition.
"""
import numpy as np
import pytest

from _data import Case, assert_close
from oracle import attention as oatt
from oracle import layer as olayer
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
}


def _run_gpu(case, q_scale=1.0):
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
    o_static_cpu = o_static.cpu().numpy()
    res = moga.visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], case.wl.M,
                                        case.geom, case.wl.alpha)
    res_unfused = moga.visual_attention_forward(t["x"], t["w_r"], t["bias"], t["q"], t["k"], t["v"], case.wl.M,
                                                case.geom, case.wl.alpha, fused_mean=False)
    moga.device_status()
    out = res["out"].float().cpu().numpy()
    # bf16 bit patterns of the fused and the two-call output
    _run_gpu.last_bits = (res["out"].view(torch.int16).cpu().numpy(), res_unfused["out"].view(torch.int16).cpu().numpy())
    return o_moga_cpu, o_static_cpu, out


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
    case, ref, (o_moga, _, _), _ = small
    assert_close(o_moga, ref["moga"], "moga " + case.wl.name)


def test_stga_attention_small(small):
    case, ref, (_, o_static, _), _ = small
    assert_close(o_static, ref["win"] + ref["frame"], "stga " + case.wl.name)


def test_layer_output_small(small):
    case, ref, (_, _, out), _ = small
    # the output is bf16: add its half-ulp rounding to the budget through the same tolerance
    assert_close(out, ref["out"], "layer " + case.wl.name)


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
    o_moga, o_static, _ = _run_gpu(case, q_scale=4.0)
    assert_close(o_moga, oatt.moga(q, k, v, g, p_g, case.wl.M, scale), "peaky moga")
    ref = oatt.grouped(q, k, v, ostga.window_groups(case.geom), scale) + \
        oatt.grouped(q, k, v, ostga.frame_groups(case.geom), scale)
    assert_close(o_static, ref, "peaky stga")


def _sample_tokens(case, n_per_group=48, seed=0):
    """Stratified token sample: every MoGA group, every frame of shot boundaries, every window."""
    rs = np.random.default_rng(seed)
    g, _, _ = case.route64()
    toks = []
    for i in range(case.wl.M):
        mem = np.nonzero(g == i)[0]
        if len(mem):
            toks.append(rs.choice(mem, size=min(n_per_group, len(mem)), replace=False))
            toks.append(mem[-1:])   # the ragged tail row of the group
    hw = case.wl.hw
    starts = np.concatenate([[0], np.cumsum(case.wl.shots)])
    for f in sorted(set(int(s) for s in starts[:-1]) | set(int(s) - 1 for s in starts[1:])):
        toks.append(f * hw + rs.integers(0, hw, 8))
    return np.unique(np.concatenate(toks))


@pytest.mark.parametrize("wl", [W.WAN13B_5S, W.MULTISHOT_10S], ids=lambda w: w.name)
def test_sampled_rows_full_size(wl, cuda_device):
    """Full-size workload in the benchmark's launch configuration; oracle on sampled rows."""
    case = Case(wl)
    o_moga, o_static, out = _run_gpu(case)
    g, p_g, _ = case.route64()
    toks = _sample_tokens(case)
    scale = 1.0 / np.sqrt(wl.hd)
    wgroups = ostga.window_groups(case.geom)
    owner = {}
    for gi, (qt, _) in enumerate(wgroups):
        for t in qt.tolist():
            owner[t] = gi
    ref_m = np.zeros((len(toks), wl.H, wl.hd))
    ref_s = np.zeros_like(ref_m)
    for h in range(wl.H):
        qh, kh, vh = (case.head64(n, h) for n in ("q", "k", "v"))
        for i in range(wl.M):
            sel = np.nonzero(g[toks] == i)[0]
            if len(sel) == 0:
                continue
            mem = np.nonzero(g == i)[0]
            ref_m[sel, h] = oatt.rows_of_group(qh[toks[sel]], kh[mem], vh[mem], scale, p_g[toks[sel]])
        for j, t in enumerate(toks.tolist()):
            qt, kvt = wgroups[owner[t]]
            fr = np.arange((t // wl.hw) * wl.hw, (t // wl.hw + 1) * wl.hw)
            ref_s[j, h] = oatt.attend(qh[t:t + 1], kh[kvt], vh[kvt], scale)[0] + \
                oatt.attend(qh[t:t + 1], kh[fr], vh[fr], scale)[0]
    assert_close(o_moga[toks], ref_m, "moga sampled " + wl.name)
    assert_close(o_static[toks], ref_s, "stga sampled " + wl.name)
    assert_close(out[toks], (ref_m + ref_s) / 3.0, "layer sampled " + wl.name)
