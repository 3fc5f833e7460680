"""GPU parity at the full sizes of the long-video workloads, on sampled outputs.

30 s multi-shot (282,360 tokens, 40 heads, M = 5 and M = 20) and 60 s ten-shot
clustered (563,160 tokens, M = 20).  Routing, permutation and the balance loss
are compared on every token (bit-exact ids/perm/cu_seqlens/counts, loss to a
relative 1e-5); the MoGA branch, the two static branches and the layer output
are compared on a stratified sample of tokens for a sample of heads, each
sampled row computed by the oracle from its full definition.
"""
import numpy as np
import pytest

from _data import GATE_REL, LOSS_REL, assert_close
from oracle import attention as oatt
from oracle import layer as olayer
from oracle import permute as opermute
from oracle import route as oroute
from oracle import stga as ostga
from synth import workloads as W

pytestmark = pytest.mark.gpu

CASES = [W.WAN14B_30S_M5, W.WAN14B_30S_M20, W.LONG_60S]
HEADS = (0, 17, 39)


def _route_all(wl, redraw, x_st):
    w = W.w_r_f64(wl)
    g = np.empty(wl.N, dtype=np.int64)
    p_g = np.empty(wl.N)
    p = np.empty((wl.N, wl.M))

    def fill(a, b):
        x = W.bf16_bits_to_f64(x_st[a:b])
        gg, pg, pp = oroute.route(x, w, W.bias_f64(wl))
        g[a:b], p_g[a:b], p[a:b] = gg, pg, pp
    W._parallel_chunks(wl.N, 16384, fill)
    return g, p_g, p


def _sample(wl, g, seed=1):
    rs = np.random.default_rng(seed)
    toks = []
    for i in range(wl.M):
        mem = np.nonzero(g == i)[0]
        if len(mem):
            toks.append(rs.choice(mem, size=min(12, len(mem)), replace=False))
            toks.append(mem[-1:])
    starts = np.concatenate([[0], np.cumsum(wl.shots)])
    for f in sorted(set(int(s) for s in starts[:-1]) | set(int(s) - 1 for s in starts[1:])):
        toks.append(f * wl.hw + rs.integers(0, wl.hw, 3))
    return np.unique(np.concatenate(toks))


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_full_size_sampled(wl, cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    redraw = W.redraw_map(wl)
    assert redraw or wl.M == 1, "stored margin redraws missing for " + wl.name
    x_st = W.x_stored(wl, redraw)
    w_st = W.w_r_stored(wl)
    qb, kb, vb = (W.qkv_stored(wl, n, redraw) for n in "qkv")
    dev = cuda_device

    def up(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    x, w_r, q, k, v = up(x_st), up(w_st), up(qb), up(kb), up(vb)
    gg, gate, rws = moga.moga_route(x, w_r, None)
    perm, cu, counts, mx = moga.moga_permute(gg, wl.M)
    loss = moga.moga_balance_loss(counts, rws, wl.N, wl.M, wl.alpha)
    ws = moga.attn_workspace(q)
    o = moga.moga_group_attn(q, k, v, perm, cu, gate, wl.M, ws=ws)
    moga.device_status()

    g, p_g, p = _route_all(wl, redraw, x_st)
    assert np.array_equal(gg.cpu().numpy(), g.astype(np.int32))
    np.testing.assert_allclose(gate.cpu().numpy(), p_g, rtol=GATE_REL, atol=0)
    operm, ocu, ocounts, omx = opermute.permute(g, wl.M)
    assert np.array_equal(perm.cpu().numpy(), operm.astype(np.int32))
    assert np.array_equal(cu.cpu().numpy(), ocu.astype(np.int32))
    assert np.array_equal(counts.cpu().numpy(), ocounts.astype(np.int32))
    assert int(mx.item()) == omx
    assert float(loss.item()) == pytest.approx(olayer.balance_loss(ocounts, p, wl.alpha), rel=LOSS_REL)

    toks = _sample(wl, g)
    tt = torch.from_numpy(toks).to(dev)
    hh = list(HEADS)
    o_m = o[tt][:, hh].cpu().numpy()
    o_fused = o.clone()
    moga.stga_attn(q, k, v, W.stga_shape(wl), o_acc=o, ws=ws)
    o_ms = o[tt][:, hh].cpu().numpy()
    out = moga.visual_attn_mean(o)
    out_s = out[tt][:, hh].float().cpu().numpy()
    # the mean fused into the frame pass gives the same bf16 output bit for bit
    out_f = moga.stga_attn_mean(q, k, v, W.stga_shape(wl), o_acc=o_fused, ws=ws)
    moga.device_status()
    assert torch.equal(out_f.view(torch.int16), out.view(torch.int16)), wl.name
    del o, o_fused, out, out_f, ws, q, k, v, x

    scale = 1.0 / np.sqrt(wl.hd)
    wgroups = ostga.window_groups(W.stga_shape(wl))
    owner = np.empty(wl.N, dtype=np.int64)
    for gi, (qt, _) in enumerate(wgroups):
        owner[qt] = gi
    ref_m = np.zeros((len(toks), len(hh), wl.hd))
    ref_s = np.zeros_like(ref_m)
    for j, h in enumerate(hh):
        qh, kh, vh = (W.bf16_bits_to_f64(a[:, h, :]) for a in (qb, kb, vb))
        for i in range(wl.M):
            sel = np.nonzero(g[toks] == i)[0]
            if len(sel):
                mem = operm[ocu[i]:ocu[i + 1]]
                ref_m[sel, j] = oatt.rows_of_group(qh[toks[sel]], kh[mem], vh[mem], scale, p_g[toks[sel]])
        for r, t in enumerate(toks.tolist()):
            _, kvt = wgroups[owner[t]]
            fr = slice((t // wl.hw) * wl.hw, (t // wl.hw + 1) * wl.hw)
            ref_s[r, j] = oatt.attend(qh[t:t + 1], kh[kvt], vh[kvt], scale)[0] + \
                oatt.attend(qh[t:t + 1], kh[fr], vh[fr], scale)[0]
    assert_close(o_m, ref_m, "moga " + wl.name)
    assert_close(o_ms - o_m, ref_s, "stga " + wl.name)
    assert_close(out_s, (ref_m + ref_s) / 3.0, "layer " + wl.name)
