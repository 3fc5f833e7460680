"""GPU parity at the full sizes of the long-video workloads, on sampled outputs.

30 s multi-shot (282,360 tokens, 40 heads, M = 5 and M = 20) and 60 s ten-shot
clustered (563,160 tokens, M = 20, the benchmark's default workload, run in
its launch configuration).  Routing, permutation and the balance loss are
compared on every token (bit-exact ids/perm/cu_seqlens/counts, loss to a
relative 1e-5).  The MoGA branch, the window branch, the frame branch (each
on its own) and the layer output are compared on a stratified sample of
>= 4096 (token, head) rows over 8 heads: every MoGA group (its first, last
and random members), every window group, one token per window in each of the
two frames on either side of every shot cut (the borrowed frames and the
queries that borrow them) and every frame; each sampled row is computed by
the oracle from its full definition.  The accumulating static call is
checked to add exactly the branch values, bit for bit.
"""
import numpy as np
import pytest

from _data import GATE_REL, LOSS_REL, assert_close
from oracle import layer as olayer
from oracle import permute as opermute
from oracle import route as oroute
from oracle import sample as osample
from synth import workloads as W

pytestmark = pytest.mark.gpu

CASES = [W.WAN14B_30S_M5, W.WAN14B_30S_M20, W.LONG_60S]


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


def _equal_chunked(a, b_fn, rows=65536):
    """a == b_fn(slice) bit for bit, in row chunks (bounded temporaries)."""
    import torch
    for r0 in range(0, a.shape[0], rows):
        sl = slice(r0, min(r0 + rows, a.shape[0]))
        if not torch.equal(a[sl], b_fn(sl)):
            return False
    return True


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
    geom = W.stga_shape(wl)

    def up(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    x, w_r, q, k, v = up(x_st), up(w_st), up(qb), up(kb), up(vb)
    gg, gate, rws = moga.moga_route(x, w_r, None)
    del x
    perm, cu, counts, mx = moga.moga_permute(gg, wl.M)
    loss = moga.moga_balance_loss(counts, rws, wl.N, wl.M, wl.alpha)
    ws = moga.attn_workspace(q)
    o = moga.moga_group_attn(q, k, v, perm, cu, gate, wl.M, ws=ws)
    o_win, _, o_frame, _ = moga.stga_attn_train(q, k, v, geom, ws=ws)
    acc = o.clone()
    moga.stga_attn(q, k, v, geom, o_acc=acc, ws=ws)
    moga.device_status()
    # the accumulating call adds the very values the split call writes
    assert _equal_chunked(acc, lambda sl: (o[sl] + o_win[sl]) + o_frame[sl]), wl.name
    # the three branches with one gather pass give the same bits
    del ws
    one = moga.visual_attn_branches(q, k, v, perm, cu, gate, wl.M, geom)
    moga.device_status()
    assert _equal_chunked(acc, lambda sl: one[sl]), wl.name
    del one
    ws = moga.attn_workspace(q)

    g, p_g, p = _route_all(wl, redraw, x_st)
    del x_st
    assert np.array_equal(gg.cpu().numpy(), g.astype(np.int32))
    np.testing.assert_allclose(gate.cpu().numpy(), p_g, rtol=GATE_REL, atol=0)
    operm, ocu, ocounts, omx = opermute.permute(g, wl.M)
    assert np.array_equal(perm.cpu().numpy(), operm.astype(np.int32))
    assert np.array_equal(cu.cpu().numpy(), ocu.astype(np.int32))
    assert np.array_equal(counts.cpu().numpy(), ocounts.astype(np.int32))
    assert int(mx.item()) == omx
    assert float(loss.item()) == pytest.approx(olayer.balance_loss(ocounts, p, wl.alpha), rel=LOSS_REL)

    rows = osample.stratified_rows(geom, g, wl.M, wl.H, n_heads=8, per_head=512)
    assert sum(len(t) for t in rows.values()) >= 4096

    def take(t):
        return {h: t[torch.from_numpy(toks).to(dev), h].float().cpu().numpy() for h, toks in rows.items()}
    got = dict(moga=take(o), win=take(o_win), frame=take(o_frame))
    del o_win, o_frame
    out = moga.visual_attn_mean(acc)
    got["out"] = take(out)
    # the mean fused into the frame pass gives the same bf16 output bit for bit
    out_f = moga.stga_attn_mean(q, k, v, geom, o_acc=o, ws=ws)
    moga.device_status()
    assert torch.equal(out_f.view(torch.int16), out.view(torch.int16)), wl.name
    del o, acc, out, out_f, ws, q, k, v

    scale = 1.0 / np.sqrt(wl.hd)
    ref = {n: {} for n in got}
    for h, toks in rows.items():
        qh, kh, vh = (W.bf16_bits_to_f64(a[:, h, :]) for a in (qb, kb, vb))
        om, ow, of = osample.branch_rows(qh, kh, vh, toks, g, p_g, wl.M, geom, scale)
        ref["moga"][h], ref["win"][h], ref["frame"][h] = om, ow, of
        ref["out"][h] = olayer.mean3(om, ow, of)
    for n in got:
        a = np.concatenate([got[n][h] for h in rows])
        b = np.concatenate([ref[n][h] for h in rows])
        assert_close(a, b, "%s %s" % (n, wl.name))
