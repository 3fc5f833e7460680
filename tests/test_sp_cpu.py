"""The sequence-parallel exchange on CPU: 2 and 3 gloo ranks, no GPU.

`sp_visual_attention_forward` takes its local steps from an ops object; here
they are the fp64 oracle's (test infrastructure), so the test checks the
exchange itself — the routing all-gather, the head-shard all-to-all, the
return all-to-all and the loss shares — against the oracle's single-process
forward of the whole video: the gathered outputs must match to rounding and
the loss to 1e-12.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GEOM = dict(T=4, h=4, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=0, aug=1)
N, D, M, HD = 64, 8, 3, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(H):
    rs = np.random.default_rng(21)
    return dict(x=rs.standard_normal((N, D)), w_r=rs.standard_normal((D, M)),
                q=rs.standard_normal((N, H, HD)), k=rs.standard_normal((N, H, HD)), v=rs.standard_normal((N, H, HD)))


class OracleOps:
    """The local steps in fp64 from the oracle (CPU tensors)."""

    def route(self, x, w_r, bias):
        from oracle import route
        g, p_g, p = route.route(x.numpy(), w_r.numpy(), None)
        return torch.from_numpy(g.astype(np.int64)), torch.from_numpy(p_g), torch.from_numpy(p)

    def permute(self, g, M):
        from oracle import permute
        perm, cu, counts, mx = permute.permute(g.numpy(), M)
        return torch.from_numpy(perm), torch.from_numpy(cu), torch.from_numpy(counts), mx

    def pack_heads(self, t, P):
        n, H, hd = t.shape
        return t.reshape(n, P, H // P, hd).transpose(0, 1).reshape(P * n, H // P, hd).contiguous()

    def unpack_heads(self, t, n, H, hd, P):
        return t.reshape(P, n, H // P, hd).transpose(0, 1).reshape(n, H, hd).contiguous()

    def layer_heads(self, q, k, v, perm, cu, gate, M, geom, scale):
        from oracle import attention, layer, stga
        q, k, v, g_all = q.numpy(), k.numpy(), v.numpy(), self.g_all
        o1 = attention.moga(q, k, v, g_all, gate.numpy(), M, scale)
        o2 = attention.grouped(q, k, v, stga.window_groups(geom), scale)
        o3 = attention.grouped(q, k, v, stga.frame_groups(geom), scale)
        return torch.from_numpy(layer.mean3(o1, o2, o3))

    def loss_part(self, counts, route_ws, n, N, M, alpha):
        F = counts.numpy().astype(np.float64) / N
        P = route_ws.numpy().sum(axis=0) / N
        return torch.tensor([alpha * M * float(np.sum(F * P))], dtype=torch.float64)


class _Ops(OracleOps):
    # the oracle's MoGA takes the group ids rather than perm/cu: keep the gathered ids
    def permute(self, g, M):
        self.g_all = g.numpy()
        return super().permute(g, M)


def _worker(rank, world, port, H, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from sparse_attention_long_moga_b200.sp import sp_visual_attention_forward
    inp = _inputs(H)
    n = N // world
    sl = slice(rank * n, (rank + 1) * n)
    t = {k: torch.from_numpy(np.ascontiguousarray(v[sl] if k != "w_r" else v)) for k, v in inp.items()}
    res = sp_visual_attention_forward(t["x"], t["w_r"], None, t["q"], t["k"], t["v"], M, GEOM, 0.1, ops=_Ops())
    q.put((rank, res["out"].numpy(), float(res["loss"].item())))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,H", [(2, 2), (2, 4), (4, 4)])
def test_sp_exchange_matches_single_process_oracle(world, H):
    from oracle import layer
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, H, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs(H)
    ref = layer.forward(inp["x"], inp["w_r"], None, inp["q"], inp["k"], inp["v"], M, GEOM, alpha=0.1)
    out = np.concatenate([r[1] for r in res])
    np.testing.assert_allclose(out, ref["out"], rtol=1e-12, atol=1e-13)
    for r in res:
        assert r[2] == pytest.approx(ref["loss"], rel=1e-12)


def test_sp_rejects_heads_not_divisible(monkeypatch):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from sparse_attention_long_moga_b200.sp import sp_visual_attention_forward
    monkeypatch.setattr(dist, "get_world_size", lambda group=None: 3)
    t = torch.zeros(4, 2, 4)
    with pytest.raises(ValueError):
        sp_visual_attention_forward(torch.zeros(4, 8), torch.zeros(8, 3), None, t, t, t, 3, GEOM, 0.1)
