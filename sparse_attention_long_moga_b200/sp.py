"""Sequence-parallel forward of the layer over the ranks of a process group.

MoGA note, key design 2 (and the translation's method section): under
sequence parallelism each rank routes its own tokens, which carry every head,
the routing results of all tokens are collected, and only then is the
sequence gathered / the heads scattered for attention.  With P ranks, rank r
holding the n = N / P consecutive tokens [r n, (r+1) n) of one video:

  1. route the local tokens (g, gate, router workspace)
  2. all-gather g and gate: every rank holds the routing of all N tokens
  3. all-to-all Q, K, V: sequence shards [n][H][hd] -> head shards
     [N][H/P][hd] (heads [r H/P, (r+1) H/P) of every token)
  4. permute all N tokens (identical on every rank), MoGA, STGA and the
     mean for the local heads
  5. all-to-all the output back: [N][H/P][hd] -> [n][H][hd]
  6. L_gb: each rank's share (global F_i, its own tokens' P_i), all-reduced

Collectives go through torch.distributed (NCCL on GPUs); every local step is
one of the library's kernels (the `CudaOps` below).  The exchange logic takes
its local steps from an `ops` object so that it can be exercised on CPU with
other implementations of the same steps.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import _ptr, _stream, check, lib, moga_group_attn, moga_permute, moga_route, stga_attn, visual_attn_mean


class CudaOps:
    """The local steps on this rank's GPU, through the C ABI."""

    def route(self, x, w_r, bias):
        return moga_route(x, w_r, bias)

    def permute(self, g, M: int):
        return moga_permute(g, M)

    def pack_heads(self, t: torch.Tensor, P: int) -> torch.Tensor:
        n, H, hd = t.shape
        out = torch.empty((P * n, H // P, hd), dtype=t.dtype, device=t.device)
        check(lib().moga_sp_pack_heads(_ptr(t), n, H, hd, P, _ptr(out), _stream()), "moga_sp_pack_heads")
        return out

    def unpack_heads(self, t: torch.Tensor, n: int, H: int, hd: int, P: int) -> torch.Tensor:
        out = torch.empty((n, H, hd), dtype=t.dtype, device=t.device)
        check(lib().moga_sp_unpack_heads(_ptr(t), n, H, hd, P, _ptr(out), _stream()), "moga_sp_unpack_heads")
        return out

    def layer_heads(self, q, k, v, perm, cu, gate, M: int, geom: dict, scale: float):
        o = moga_group_attn(q, k, v, perm, cu, gate, M, scale)
        stga_attn(q, k, v, geom, scale, o_acc=o)
        return visual_attn_mean(o)

    def loss_part(self, counts, route_ws, n: int, N: int, M: int, alpha: float):
        loss = torch.empty(1, dtype=torch.float64, device=counts.device)
        check(lib().moga_balance_loss_part(_ptr(counts), _ptr(route_ws), n, N, M, alpha, _ptr(loss), _stream()),
              "moga_balance_loss_part")
        return loss


def _all_gather_cat(t: torch.Tensor, P: int, group) -> torch.Tensor:
    parts = [torch.empty_like(t) for _ in range(P)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.cat(parts)


def sp_visual_attention_forward(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float, group=None,
                                softmax_scale: float | None = None, ops=None) -> dict:
    """x [n, d], q/k/v [n, H, hd]: this rank's n consecutive tokens of one video
    of N = n * P tokens (geom describes the whole video).  Returns dict(out
    [n, H, hd], loss [1] (the whole video's L_gb, on every rank), g, gate of the
    local tokens, and the permute of all N tokens)."""
    P = dist.get_world_size(group)
    n = x.shape[0]
    H, hd = q.shape[1], q.shape[2]
    if H % P:
        raise ValueError("heads (%d) must be a multiple of the ranks (%d)" % (H, P))
    if q.shape[0] != n or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("x, q, k, v must hold the same n tokens")
    N = n * P
    if N != geom["T"] * geom["h"] * geom["w"]:
        raise ValueError("n * P = %d tokens does not match the geometry" % N)
    ops = CudaOps() if ops is None else ops
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    g, gate, route_ws = ops.route(x, w_r, bias)
    g_all = _all_gather_cat(g, P, group)
    gate_all = _all_gather_cat(gate, P, group)
    heads = []
    for t in (q, k, v):
        send = ops.pack_heads(t, P)
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)   # -> [N][H/P][hd], token order
        heads.append(recv)
    perm, cu, counts, max_seqlen = ops.permute(g_all, M)
    out_h = ops.layer_heads(heads[0], heads[1], heads[2], perm, cu, gate_all, M, geom, scale)
    back = torch.empty_like(out_h)
    dist.all_to_all_single(back, out_h.contiguous(), group=group)   # chunk j: rank j's heads, local tokens
    out = ops.unpack_heads(back, n, H, hd, P)
    loss = ops.loss_part(counts, route_ws, n, N, M, alpha)
    dist.all_reduce(loss, group=group)
    return dict(out=out, loss=loss, g=g, gate=gate, perm=perm, cu_seqlens=cu, counts=counts, max_seqlen=max_seqlen)


__all__ = ["CudaOps", "sp_visual_attention_forward"]
