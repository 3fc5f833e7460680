"""MoGA visual-attention layer forward on B200 (sm_100a).

Thin Python face of libmoga.so (include/moga.h).  Tensors are torch CUDA
tensors; torch supplies device memory and the current stream, the library's
kernels do every step of the layer:

    g, gate, ws = moga_route(x, w_r, bias)          # linear top-1 router
    perm, cu, counts, maxlen = moga_permute(g, M)   # stable group permute
    o = moga_group_attn(q, k, v, perm, cu, gate, M) # MoGA groups (o = ...)
    stga_attn(q, k, v, geom, o_acc=o)               # windows + frames (o += ...)
    out = visual_attn_mean(o)                       # bf16 (o / 3)
    # or, mean fused into the frame pass:
    # out = stga_attn_mean(q, k, v, geom, o_acc=o)
    loss = moga_balance_loss(counts, ws, N, M, a)   # L_gb (fp64 scalar)

`visual_attention_forward` chains the six calls.
"""
from __future__ import annotations

import ctypes
import math

import torch

from ._lib import MOGA_BF16, MOGA_F32, MogaError, StgaGeom, check, lib  # noqa: F401

__all__ = ["moga_route", "moga_permute", "moga_group_attn", "stga_attn", "stga_attn_train", "stga_attn_mean",
           "visual_attn_branches",
           "visual_attn_mean", "moga_balance_loss", "visual_attention_forward", "attn_workspace", "device_status",
           "MogaError", "geom_struct", "visual_attention_forward_train", "visual_attention_backward"]


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, name, dim=None, shape=None, device=True):
    """Type, rank, shape and layout (the library sees only pointers, so a short
    buffer would be read past its end), then, unless device=False (the caller
    checks all its tensors' residence at once with _on_device after their
    shapes), residence on the current CUDA device."""
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if dim is not None and t.dim() != dim:
        raise ValueError("%s must have %d dims" % (name, dim))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if device:
        _on_device(**{name: t})


def _on_device(**tensors):
    """Every tensor on the current CUDA device (the calls launch on its current stream)."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
        if t.device.index != torch.cuda.current_device():
            raise ValueError("%s is on %s but the calls run on the current device cuda:%d"
                             % (name, t.device, torch.cuda.current_device()))


def _check_geom(geom: dict, N: int):
    """stga_attn takes the token count from the geometry: it must match q's rows."""
    n = geom["T"] * geom["h"] * geom["w"]
    if n != N:
        raise ValueError("geometry has T*h*w = %d tokens but q, k, v have %d rows" % (n, N))


def moga_route(x: torch.Tensor, w_r: torch.Tensor, bias: torch.Tensor | None = None):
    """r = x W_r (+bias), p = softmax(r), g = argmax p.  Returns (g int32 [N], gate fp32 [N], ws)."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be float32 or bfloat16")
    _need(x, x.dtype, "x", 2, device=False)
    _need(w_r, x.dtype, "w_r", 2, device=False)
    N, d = x.shape
    M = w_r.shape[1]
    if w_r.shape[0] != d:
        raise ValueError("w_r must be [d, M]")
    if bias is not None:
        _need(bias, torch.float32, "bias", 1, (M,), device=False)
    _on_device(x=x, w_r=w_r, bias=bias)
    L = lib()
    ws_bytes = L.moga_route_ws_bytes(N, d, M)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)
    g = torch.empty(N, dtype=torch.int32, device=x.device)
    gate = torch.empty(N, dtype=torch.float32, device=x.device)
    dt = MOGA_BF16 if x.dtype == torch.bfloat16 else MOGA_F32
    check(L.moga_route(_ptr(x), _ptr(w_r), dt, _ptr(bias), N, d, M, _ptr(g), _ptr(gate), _ptr(ws), ws.numel(),
                       _stream()), "moga_route")
    return g, gate, ws


def moga_qkv_route(x: torch.Tensor, w_qkv: torch.Tensor, w_r: torch.Tensor, bias: torch.Tensor | None, H: int,
                   hd: int):
    """The Q/K/V projection with the router fused in: x [N, d] bf16, w_qkv [3*H*hd, d] bf16
    (a linear layer's weight), w_r [d, M] bf16.  Returns (q, k, v [N, H, hd] bf16, g, gate, ws)."""
    _need(x, torch.bfloat16, "x", 2, device=False)
    _need(w_qkv, torch.bfloat16, "w_qkv", 2, device=False)
    _need(w_r, torch.bfloat16, "w_r", 2, device=False)
    N, d = x.shape
    M = w_r.shape[1]
    if w_qkv.shape != (3 * H * hd, d) or w_r.shape[0] != d:
        raise ValueError("w_qkv must be [3*H*hd, d] and w_r [d, M]")
    if bias is not None:
        _need(bias, torch.float32, "bias", 1, (M,), device=False)
    _on_device(x=x, w_qkv=w_qkv, w_r=w_r, bias=bias)
    L = lib()
    ws = torch.empty(max(L.moga_qkv_route_ws_bytes(N, d, M), 16), dtype=torch.uint8, device=x.device)
    q, k, v = (torch.empty((N, H, hd), dtype=torch.bfloat16, device=x.device) for _ in range(3))
    g = torch.empty(N, dtype=torch.int32, device=x.device)
    gate = torch.empty(N, dtype=torch.float32, device=x.device)
    check(L.moga_qkv_route(_ptr(x), _ptr(w_qkv), _ptr(w_r), _ptr(bias), N, d, H, hd, M, _ptr(q), _ptr(k), _ptr(v),
                           _ptr(g), _ptr(gate), _ptr(ws), ws.numel(), _stream()), "moga_qkv_route")
    return q, k, v, g, gate, ws


def moga_permute(group_id: torch.Tensor, M: int):
    """Stable group permute.  Returns (perm [N], cu_seqlens [M+1], counts [M], max_seqlen [1]), int32."""
    _need(group_id, torch.int32, "group_id", 1)
    N = group_id.shape[0]
    L = lib()
    ws_bytes = L.moga_permute_ws_bytes(N, M)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=group_id.device)
    dev = group_id.device
    perm = torch.empty(N, dtype=torch.int32, device=dev)
    cu = torch.empty(M + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(M, dtype=torch.int32, device=dev)
    mx = torch.empty(1, dtype=torch.int32, device=dev)
    check(L.moga_permute(_ptr(group_id), N, M, _ptr(perm), _ptr(cu), _ptr(counts), _ptr(mx), _ptr(ws), ws.numel(),
                         _stream()), "moga_permute")
    return perm, cu, counts, mx


def _check_qkv(q, k, v, device=True):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, name, 3, device=False)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share the shape [N, H, hd]")
    if device:
        _on_device(q=q, k=k, v=v)
    return q.shape


def attn_workspace(q: torch.Tensor) -> torch.Tensor:
    """Scratch for the attention calls (Q, K, V copied into segment order)."""
    N, H, hd = q.shape
    n = lib().moga_attn_ws_bytes(N, H, hd)
    if n == 0:
        raise ValueError("unsupported attention shape %s" % (tuple(q.shape),))
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def moga_group_attn(q, k, v, perm, cu_seqlens, gate_prob, M: int, softmax_scale: float | None = None,
                    o_acc: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """o_acc[perm[j]] = gate * softmax(q k^T * scale) v inside each group (written, fp32)."""
    N, H, hd = _check_qkv(q, k, v, device=False)
    _need(perm, torch.int32, "perm", 1, (N,), device=False)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1, (M + 1,), device=False)
    _need(gate_prob, torch.float32, "gate_prob", 1, (N,), device=False)
    if o_acc is not None:
        _need(o_acc, torch.float32, "o_acc", 3, (N, H, hd), device=False)
    _on_device(q=q, k=k, v=v, perm=perm, cu_seqlens=cu_seqlens, gate_prob=gate_prob, o_acc=o_acc, ws=ws)
    if o_acc is None:
        o_acc = torch.empty((N, H, hd), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    ws = attn_workspace(q) if ws is None else ws
    check(lib().moga_group_attn(_ptr(q), _ptr(k), _ptr(v), N, H, hd, _ptr(perm), _ptr(cu_seqlens), M,
                                _ptr(gate_prob), scale, _ptr(o_acc), _ptr(ws), ws.numel(), _stream()),
          "moga_group_attn")
    return o_acc


def geom_struct(geom: dict):
    """C geometry struct from a dict(T, h, w, win_h, win_w, shots, tg_max, aug); keeps the shot array alive."""
    shots = (ctypes.c_int32 * len(geom["shots"]))(*geom["shots"])
    s = StgaGeom(geom["T"], geom["h"], geom["w"], geom["win_h"], geom["win_w"], len(geom["shots"]),
                 ctypes.cast(shots, ctypes.POINTER(ctypes.c_int32)), geom["tg_max"], geom["aug"])
    return s, shots


def stga_attn(q, k, v, geom: dict, softmax_scale: float | None = None, o_acc: torch.Tensor | None = None,
              ws: torch.Tensor | None = None):
    """o_acc += window-group attention + per-frame attention (fp32)."""
    N, H, hd = _check_qkv(q, k, v, device=False)
    _check_geom(geom, N)
    if o_acc is not None:
        _need(o_acc, torch.float32, "o_acc", 3, (N, H, hd), device=False)
    _on_device(q=q, k=k, v=v, o_acc=o_acc, ws=ws)
    if o_acc is None:
        o_acc = torch.zeros((N, H, hd), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    s, keep = geom_struct(geom)
    ws = attn_workspace(q) if ws is None else ws
    check(lib().stga_attn(_ptr(q), _ptr(k), _ptr(v), H, hd, ctypes.byref(s), scale, _ptr(o_acc), _ptr(ws),
                          ws.numel(), _stream()), "stga_attn")
    del keep
    return o_acc


def visual_attn_branches(q, k, v, perm, cu_seqlens, gate_prob, M: int, geom: dict,
                         softmax_scale: float | None = None, o_acc: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None):
    """o_acc = MoGA attention (written) + window and frame attention (added), with one
    gather of Q, K, V into both segment orders; equals moga_group_attn + stga_attn."""
    N, H, hd = _check_qkv(q, k, v, device=False)
    _check_geom(geom, N)
    _need(perm, torch.int32, "perm", 1, (N,), device=False)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1, (M + 1,), device=False)
    _need(gate_prob, torch.float32, "gate_prob", 1, (N,), device=False)
    if o_acc is not None:
        _need(o_acc, torch.float32, "o_acc", 3, (N, H, hd), device=False)
    _on_device(q=q, k=k, v=v, perm=perm, cu_seqlens=cu_seqlens, gate_prob=gate_prob, o_acc=o_acc, ws=ws)
    if o_acc is None:
        o_acc = torch.empty((N, H, hd), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    if ws is None:
        ws = torch.empty(lib().visual_attn_ws_bytes(N, H, hd), dtype=torch.uint8, device=q.device)
    s, keep = geom_struct(geom)
    check(lib().visual_attn_branches(_ptr(q), _ptr(k), _ptr(v), N, H, hd, _ptr(perm), _ptr(cu_seqlens), M,
                                     _ptr(gate_prob), ctypes.byref(s), scale, _ptr(o_acc), _ptr(ws), ws.numel(),
                                     _stream()), "visual_attn_branches")
    del keep
    return o_acc


def stga_attn_train(q, k, v, geom: dict, softmax_scale: float | None = None, ws: torch.Tensor | None = None):
    """Window-group and per-frame attention written to separate buffers, each with its
    log2-domain log-sum-exp.  Returns (o_win, lse_win, o_frame, lse_frame)."""
    N, H, hd = _check_qkv(q, k, v, device=False)
    _check_geom(geom, N)
    _on_device(q=q, k=k, v=v, ws=ws)
    f32 = dict(dtype=torch.float32, device=q.device)
    o_win, o_frame = (torch.empty((N, H, hd), **f32) for _ in range(2))
    lse_win, lse_frame = (torch.empty((N, H), **f32) for _ in range(2))
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    s, keep = geom_struct(geom)
    ws = attn_workspace(q) if ws is None else ws
    check(lib().stga_attn_train(_ptr(q), _ptr(k), _ptr(v), H, hd, ctypes.byref(s), scale, _ptr(o_win),
                                _ptr(lse_win), _ptr(o_frame), _ptr(lse_frame), _ptr(ws), ws.numel(), _stream()),
          "stga_attn_train")
    del keep
    return o_win, lse_win, o_frame, lse_frame


def stga_attn_mean(q, k, v, geom: dict, o_acc: torch.Tensor, softmax_scale: float | None = None,
                   out: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """out = bf16((o_acc + window-group attention + per-frame attention) / 3), mean fused into the frame pass."""
    N, H, hd = _check_qkv(q, k, v, device=False)
    _check_geom(geom, N)
    _need(o_acc, torch.float32, "o_acc", 3, (N, H, hd), device=False)
    if out is not None:
        _need(out, torch.bfloat16, "out", 3, (N, H, hd), device=False)
    _on_device(q=q, k=k, v=v, o_acc=o_acc, out=out, ws=ws)
    if out is None:
        out = torch.empty((N, H, hd), dtype=torch.bfloat16, device=q.device)
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    s, keep = geom_struct(geom)
    ws = attn_workspace(q) if ws is None else ws
    check(lib().stga_attn_mean(_ptr(q), _ptr(k), _ptr(v), H, hd, ctypes.byref(s), scale, _ptr(o_acc), _ptr(out),
                               _ptr(ws), ws.numel(), _stream()), "stga_attn_mean")
    del keep
    return out


def visual_attn_mean(o_acc: torch.Tensor, out: torch.Tensor | None = None):
    """out = bf16(o_acc / 3)."""
    _need(o_acc, torch.float32, "o_acc", device=False)
    if out is not None:
        _need(out, torch.bfloat16, "out", shape=o_acc.shape, device=False)
    _on_device(o_acc=o_acc, out=out)
    if out is None:
        out = torch.empty(o_acc.shape, dtype=torch.bfloat16, device=o_acc.device)
    check(lib().visual_attn_mean(_ptr(o_acc), o_acc.numel(), _ptr(out), _stream()), "visual_attn_mean")
    return out


def moga_balance_loss(counts, route_ws, N: int, M: int, alpha: float, loss: torch.Tensor | None = None):
    """L_gb = alpha * M * sum_i F_i P_i as a fp64 device scalar."""
    _need(counts, torch.int32, "counts", 1, (M,), device=False)
    _need(route_ws, torch.uint8, "route_ws", 1, device=False)
    if route_ws.numel() < 4 * M * -(-N // 32):
        raise ValueError("route_ws holds %d bytes, fewer than the router's per-32-token sums for N=%d, M=%d"
                         % (route_ws.numel(), N, M))
    if loss is not None:
        _need(loss, torch.float64, "loss", 1, (1,), device=False)
    _on_device(counts=counts, route_ws=route_ws, loss=loss)
    if loss is None:
        loss = torch.empty(1, dtype=torch.float64, device=counts.device)
    check(lib().moga_balance_loss(_ptr(counts), _ptr(route_ws), N, M, alpha, _ptr(loss), _stream()),
          "moga_balance_loss")
    return loss


def device_status():
    """Synchronises the current stream and raises if a kernel recorded a device-side error."""
    check(lib().moga_device_status(_stream()), "moga_device_status")


def visual_attention_forward(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float,
                             softmax_scale: float | None = None, fused_mean: bool = True):
    """The whole layer: returns dict(out bf16 [N,H,hd], loss fp64 [1], g, gate, perm, cu_seqlens, counts).

    fused_mean=True takes the mean inside the STGA frame pass (stga_attn_mean);
    False runs stga_attn then visual_attn_mean."""
    if x.dim() != 2 or q.dim() != 3 or x.shape[0] != q.shape[0]:
        raise ValueError("x must be [N, d] and q, k, v [N, H, hd] with the same N")
    _check_geom(geom, q.shape[0])
    g, gate, ws = moga_route(x, w_r, bias)
    perm, cu, counts, mx = moga_permute(g, M)
    ws_attn = attn_workspace(q)
    o = moga_group_attn(q, k, v, perm, cu, gate, M, softmax_scale, ws=ws_attn)
    if fused_mean:
        out = stga_attn_mean(q, k, v, geom, o, softmax_scale, ws=ws_attn)
    else:
        stga_attn(q, k, v, geom, softmax_scale, o_acc=o, ws=ws_attn)
        out = visual_attn_mean(o)
    loss = moga_balance_loss(counts, ws, x.shape[0], M, alpha)
    return dict(out=out, loss=loss, g=g, gate=gate, perm=perm, cu_seqlens=cu, counts=counts, max_seqlen=mx)


# ---------------------------------------------------------------- batch
#
# B videos of the same shape, video-major: x [B, N, d], q/k/v [B, N, H, hd].
# The router is shared; a token's MoGA group holds tokens of its own video
# (segments b * M + g), the STGA groups are per video, and L_gb is taken over
# the whole batch.

def moga_permute_batched(group_id: torch.Tensor, B: int, M: int):
    """Stable permute by b * M + g of B * n_per flattened tokens.  Returns
    (perm [B*n_per], cu_seqlens [B*M+1], counts [B*M], max_seqlen [1]), int32."""
    _need(group_id, torch.int32, "group_id", 1)
    n = group_id.shape[0]
    if B < 1 or n % B:
        raise ValueError("group_id length %d is not a multiple of B=%d" % (n, B))
    L = lib()
    ws_bytes = L.moga_permute_batched_ws_bytes(n // B, B, M)
    if ws_bytes == 0:
        raise ValueError("unsupported batch: B=%d, M=%d, n_per=%d" % (B, M, n // B))
    dev = group_id.device
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    perm = torch.empty(n, dtype=torch.int32, device=dev)
    cu = torch.empty(B * M + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(B * M, dtype=torch.int32, device=dev)
    mx = torch.empty(1, dtype=torch.int32, device=dev)
    check(L.moga_permute_batched(_ptr(group_id), n // B, B, M, _ptr(perm), _ptr(cu), _ptr(counts), _ptr(mx),
                                 _ptr(ws), ws.numel(), _stream()), "moga_permute_batched")
    return perm, cu, counts, mx


def visual_attention_forward_batched(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float,
                                     softmax_scale: float | None = None):
    """The layer over a batch of B videos: x [B, N, d], q/k/v [B, N, H, hd] bf16.
    Returns dict(out bf16 [B, N, H, hd], loss fp64 [1], g, gate, perm, cu_seqlens, counts)."""
    if x.dim() != 3 or q.dim() != 4:
        raise ValueError("x must be [B, N, d] and q, k, v [B, N, H, hd]")
    B, N, d = x.shape
    if q.shape[:2] != (B, N) or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be [B, N, H, hd] with x's B and N")
    H, hd = q.shape[2], q.shape[3]
    _check_geom(geom, N)
    qf, kf, vf = (t.reshape(B * N, H, hd) for t in (q, k, v))
    g, gate, rws = moga_route(x.reshape(B * N, d), w_r, bias)
    perm, cu, counts, mx = moga_permute_batched(g, B, M)
    L = lib()
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    ws = attn_workspace(qf)
    o = torch.empty((B * N, H, hd), dtype=torch.float32, device=q.device)
    check(L.moga_group_attn_batched(_ptr(qf), _ptr(kf), _ptr(vf), N, B, H, hd, _ptr(perm), _ptr(cu), M, _ptr(gate),
                                    scale, _ptr(o), None, _ptr(ws), ws.numel(), _stream()), "moga_group_attn_batched")
    s, keep = geom_struct(geom)
    check(L.stga_attn_batched(_ptr(qf), _ptr(kf), _ptr(vf), B, H, hd, ctypes.byref(s), scale, _ptr(o), _ptr(ws),
                              ws.numel(), _stream()), "stga_attn_batched")
    del keep
    out = visual_attn_mean(o).reshape(B, N, H, hd)
    loss = torch.empty(1, dtype=torch.float64, device=x.device)
    check(L.moga_balance_loss_batched(_ptr(counts), B, _ptr(rws), B * N, M, alpha, _ptr(loss), _stream()),
          "moga_balance_loss_batched")
    return dict(out=out, loss=loss, g=g, gate=gate, perm=perm, cu_seqlens=cu, counts=counts, max_seqlen=mx)


def _check_layer_args(x, w_r, q, k, v, M: int, geom: dict, bias=None, dout=None):
    """Shapes of the training calls' inputs, then their residence: x [N, d]
    (fp32 or bf16) and w_r [d, M] of x's dtype, q/k/v [N, H, hd] bf16, bias
    [M] fp32, dout [N, H, hd] bf16, a geometry of N tokens."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be float32 or bfloat16")
    _need(x, x.dtype, "x", 2, device=False)
    N, d = x.shape
    _need(w_r, x.dtype, "w_r", 2, (d, M), device=False)
    Nq, H, hd = _check_qkv(q, k, v, device=False)
    if Nq != N:
        raise ValueError("x has %d rows, q, k, v %d" % (N, Nq))
    _check_geom(geom, N)
    if bias is not None:
        _need(bias, torch.float32, "bias", 1, (M,), device=False)
    if dout is not None:
        _need(dout, torch.bfloat16, "dout", 3, (N, H, hd), device=False)
    _on_device(x=x, w_r=w_r, q=q, k=k, v=v, bias=bias, dout=dout)
    return N, d, H, hd


# ---------------------------------------------------------------- training
#
# The training forward keeps the router probabilities, the three branch
# outputs and each branch's per-row log-sum-exp; the backward differentiates
# J = sum(dout * out) + dloss * L_gb (argmax and counts are constants).

def visual_attention_forward_train(x, w_r, bias, q, k, v, M: int, geom: dict, alpha: float,
                                   softmax_scale: float | None = None):
    """Forward that saves what the backward needs.  Returns dict(out, loss, saved)."""
    L = lib()
    N, d, H, hd = _check_layer_args(x, w_r, q, k, v, M, geom, bias=bias)
    dev = x.device
    scale = 1.0 / math.sqrt(hd) if softmax_scale is None else softmax_scale
    rws = torch.empty(max(L.moga_route_ws_bytes(N, d, M), 16), dtype=torch.uint8, device=dev)
    g = torch.empty(N, dtype=torch.int32, device=dev)
    gate = torch.empty(N, dtype=torch.float32, device=dev)
    probs = torch.empty((N, M), dtype=torch.float32, device=dev)
    dt = MOGA_BF16 if x.dtype == torch.bfloat16 else MOGA_F32
    check(L.moga_route_train(_ptr(x), _ptr(w_r), dt, _ptr(bias), N, d, M, _ptr(g), _ptr(gate), _ptr(probs),
                             _ptr(rws), rws.numel(), _stream()), "moga_route_train")
    perm, cu, counts, mx = moga_permute(g, M)
    ws = attn_workspace(q)
    f32 = dict(dtype=torch.float32, device=dev)
    o_moga, o_win, o_frame = (torch.empty((N, H, hd), **f32) for _ in range(3))
    lse_moga, lse_win, lse_frame = (torch.empty((N, H), **f32) for _ in range(3))
    check(L.moga_group_attn_train(_ptr(q), _ptr(k), _ptr(v), N, H, hd, _ptr(perm), _ptr(cu), M, _ptr(gate), scale,
                                  _ptr(o_moga), _ptr(lse_moga), _ptr(ws), ws.numel(), _stream()),
          "moga_group_attn_train")
    s, keep = geom_struct(geom)
    check(L.stga_attn_train(_ptr(q), _ptr(k), _ptr(v), H, hd, ctypes.byref(s), scale, _ptr(o_win), _ptr(lse_win),
                            _ptr(o_frame), _ptr(lse_frame), _ptr(ws), ws.numel(), _stream()), "stga_attn_train")
    del keep
    out = torch.empty((N, H, hd), dtype=torch.bfloat16, device=dev)
    check(L.visual_attn_mean3(_ptr(o_moga), _ptr(o_win), _ptr(o_frame), out.numel(), _ptr(out), _stream()),
          "visual_attn_mean3")
    loss = moga_balance_loss(counts, rws, N, M, alpha)
    saved = dict(g=g, gate=gate, probs=probs, perm=perm, cu_seqlens=cu, counts=counts, o_moga=o_moga,
                 lse_moga=lse_moga, o_win=o_win, lse_win=lse_win, o_frame=o_frame, lse_frame=lse_frame,
                 scale=scale)
    return dict(out=out, loss=loss, saved=saved)


def visual_attention_backward(saved: dict, x, w_r, q, k, v, M: int, geom: dict, alpha: float, dout, dloss: float,
                              with_bias: bool = False):
    """Gradients of sum(dout * out) + dloss * L_gb.  dout [N, H, hd] bf16.

    Returns dict(dq, dk, dv [N, H, hd] fp32, dx [N, d] fp32, dw_r [d, M] fp32,
    dbias [M] fp32 or None, dgate [N] fp32)."""
    L = lib()
    N, d, H, hd = _check_layer_args(x, w_r, q, k, v, M, geom, dout=dout)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.zeros((N, H, hd), **f32) for _ in range(3))
    dgate = torch.empty(N, **f32)
    ws = torch.empty(L.moga_attn_bwd_ws_bytes(N, H, hd), dtype=torch.uint8, device=dev)
    sc = saved["scale"]
    check(L.moga_group_attn_bwd(_ptr(q), _ptr(k), _ptr(v), N, H, hd, _ptr(saved["perm"]), _ptr(saved["cu_seqlens"]),
                                M, _ptr(saved["gate"]), sc, _ptr(saved["o_moga"]), _ptr(saved["lse_moga"]),
                                _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate), _ptr(ws), ws.numel(),
                                _stream()), "moga_group_attn_bwd")
    s, keep = geom_struct(geom)
    check(L.stga_attn_bwd(_ptr(q), _ptr(k), _ptr(v), H, hd, ctypes.byref(s), sc, _ptr(saved["o_win"]),
                          _ptr(saved["lse_win"]), _ptr(saved["o_frame"]), _ptr(saved["lse_frame"]), _ptr(dout),
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream()), "stga_attn_bwd")
    del keep
    dx = torch.empty((N, d), **f32)
    dw_r = torch.empty((d, M), **f32)
    dbias = torch.empty(M, **f32) if with_bias else None
    rws = torch.empty(L.moga_route_bwd_ws_bytes(N, d, M), dtype=torch.uint8, device=dev)
    dt = MOGA_BF16 if x.dtype == torch.bfloat16 else MOGA_F32
    check(L.moga_route_bwd(_ptr(x), _ptr(w_r), dt, N, d, M, _ptr(saved["g"]), _ptr(saved["probs"]), _ptr(dgate),
                           _ptr(saved["counts"]), alpha, dloss, _ptr(dx), _ptr(dw_r), _ptr(dbias), _ptr(rws),
                           rws.numel(), _stream()), "moga_route_bwd")
    return dict(dq=dq, dk=dk, dv=dv, dx=dx, dw_r=dw_r, dbias=dbias, dgate=dgate)
