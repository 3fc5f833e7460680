"""The Python binding's argument checks (CPU only).

The C ABI receives plain pointers, so buffer lengths are checked above it: a
companion tensor of the wrong shape, a geometry whose T*h*w differs from q's
rows, or a router workspace too small for the loss's reads must raise before
any call, and tensors that are not on the current CUDA device are refused.
On this CPU-only machine a correctly shaped call therefore stops at the
residence check, which shows the shape checks run first.
"""
import pytest
import torch

import sparse_attention_long_moga_b200 as moga

N, H, HD, M = 96, 2, 64, 4
GEOM = dict(T=6, h=4, w=4, win_h=2, win_w=2, shots=[3, 3], tg_max=0, aug=2)   # 96 tokens


def _qkv(n=N):
    return tuple(torch.zeros((n, H, HD), dtype=torch.bfloat16) for _ in range(3))


def _i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def test_group_attention_companion_shapes():
    q, k, v = _qkv()
    ok = dict(perm=_i32(N), cu_seqlens=_i32(M + 1), gate_prob=_f32(N))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.moga_group_attn(q, k, v, M=M, **ok)
    for name, bad in (("perm", _i32(N - 1)), ("cu_seqlens", _i32(M)), ("gate_prob", _f32(N + 1))):
        with pytest.raises(ValueError, match="%s must have shape" % name):
            moga.moga_group_attn(q, k, v, M=M, **dict(ok, **{name: bad}))
    with pytest.raises(ValueError, match="o_acc must have shape"):
        moga.moga_group_attn(q, k, v, M=M, o_acc=_f32(N, H, HD + 1), **ok)
    with pytest.raises(ValueError, match="perm must be torch.int32"):
        moga.moga_group_attn(q, k, v, M=M, **dict(ok, perm=torch.zeros(N, dtype=torch.int64)))
    with pytest.raises(ValueError, match="share the shape"):
        moga.moga_group_attn(q, k[:-1], v, M=M, **ok)


def test_static_groups_take_their_token_count_from_the_geometry():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.stga_attn(q, k, v, GEOM)
    for geom in (dict(GEOM, T=5, shots=[3, 2]), dict(GEOM, w=8)):
        with pytest.raises(ValueError, match="geometry has"):
            moga.stga_attn(q, k, v, geom)
        with pytest.raises(ValueError, match="geometry has"):
            moga.stga_attn_mean(q, k, v, geom, o_acc=_f32(N, H, HD))
    with pytest.raises(ValueError, match="o_acc must have shape"):
        moga.stga_attn(q, k, v, GEOM, o_acc=_f32(N - 1, H, HD))
    with pytest.raises(ValueError, match="out must have shape"):
        moga.stga_attn_mean(q, k, v, GEOM, o_acc=_f32(N, H, HD), out=torch.zeros((N, H, 32), dtype=torch.bfloat16))


def test_mean_and_loss_buffers():
    with pytest.raises(ValueError, match="out must have shape"):
        moga.visual_attn_mean(_f32(N, H, HD), out=torch.zeros((N, H), dtype=torch.bfloat16))
    ws_need = 4 * M * (-(-N // 32))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.moga_balance_loss(_i32(M), torch.zeros(ws_need, dtype=torch.uint8), N, M, 0.1)
    with pytest.raises(ValueError, match="route_ws holds"):
        moga.moga_balance_loss(_i32(M), torch.zeros(ws_need - 4, dtype=torch.uint8), N, M, 0.1)
    with pytest.raises(ValueError, match="counts must have shape"):
        moga.moga_balance_loss(_i32(M + 1), torch.zeros(ws_need, dtype=torch.uint8), N, M, 0.1)
    with pytest.raises(ValueError, match="route_ws must be torch.uint8"):
        moga.moga_balance_loss(_i32(M), _f32(ws_need), N, M, 0.1)


def test_router_and_layer_shapes():
    x = torch.zeros((N, 64), dtype=torch.bfloat16)
    w = torch.zeros((64, M), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.moga_route(x, w)
    with pytest.raises(ValueError, match="bias must have shape"):
        moga.moga_route(x, w, _f32(M + 1))
    with pytest.raises(ValueError, match="w_r must be"):
        moga.moga_route(x, torch.zeros((32, M), dtype=torch.bfloat16))
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="same N"):
        moga.visual_attention_forward(x[:-1], w, None, q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="geometry has"):
        moga.visual_attention_forward(x, w, None, q, k, v, M, dict(GEOM, h=2, win_h=1), 0.1)
    wq = torch.zeros((3 * H * HD, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="w_qkv must be"):
        moga.moga_qkv_route(x, wq[:-1], w, None, H, HD)


def test_training_call_shapes():
    x = torch.zeros((N, 64), dtype=torch.bfloat16)
    w = torch.zeros((64, M), dtype=torch.bfloat16)
    q, k, v = _qkv()
    dout = torch.zeros((N, H, HD), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.visual_attention_forward_train(x, w, None, q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="w_r must be torch.bfloat16"):
        moga.visual_attention_forward_train(x, w.float(), None, q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="w_r must have shape"):
        moga.visual_attention_forward_train(x, w[:, :-1], None, q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="bias must have shape"):
        moga.visual_attention_forward_train(x, w, _f32(M - 1), q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="rows"):
        moga.visual_attention_forward_train(x[:-32], w, None, q, k, v, M, GEOM, 0.1)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        moga.visual_attention_backward({}, x, w, q, k, v, M, GEOM, 0.1, dout, 1.0)
    with pytest.raises(ValueError, match="dout must have shape"):
        moga.visual_attention_backward({}, x, w, q, k, v, M, GEOM, 0.1, dout[:-1], 1.0)
    with pytest.raises(ValueError, match="geometry has"):
        moga.visual_attention_backward({}, x, w, q, k, v, M, dict(GEOM, T=3, shots=[3]), 0.1, dout, 1.0)
