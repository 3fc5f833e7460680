"""The C ABI library loads, exports every declared symbol and validates arguments on the host (CPU only)."""
import ctypes
import os
import re

import pytest

from sparse_attention_long_moga_b200 import _lib
from sparse_attention_long_moga_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moga.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions(path=HEADER):
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:moga_status|size_t|const char\s*\*|void)\s+(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_six_calls():
    names = declared_functions()
    for n in ("moga_route", "moga_permute", "moga_group_attn", "stga_attn", "visual_attn_mean",
              "moga_balance_loss"):
        assert n in names
    assert set(names) == set(_lib.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_workspace_sizes(lib):
    assert lib.moga_route_ws_bytes(0, 1536, 5) == 0
    assert lib.moga_route_ws_bytes(1000, 1536, 33) == 0
    assert lib.moga_route_ws_bytes(1000, 12, 4) == 0
    # one partial row per 32 tokens (256-byte aligned) + W_r^T padded to 32 groups x 64-multiple of d
    assert lib.moga_route_ws_bytes(32760, 1536, 5) == 1024 * 5 * 4 + 32 * 1536 * 2
    assert lib.moga_route_ws_bytes(100, 72, 3) == 256 + 32 * 128 * 2
    assert lib.moga_route_ws_bytes(33, 8, 32) == 256 + 32 * 64 * 2
    assert lib.moga_permute_ws_bytes(32760, 5) == 2 * 16 * 5 * 4
    assert lib.moga_permute_ws_bytes(-1, 5) == 0


FAKE = ctypes.c_void_p(4096)   # never dereferenced: validation fails first


def test_route_argument_checks(lib):
    st = lib.moga_route(None, FAKE, 1, None, 10, 8, 4, FAKE, FAKE, FAKE, 4096, None)
    assert st == 1 and b"null" in lib.moga_last_error()
    assert lib.moga_route(FAKE, FAKE, 1, None, 10, 8, 33, FAKE, FAKE, FAKE, 4096, None) == 1
    assert lib.moga_route(FAKE, FAKE, 1, None, 10, 12, 4, FAKE, FAKE, FAKE, 4096, None) == 1   # d % 8
    assert lib.moga_route(FAKE, FAKE, 7, None, 10, 8, 4, FAKE, FAKE, FAKE, 4096, None) == 1    # dtype
    assert lib.moga_route(FAKE, FAKE, 1, None, 0, 8, 4, FAKE, FAKE, FAKE, 4096, None) == 1     # N
    assert lib.moga_route(FAKE, FAKE, 1, None, 1000, 8, 4, FAKE, FAKE, FAKE, 4, None) == 3     # workspace


def test_permute_argument_checks(lib):
    assert lib.moga_permute(FAKE, 100, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, None) == 1
    assert lib.moga_permute(FAKE, 100000, 8, FAKE, FAKE, FAKE, FAKE, FAKE, 8, None) == 3
    assert lib.moga_permute(None, 100, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, None) == 1


def test_attention_argument_checks(lib):
    W = 1 << 40
    ga = lambda *a: lib.moga_group_attn(*a)  # noqa: E731
    assert ga(FAKE, FAKE, FAKE, 100, 2, 96, FAKE, FAKE, 4, FAKE, 0.1, FAKE, FAKE, W, None) == 2
    assert b"head_dim" in lib.moga_last_error()
    assert ga(FAKE, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 40, FAKE, 0.1, FAKE, FAKE, W, None) == 1
    assert ga(FAKE, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 4, FAKE, -1.0, FAKE, FAKE, W, None) == 1
    assert ga(FAKE, FAKE, FAKE, 1 << 30, 4, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, FAKE, W, None) == 1
    mis = ctypes.c_void_p(4096 + 8)
    assert ga(mis, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, FAKE, W, None) == 1
    assert ga(FAKE, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, FAKE, 1000, None) == 3
    assert ga(FAKE, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, None, W, None) == 1
    assert lib.moga_attn_ws_bytes(100, 2, 128) == 3 * 100 * 2 * 128 * 2
    assert lib.moga_attn_ws_bytes(100, 2, 96) == 0


def _geom(**kw):
    g = dict(T=4, h=4, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=0, aug=2)
    g.update(kw)
    return g


@pytest.mark.parametrize("bad,msg", [
    (dict(shots=[2, 1]), b"sum"),
    (dict(win_h=3), b"tile"),
    (dict(shots=[4, 0], T=4), b"length"),
    (dict(tg_max=-1), b"geometry"),
])
def test_stga_geometry_checks(lib, bad, msg):
    s, keep = _geom_struct(_geom(**bad))
    st = lib.stga_attn(FAKE, FAKE, FAKE, 2, 128, ctypes.byref(s), 0.1, FAKE, FAKE, 1 << 40, None)
    assert st == 1 and msg in lib.moga_last_error(), lib.moga_last_error()


def _geom_struct(g):
    shots = (ctypes.c_int32 * len(g["shots"]))(*g["shots"])
    s = _lib.StgaGeom(g["T"], g["h"], g["w"], g["win_h"], g["win_w"], len(g["shots"]),
                      ctypes.cast(shots, ctypes.POINTER(ctypes.c_int32)), g["tg_max"], g["aug"])
    return s, shots


def test_mean_and_loss_argument_checks(lib):
    assert lib.visual_attn_mean(None, 10, FAKE, None) == 1
    assert lib.visual_attn_mean(FAKE, 0, FAKE, None) == 1
    assert lib.visual_attn_mean(ctypes.c_void_p(4100), 10, FAKE, None) == 1
    assert lib.moga_balance_loss(FAKE, FAKE, 10, 0, 0.1, FAKE, None) == 1
    assert lib.moga_balance_loss(None, FAKE, 10, 4, 0.1, FAKE, None) == 1


def test_version(lib):
    assert b"sm_100a" in lib.moga_version()
    assert b"checking" not in lib.moga_version()


def test_branches_workspace_and_argument_checks(lib):
    assert lib.visual_attn_ws_bytes(1000, 4, 128) == 2 * lib.moga_attn_ws_bytes(1000, 4, 128)
    assert lib.visual_attn_ws_bytes(1000, 4, 96) == 0
    shots = (ctypes.c_int32 * 2)(2, 2)
    g = _lib.StgaGeom(4, 4, 8, 2, 4, 2, ctypes.cast(shots, ctypes.POINTER(ctypes.c_int32)), 0, 2)
    p = ctypes.c_void_p(4096)
    N, H, hd = 128, 2, 128
    small = lib.moga_attn_ws_bytes(N, H, hd)
    # a workspace for one copy only is refused before any launch
    st = lib.visual_attn_branches(p, p, p, N, H, hd, p, p, 3, p, ctypes.byref(g), ctypes.c_float(0.1), p, p, small,
                                  None)
    assert st == 3 and b"workspace" in lib.moga_last_error()
    # N must be the geometry's token count
    st = lib.visual_attn_branches(p, p, p, N + 1, H, hd, p, p, 3, p, ctypes.byref(g), ctypes.c_float(0.1), p, p,
                                  2 * small, None)
    assert st == 1 and b"geometry" in lib.moga_last_error()


def test_status_codes_match_header():
    text = open(HEADER).read()
    enum = dict((n, int(v)) for n, v in re.findall(r"(MOGA_OK|MOGA_ERR_\w+)\s*=\s*(\d+)", text))
    assert {v: k for k, v in enum.items()} == _lib.STATUS


def test_checking_build_loads_and_validates_like_the_default():
    """The checking build (device-side index checks) exports the same ABI and
    rejects the same host-side arguments; its kernels need a GPU."""
    build()
    dbg = _lib.load(_lib.DEBUG_LIB_PATH)
    assert b"checking build" in dbg.moga_version()
    for name in declared_functions():
        assert hasattr(dbg, name), name
    # host validation is shared code: a bad M is refused before any launch
    assert dbg.moga_permute(ctypes.c_void_p(16), 100, 33, ctypes.c_void_p(16), ctypes.c_void_p(16),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 1 << 20, None) == 1
    assert b"M=33" in dbg.moga_last_error()


def test_batch_sp_and_projection_workspace_sizes(lib):
    assert lib.moga_permute_batched_ws_bytes(1000, 65, 16) == 0          # 1040 keys > 1024
    assert lib.moga_permute_batched_ws_bytes(1000, 4, 5) == 2 * 2 * 20 * 4   # 2 tiles of 2048 tokens, 20 keys
    assert lib.moga_qkv_route_ws_bytes(32760, 1536, 5) == 1024 * 5 * 4 + 64 * 1536 * 2
    assert lib.moga_qkv_route_ws_bytes(32760, 12, 5) == 0                # d % 8
    assert lib.moga_route_bwd_ws_bytes(100, 12, 4) == 0
    assert lib.moga_attn_bwd_ws_bytes(1000, 2, 96) == 0                  # head_dim


def test_batch_argument_checks(lib):
    P = lib.moga_permute_batched
    assert P(None, 100, 2, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, None) == 1
    assert P(FAKE, 100, 0, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, None) == 1         # B
    assert P(FAKE, 100, 2, 33, FAKE, FAKE, FAKE, FAKE, FAKE, 4096, None) == 1        # M
    assert P(FAKE, 100, 65, 16, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2    # too many keys
    assert P(FAKE, 100, 2, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == 3            # workspace
    W = 1 << 30
    ga = lib.moga_group_attn_batched
    assert ga(FAKE, FAKE, FAKE, 100, 0, 2, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, None, FAKE, W, None) == 1
    assert ga(FAKE, FAKE, FAKE, 100, 2, 2, 128, FAKE, FAKE, 40, FAKE, 0.1, FAKE, None, FAKE, W, None) == 1
    assert lib.stga_attn_batched(FAKE, FAKE, FAKE, 0, 2, 128, None, 0.1, FAKE, FAKE, W, None) == 1
    assert lib.moga_balance_loss_batched(FAKE, 3, FAKE, 100, 4, 0.1, FAKE, None) == 1   # N % B
    assert lib.moga_balance_loss_batched(FAKE, 2, FAKE, 100, 0, 0.1, FAKE, None) == 1


def test_sequence_parallel_argument_checks(lib):
    assert lib.moga_sp_pack_heads(FAKE, 100, 12, 128, 5, FAKE, None) == 1      # 12 heads on 5 ranks
    assert lib.moga_sp_unpack_heads(None, 100, 12, 128, 4, FAKE, None) == 1
    mis = ctypes.c_void_p(4104)
    assert lib.moga_sp_pack_heads(mis, 100, 12, 128, 4, FAKE, None) == 1       # alignment
    assert lib.moga_balance_loss_part(FAKE, FAKE, 200, 100, 4, 0.1, FAKE, None) == 1   # n_local > N


def test_projection_and_backward_argument_checks(lib):
    q = lib.moga_qkv_route
    W = 1 << 30
    assert q(FAKE, FAKE, FAKE, None, 100, 12, 2, 128, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, W, None) == 1   # d % 8
    assert q(FAKE, FAKE, FAKE, None, 100, 128, 2, 96, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, W, None) == 2   # head_dim
    assert q(FAKE, FAKE, FAKE, None, 100, 128, 2, 128, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == 3  # workspace
    assert q(FAKE, FAKE, None, None, 100, 128, 2, 128, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, W, None) == 1
    rb = lib.moga_route_bwd
    assert rb(FAKE, FAKE, 1, 100, 12, 4, FAKE, FAKE, FAKE, FAKE, 0.1, 1.0, FAKE, FAKE, None, FAKE, W, None) == 1
    assert rb(FAKE, FAKE, 1, 100, 16, 40, FAKE, FAKE, FAKE, FAKE, 0.1, 1.0, FAKE, FAKE, None, FAKE, W, None) == 1
    gb = lib.moga_group_attn_bwd
    assert gb(FAKE, FAKE, FAKE, 100, 2, 128, FAKE, FAKE, 4, FAKE, 0.1, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE,
              FAKE, W, None) == 1   # null dout
