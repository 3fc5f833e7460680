"""Device-side index checks, through the C ABI.

Group ids outside [0, M) are recorded by the permute in every build and
skipped.  The checking build (libmoga_debug.so, -DMOGA_DEBUG) also checks
every perm entry a kernel dereferences and the cu_seqlens split before the
access it guards.  A failed check records MOGA_ERR_BAD_INDEX in the device
error word, which moga_device_status() returns, and the guarded access is
skipped: nothing faults, and the next well-formed call on the same context
is correct.  Bad perm / cu_seqlens inputs are only ever given to the checking
build (the default build does not check them).
"""
import ctypes

import numpy as np
import pytest

from _data import Case
from synth import workloads as W

pytestmark = pytest.mark.gpu

BAD_INDEX = 6
EDGE = W.Workload("edge_300", T=5, h=6, w=10, d=64, H=3, hd=128, M=7, shots=(2, 1, 2), tg_max=2,
                  win_h=3, win_w=5)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _s():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.fixture(scope="module")
def libs(cuda_device):
    from sparse_attention_long_moga_b200 import _lib
    return dict(default=_lib.load(_lib.LIB_PATH), debug=_lib.load(_lib.DEBUG_LIB_PATH))


def _permute(L, g, M):
    import torch
    N = g.numel()
    dev = g.device
    ws = torch.empty(max(L.moga_permute_ws_bytes(N, M), 16), dtype=torch.uint8, device=dev)
    perm = torch.full((N,), -1, dtype=torch.int32, device=dev)
    cu = torch.empty(M + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(M, dtype=torch.int32, device=dev)
    mx = torch.empty(1, dtype=torch.int32, device=dev)
    assert L.moga_permute(_p(g), N, M, _p(perm), _p(cu), _p(counts), _p(mx), _p(ws), ws.numel(), _s()) == 0
    return perm, cu, counts, mx


@pytest.mark.parametrize("flavour", ["default", "debug"])
def test_bad_group_ids_recorded_and_skipped(libs, flavour, cuda_device):
    import torch
    L = libs[flavour]
    N, M = 5000, 5
    rs = np.random.default_rng(4)
    g = rs.integers(0, M, N).astype(np.int32)
    bad = np.array([5, 17, 2047, 2048, 4999])
    g[bad] = [M, -1, 1 << 20, M + 3, -7]
    perm, cu, counts, _ = _permute(L, torch.from_numpy(g).to(cuda_device), M)
    assert L.moga_device_status(_s()) == BAD_INDEX
    # the valid tokens are permuted as if the bad ones were absent
    ok = np.ones(N, bool)
    ok[bad] = False
    want_counts = np.bincount(g[ok], minlength=M)
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    assert np.array_equal(cu.cpu().numpy(), np.concatenate([[0], np.cumsum(want_counts)]))
    want_perm = np.nonzero(ok)[0][np.argsort(g[ok], kind="stable")]
    assert np.array_equal(perm.cpu().numpy()[:ok.sum()], want_perm)
    # the word was cleared by the read; a clean call reports nothing
    _permute(L, torch.from_numpy(np.where(ok, g, 0).astype(np.int32)).to(cuda_device), M)
    assert L.moga_device_status(_s()) == 0


def _attn_inputs(cuda_device):
    import torch
    import sparse_attention_long_moga_b200 as moga
    case = Case(EDGE)
    t = case.gpu(cuda_device)
    g, gate, _ = moga.moga_route(t["x"], t["w_r"], t["bias"])
    perm, cu, counts, _ = moga.moga_permute(g, case.wl.M)
    moga.device_status()
    N, H, hd = t["q"].shape
    ws = torch.empty(moga.lib().moga_attn_ws_bytes(N, H, hd), dtype=torch.uint8, device=cuda_device)
    return case, t, perm, cu, gate, ws


def _moga_call(L, t, perm, cu, gate, M, ws, o):
    N, H, hd = t["q"].shape
    return L.moga_group_attn(_p(t["q"]), _p(t["k"]), _p(t["v"]), N, H, hd, _p(perm), _p(cu), M, _p(gate),
                             ctypes.c_float(1.0 / np.sqrt(hd)), _p(o), _p(ws), ws.numel(), _s())


def test_checking_build_matches_default_build(libs, cuda_device):
    """The checks change no result: both builds give identical bits on good inputs."""
    import torch
    import sparse_attention_long_moga_b200 as moga
    case, t, perm, cu, gate, ws = _attn_inputs(cuda_device)
    outs = {}
    for name, L in libs.items():
        o = torch.zeros(t["q"].shape, dtype=torch.float32, device=cuda_device)
        assert _moga_call(L, t, perm, cu, gate, case.wl.M, ws, o) == 0
        s, keep = moga.geom_struct(case.geom)
        N, H, hd = t["q"].shape
        assert L.stga_attn(_p(t["q"]), _p(t["k"]), _p(t["v"]), H, hd, ctypes.byref(s),
                           ctypes.c_float(1.0 / np.sqrt(hd)), _p(o), _p(ws), ws.numel(), _s()) == 0
        assert L.moga_device_status(_s()) == 0
        outs[name] = o.clone()
        del keep
    assert torch.equal(outs["default"], outs["debug"])


def test_checking_build_bad_perm_entry(libs, cuda_device):
    import torch
    L = libs["debug"]
    case, t, perm, cu, gate, ws = _attn_inputs(cuda_device)
    N = t["q"].shape[0]
    bad = perm.clone()
    bad[3] = N + 7
    bad[N - 1] = -2
    o = torch.zeros(t["q"].shape, dtype=torch.float32, device=cuda_device)
    assert _moga_call(L, t, bad, cu, gate, case.wl.M, ws, o) == 0
    assert L.moga_device_status(_s()) == BAD_INDEX
    # the context is intact: a good call afterwards matches the default build
    ref = torch.zeros_like(o)
    assert _moga_call(libs["default"], t, perm, cu, gate, case.wl.M, ws, ref) == 0
    assert _moga_call(L, t, perm, cu, gate, case.wl.M, ws, o) == 0
    assert L.moga_device_status(_s()) == 0 and libs["default"].moga_device_status(_s()) == 0
    assert torch.equal(o, ref)


@pytest.mark.parametrize("how", ["decreasing", "past_end", "negative_start"])
def test_checking_build_bad_cu_seqlens(libs, how, cuda_device):
    import torch
    L = libs["debug"]
    case, t, perm, cu, gate, ws = _attn_inputs(cuda_device)
    N = t["q"].shape[0]
    bad = cu.clone()
    if how == "decreasing":
        bad[2], bad[3] = cu[3], cu[2] - 1
    elif how == "past_end":
        bad[-1] = N + 100
    else:
        bad[0] = -5
    sentinel = torch.full(t["q"].shape, 7.0, dtype=torch.float32, device=cuda_device)
    assert _moga_call(L, t, perm, bad, gate, case.wl.M, ws, sentinel) == 0
    assert L.moga_device_status(_s()) == BAD_INDEX
    # the launch did no attention work: the output buffer is untouched
    assert bool((sentinel == 7.0).all())
