"""Failure detection on the GPU without a GPU fault.

A test-only flag makes the attention kernel's producer skip the query-tile
load, so the MMA warp's bounded wait on it runs out (a barrier that nothing
completes).  The kernel must record MOGA_ERR_TIMEOUT in the device error word,
drain its in-flight copies, release its tensor memory and exit; the host reads
the status, and the next normal launch must work and stay correct.
"""
import ctypes

import numpy as np
import pytest

from _data import Case, assert_close
from oracle import attention as oatt
from synth import workloads as W

pytestmark = pytest.mark.gpu

WL = W.Workload("fault_case", T=4, h=8, w=16, d=64, H=2, hd=128, M=3, shots=(2, 2), tg_max=0,
                win_h=4, win_w=8)


def _hook():
    import sparse_attention_long_moga_b200 as moga
    fn = moga._lib.lib().moga_test_set_attn_debug
    fn.restype = None
    fn.argtypes = [ctypes.c_longlong, ctypes.c_int]
    return fn


def test_bounded_wait_reports_timeout_and_recovers(cuda_device):
    import sparse_attention_long_moga_b200 as moga
    case = Case(WL)
    t = case.gpu()
    g, gate, ws = moga.moga_route(t["x"], t["w_r"], t["bias"])
    perm, cu, counts, mx = moga.moga_permute(g, WL.M)
    moga.device_status()
    hook = _hook()
    hook(50_000_000, 1)          # ~25-40 ms per wait, producer skips the Q load
    try:
        moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, WL.M)
        with pytest.raises(moga.MogaError) as ei:
            moga.device_status()
        assert ei.value.status == 5   # MOGA_ERR_TIMEOUT
    finally:
        hook(0, 0)
    moga.device_status()          # the error word was cleared by the read
    o = moga.moga_group_attn(t["q"], t["k"], t["v"], perm, cu, gate, WL.M)
    moga.device_status()
    q, k, v = case.qkv64()
    gg, p_g, _ = case.route64()
    assert_close(o.cpu().numpy(), oatt.moga(q, k, v, gg, p_g, WL.M, 1 / np.sqrt(WL.hd)), "after recovery")
