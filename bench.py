#!/usr/bin/env python
"""Benchmark: MoGA visual-attention layer forward (route, permute, MoGA group
attention, STGA window + frame attention, three-way mean, balance loss) on
synthetic Wan-shaped latents.  Default workload: the 60 s ten-shot video at
24 fps, 361 frames x 30 x 52 = 563,160 tokens, d = 5120, 40 heads x 128,
M = 20, router input drawn from 20 Gaussian clusters, temporal groups of
<= 7 frames, 15 x 26 windows, two borrowed frames per side at each cut.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

One step = one full layer forward over one sequence, inputs resident in HBM.
Between timed steps a 256 MiB buffer is written to flush L2 (outside the
timed events).  Under torchrun each rank runs its own sequence (independent
problems, no data-path collective); the job time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
`--workload` picks another workload of the suite (each gives its own line).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from synth import workloads as W  # noqa: E402

METRIC = "visual-attn layer fwd tokens/s (bf16); group-attn % of tcgen05 bf16 peak"
# the headline workload: the largest single-GPU configuration of the suite
HEADLINE = W.LONG_60S
# the training, batch, sequence-parallel and projection modes default to the 5 s workload
SECONDARY = W.WAN13B_5S
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + write) of one moga_group_attn call on the 5 s Wan-1.3B
# workload (32,760 tokens x 12 heads x 128), from an ncu capture of the
# current kernels: gather3_kernel<0> 302.06 + 259.95 MB, attn_kernel<128>
# (MoGA launch) 304.74 + 158.97 MB.  Set to None whenever either kernel
# changes, until it is captured again.
# DRAM bytes (ncu dram__bytes_read.sum + dram__bytes_write.sum) of one launch
# each, captured on the 32,760-token workload (12 heads, hd 128)
TRAFFIC_UNITS = 32760 * 12 * 128
KERNEL_TRAFFIC_BYTES = 306173952 + 161697792            # attn_kernel<128>, MoGA launch
CALL_TRAFFIC_BYTES = KERNEL_TRAFFIC_BYTES + 302057472 + 259337472   # + gather3_kernel<0>


def scaled_traffic(wl, captured, what):
    """DRAM bytes of one launch (or call) on this workload: the captured
    figure, scaled by the Q/K/V elements processed for another workload (the
    copy moves every element once; the attention launch reads Q, K, V once,
    each group's K/V staying L2-resident while its tiles run, and writes the
    output once)."""
    src = "ncu dram__bytes_read.sum + dram__bytes_write.sum, " + what
    units = wl.N * wl.H * wl.hd
    if units == TRAFFIC_UNITS:
        return captured, src + " (captured on this workload)"
    return captured * units / TRAFFIC_UNITS, src + ", captured on the 32,760-token workload and scaled by N*H*hd"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return PEAKS_FALLBACK, "fallback"


def route_permute_hbm(wl, call_ms, pk):
    """Algorithmic bytes of the router (x once, g and gate out, one Σp row per 32 tokens)
    and of the permute (g in, perm out; counts and cu are negligible) over their
    CUDA-event call times, as a fraction of the measured HBM copy bandwidth; also
    the two calls as one unit (bytes of both over the sum of their times)."""
    xb = 2 if wl.x_dtype == "bf16" else 4
    route_b = wl.N * wl.d * xb + 8 * wl.N + 4 * wl.M * (-(-wl.N // 32))
    perm_b = 8 * wl.N + 8 * (wl.M + 1)
    out = {}
    tot_b, tot_ms = 0, 0.0
    for name, b in (("route", route_b), ("permute", perm_b)):
        ms = statistics.median(call_ms[name])
        gbs = b / (ms * 1e-3) / 1e9
        out[name] = {"bytes": b, "ms": ms, "gbs": gbs, "frac": gbs / pk["hbm_gbs"]}
        tot_b += b
        tot_ms += ms
    gbs = tot_b / (tot_ms * 1e-3) / 1e9
    out["unit"] = {"bytes": tot_b, "ms": tot_ms, "gbs": gbs, "frac": gbs / pk["hbm_gbs"]}
    return out


def moga_flops(counts, H, hd):
    return 4.0 * H * hd * float(np.sum(np.asarray(counts, dtype=np.float64) ** 2))


def stga_flops(wl):
    """4*H*hd*(sum over window groups n_q*n_kv + T*(hw)^2), from the geometry (readings of the pages)."""
    whw = wl.win_h * wl.win_w
    n_win = (wl.h // wl.win_h) * (wl.w // wl.win_w)
    tot = 0.0
    for s, L in enumerate(wl.shots):
        n = 1 if wl.tg_max == 0 else -(-L // wl.tg_max)
        q, r = divmod(L, n)
        for i in range(n):
            run = q + (1 if i < r else 0)
            kv = run
            if i == 0 and s > 0:
                kv += min(wl.aug, wl.shots[s - 1])
            if i == n - 1 and s + 1 < len(wl.shots):
                kv += min(wl.aug, wl.shots[s + 1])
            tot += n_win * (run * whw) * (kv * whw)
    tot += wl.T * float(wl.hw) ** 2
    return 4.0 * wl.H * wl.hd * tot


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(local_ms: float, device=None) -> float:
    """Job time: the largest per-rank device time (a one-element all-reduce outside the timed region)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, job_ms: float) -> float:
    """Whole-job tokens/s: every rank runs its own sequence of `tokens_per_rank` tokens per step."""
    return world * tokens_per_rank * steps / (job_ms / 1000.0)


def make_inputs(wl):
    """Seeded synthetic inputs (stored margin redraws applied), as numpy stored values."""
    redraw = W.redraw_map(wl)
    x = W.x_stored(wl, redraw)
    w = W.w_r_stored(wl)
    q, k, v = (W.qkv_stored(wl, n, redraw) for n in ("q", "k", "v"))
    return dict(x=x, w_r=w, q=q, k=k, v=v)


# ----------------------------------------------------------------------------- CPU oracle arm

ROUTE_CHUNK = 16384


def _f64(a):
    return W.bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def oracle_route_all(wl, inputs):
    """The oracle's routing of all N tokens (row chunks of ROUTE_CHUNK, one after another)."""
    from oracle import route as oroute
    N = wl.N
    w = _f64(inputs["w_r"])
    g = np.empty(N, dtype=np.int64)
    p_g = np.empty(N)
    p = np.empty((N, wl.M))
    for a in range(0, N, ROUTE_CHUNK):
        b = min(a + ROUTE_CHUNK, N)
        g[a:b], p_g[a:b], p[a:b] = oroute.route(_f64(inputs["x"][a:b]), w, W.bias_f64(wl))
    return g, p_g, p


def oracle_sample(wl, inputs, seed=1, n_heads=8, per_head=512, routed=None, route_fraction=1.0):
    """Times the fp64 oracle as it stands on a bounded sample of one layer forward.

    Route over all N tokens (or, with route_fraction < 1, over a contiguous
    share of them, scaled to N by token count; `routed` then supplies the
    routing of all tokens, computed outside the timed part), permute and loss
    over all N; then, for n_heads heads spread over [0, H), the three attention
    branches and the mean at a stratified sample of per_head tokens (every
    MoGA group, window group, both sides of every cut and every frame), each
    row computed from its full definition.  The attention time is
    extrapolated to the whole layer by the exact per-row cost (keys per row
    over the three branches, summed over all tokens and heads); the per-head
    widening of q, k, v to float64 is timed apart and scaled by heads.
    Returns (tokens/s, details)."""
    from oracle import layer as olayer
    from oracle import permute as opermute
    from oracle import route as oroute
    from oracle import sample as osample
    from oracle import stga as ostga

    N, H = wl.N, wl.H
    if route_fraction >= 1.0 or routed is None:
        t0 = time.perf_counter()
        g, p_g, p = oracle_route_all(wl, inputs)
        t_route = time.perf_counter() - t0
    else:
        g, p_g, p = routed
        n_r = max(1, int(N * route_fraction))
        a = (seed * 7919 * ROUTE_CHUNK) % max(N - n_r, 1)
        t0 = time.perf_counter()
        oroute.route(_f64(inputs["x"][a:a + n_r]), _f64(inputs["w_r"]), W.bias_f64(wl))
        t_route = (time.perf_counter() - t0) * N / n_r
    t0 = time.perf_counter()
    perm, cu, counts, _ = opermute.permute(g, wl.M)
    olayer.balance_loss(counts, p, wl.alpha)
    t_route += time.perf_counter() - t0

    geom = W.stga_shape(wl)
    scale = 1.0 / math.sqrt(wl.hd)
    rows = osample.stratified_rows(geom, g, wl.M, H, n_heads=n_heads, per_head=per_head, seed=seed)
    # keys per row over the three branches, for every token
    kv_moga = counts[g]
    kv_win = np.zeros(N, dtype=np.int64)
    for qt, kvt in ostga.window_groups(geom):
        kv_win[qt] = len(kvt)
    cost_tok = kv_moga + kv_win + wl.hw
    t_conv = t_rows = t_mean = 0.0
    n_rows = 0
    cost_sample = 0.0
    for h, toks in rows.items():
        t0 = time.perf_counter()
        qh, kh, vh = (W.bf16_bits_to_f64(inputs[n][:, h, :]) for n in ("q", "k", "v"))
        t_conv += time.perf_counter() - t0
        t0 = time.perf_counter()
        om, ow, of = osample.branch_rows(qh, kh, vh, toks, g, p_g, wl.M, geom, scale)
        t_rows += time.perf_counter() - t0
        t0 = time.perf_counter()
        olayer.mean3(om, ow, of)
        t_mean += time.perf_counter() - t0
        n_rows += len(toks)
        cost_sample += float(cost_tok[toks].sum())
    cost_total = float(cost_tok.sum()) * H
    t_attn = t_conv / len(rows) * H + t_rows * cost_total / cost_sample
    t_mean_all = t_mean * (N * H) / n_rows
    t_layer = t_route + t_attn + t_mean_all
    return N / t_layer, dict(t_route_s=t_route, t_conv_s=t_conv, t_rows_s=t_rows, t_mean_s=t_mean,
                             heads=len(rows), rows=n_rows, t_layer_extrapolated_s=t_layer,
                             route_fraction=min(route_fraction, 1.0) if routed is not None else 1.0)


def oracle_sample_text(wl, det):
    if det.get("route_fraction", 1.0) < 1.0:
        route = ("route timed on a contiguous %.1f %% of the tokens and scaled to all %d, permute+loss over all "
                 "(%.1f s)" % (100 * det["route_fraction"], wl.N, det["t_route_s"]))
    else:
        route = "route+permute+loss over all %d tokens (%.1f s)" % (wl.N, det["t_route_s"])
    return ("fp64 oracle, extrapolated: %s; attention (MoGA, window, frame) + mean at a stratified sample of %d "
            "(token, head) rows over %d of %d heads covering every group, window group, cut side and frame "
            "(%.1f s rows + %.1f s widening), scaled by exact per-row key counts to all %d x %d rows -> %.0f s "
            "per layer" % (route, det["rows"], det["heads"], wl.H, det["t_rows_s"], det["t_conv_s"], wl.N, wl.H,
                           det["t_layer_extrapolated_s"]))


def host_cores():
    """(cpus the host offers, BLAS threads numpy's matmul uses)."""
    blas = None
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        blas = max(n) if n else None
    except Exception:
        blas = None
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count() or 1
    return avail, (blas if blas is not None else 1)


def cpu_baseline_dict(wl, value, det):
    avail, blas = host_cores()
    return {"value": value, "unit": "tokens/s", "cores": blas, "host_cpus": avail, "blas_threads": blas,
            "kind": "oracle", "sample": oracle_sample_text(wl, det)}


def pick_workload(args, default):
    """The suite workload named by --workload (its stored skew bias filled in), else `default`."""
    return W.resolved(W.SUITE[args.workload] if args.workload else default)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = pick_workload(args, HEADLINE)
    inputs = make_inputs(wl)
    # the routing of all tokens once, outside the steps: it defines the groups
    # the attention sample needs; each step times the router on an eighth of
    # the tokens and 4 heads of attention rows, so a run of tens of steps ends
    # within a few minutes on a few host cores
    routed = oracle_route_all(wl, inputs)
    frac = 1.0 if wl.N <= 65536 else 0.125
    for i in range(args.warmup):
        oracle_sample(wl, inputs, seed=100 + i, n_heads=2, per_head=256, routed=routed, route_fraction=frac)
    t0 = time.perf_counter()
    res = [oracle_sample(wl, inputs, seed=1 + s, n_heads=4, routed=routed, route_fraction=frac)
           for s in range(args.steps)]
    el = time.perf_counter() - t0
    value = float(statistics.median([r[0] for r in res]))
    det = res[len(res) // 2][1]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(wl),
            "cpu_baseline": cpu_baseline_dict(wl, value, det),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl):
    return {"workload": wl.name, "tokens": wl.N, "frames": wl.T, "grid": [wl.h, wl.w], "d": wl.d,
            "heads": wl.H, "head_dim": wl.hd, "M": wl.M, "shots": list(wl.shots), "tg_max": wl.tg_max,
            "window": [wl.win_h, wl.win_w], "aug_frames": wl.aug, "router": router_kind(wl),
            "sequences_per_gpu": 1, "l2": "flushed between timed steps (256 MiB write); inputs exceed L2",
            "parallelism": "independent sequences per GPU"}


def router_kind(wl):
    if wl.clusters:
        return "clustered input (%d Gaussian centres)" % wl.clusters
    if wl.bias0 is not None:
        return "skewed (bias on group 0)"
    return "i.i.d. input"


# ----------------------------------------------------------------------------- GPU arm

def run_e2e(args, world, dev, inp, step, out, loss, flush, stream, N):
    """The step end to end through the C ABI: every step copies its inputs in
    from pinned host memory and its result out, inside the timed region."""
    import torch
    import torch.distributed as dist
    import sparse_attention_long_moga_b200 as moga
    hx, hq, hk, hv = (torch.from_numpy(inp[n].view(np.int16)).pin_memory() for n in ("x", "q", "k", "v"))
    hosts = (hx, hq, hk, hv)
    hout = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    hloss = torch.empty(1, dtype=torch.float64).pin_memory()
    h2d = sum(a.numel() * a.element_size() for a in hosts)
    d2h = hout.numel() * 2 + 8
    bf = lambda t: t.view(torch.bfloat16)  # noqa: E731
    # (a) serial: each step copies its inputs in, runs, and copies its result
    # out on one stream
    xd, qd, kd, vd = (torch.empty_like(a, device=dev) for a in hosts)
    e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e_evs[i][0].record(stream)
        for dst, src in zip((xd, qd, kd, vd), hosts):
            dst.copy_(src, non_blocking=True)
        step(bf(xd), bf(qd), bf(kd), bf(vd))
        hout.copy_(out, non_blocking=True)
        hloss.copy_(loss, non_blocking=True)
        e_evs[i][1].record(stream)
    torch.cuda.synchronize()
    serial_ms = sum(a.elapsed_time(b) for a, b in e_evs)
    want_out, want_loss = hout.clone(), hloss.clone()
    # (b) pipelined, as a stream of requests is served: step i's inputs go
    # into buffer set i % 2 on a host-to-device stream and its result leaves
    # output buffer i % 2 on a device-to-host stream, so the copies of one
    # step overlap the kernels of its neighbours.  Every step's copies lie
    # inside the timed region; its 400 MB of fresh inputs exceed L2.
    ins = [(xd, qd, kd, vd), tuple(torch.empty_like(a, device=dev) for a in hosts)]
    outs = [(out, loss), (torch.empty_like(out), torch.empty_like(loss))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: [torch.cuda.Event() for _ in range(args.steps)]  # noqa: E731
    copied, computed, returned = ev(), ev(), ev()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    s_in.wait_stream(stream)
    for i in range(args.steps):
        b = i & 1
        if i >= 2:
            s_in.wait_event(computed[i - 2])      # step i-2 has read buffer set b
        with torch.cuda.stream(s_in):
            for dst, src in zip(ins[b], hosts):
                dst.copy_(src, non_blocking=True)
        copied[i].record(s_in)
        stream.wait_event(copied[i])
        if i >= 2:
            stream.wait_event(returned[i - 2])    # output buffer b has left
        step(*(bf(t) for t in ins[b]), out=outs[b][0], loss=outs[b][1])
        computed[i].record(stream)
        s_out.wait_event(computed[i])
        with torch.cuda.stream(s_out):
            hout.copy_(outs[b][0], non_blocking=True)
            hloss.copy_(outs[b][1], non_blocking=True)
        returned[i].record(s_out)
    stream.wait_event(returned[-1])
    t1.record(stream)
    torch.cuda.synchronize()
    pipe_ms = t0.elapsed_time(t1)
    moga.device_status()
    # the last step's result crossed the streams intact
    if not (torch.equal(hout, want_out) and torch.equal(hloss, want_loss)):
        raise RuntimeError("pipelined end-to-end result differs from the serial one")
    e2e_value = job_throughput(world, N, args.steps, max_over_ranks(pipe_ms, dev))
    e2e_serial = job_throughput(world, N, args.steps, max_over_ranks(serial_ms, dev))
    return {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": True, "ms_per_step": pipe_ms / args.steps, "serial_value": e2e_serial,
            "serial_ms_per_step": serial_ms / args.steps}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import sparse_attention_long_moga_b200 as moga
    wl = pick_workload(args, HEADLINE)
    inp = make_inputs(wl)
    geom = W.stga_shape(wl)

    def to_dev(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev).view(torch.bfloat16) if a.dtype == np.uint16 else t.to(dev)

    x, w_r, q, k, v = (to_dev(inp[n]) for n in ("x", "w_r", "q", "k", "v"))
    N, M, H, hd = wl.N, wl.M, wl.H, wl.hd
    bias = None
    if wl.bias0 is not None:
        bias = torch.from_numpy(W.bias_f64(wl).astype(np.float32)).to(dev)
    L = moga._lib.lib()
    stream = torch.cuda.current_stream()
    sp = moga._stream()
    P = moga._ptr

    # persistent buffers: the step allocates nothing
    g = torch.empty(N, dtype=torch.int32, device=dev)
    gate = torch.empty(N, dtype=torch.float32, device=dev)
    rws = torch.empty(max(L.moga_route_ws_bytes(N, wl.d, M), 16), dtype=torch.uint8, device=dev)
    pws = torch.empty(max(L.moga_permute_ws_bytes(N, M), 16), dtype=torch.uint8, device=dev)
    perm = torch.empty(N, dtype=torch.int32, device=dev)
    cu = torch.empty(M + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(M, dtype=torch.int32, device=dev)
    mx = torch.empty(1, dtype=torch.int32, device=dev)
    o_acc = torch.empty((N, H, hd), dtype=torch.float32, device=dev)
    out = torch.empty((N, H, hd), dtype=torch.bfloat16, device=dev)
    loss = torch.empty(1, dtype=torch.float64, device=dev)
    ws_fn = L.visual_attn_ws_bytes if args.combined else L.moga_attn_ws_bytes
    aws = torch.empty(ws_fn(N, H, hd), dtype=torch.uint8, device=dev)
    gs, keep = moga.geom_struct(geom)
    scale = 1.0 / math.sqrt(hd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if args.combined:
        CALLS = ("route", "permute", "visual_attn_branches", "visual_attn_mean", "moga_balance_loss")
    elif not args.fused_mean:
        CALLS = ("route", "permute", "moga_group_attn", "stga_attn", "visual_attn_mean", "moga_balance_loss")
    else:
        CALLS = ("route", "permute", "moga_group_attn", "stga_attn_mean", "moga_balance_loss")
    evl = [torch.cuda.Event(enable_timing=True) for _ in range(len(CALLS) + 1)]
    # the attention launches alone, without their gather copies: the library
    # records these events around the attention-kernel launches of a call
    attn_calls = CALLS[2:3] if args.combined else CALLS[2:4]
    hook = L.moga_test_set_attn_events
    hook.restype = None
    hook.argtypes = [moga.ctypes.c_void_p, moga.ctypes.c_void_p]
    kev = {name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)] for name in attn_calls}
    for pairs in kev.values():
        for a, b in pairs:   # creates the handles
            a.record(stream)
            b.record(stream)
    t_index = [0]

    def step(xd, qd, kd, vd, timed=False, out=out, loss=loss):
        c = moga.check

        def mark(i):
            if timed:
                evl[i].record(stream)

        def arm(name):
            if timed:
                hook(*kev[name][t_index[0]])

        def disarm():
            if timed:
                hook(None, None)
        mark(0)
        c(L.moga_route(P(xd), P(w_r), moga.MOGA_BF16, P(bias) if bias is not None else None, N, wl.d, M, P(g),
                       P(gate), P(rws), rws.numel(), sp), "route")
        mark(1)
        c(L.moga_permute(P(g), N, M, P(perm), P(cu), P(counts), P(mx), P(pws), pws.numel(), sp), "permute")
        mark(2)
        if args.combined:
            # the three branches with one gather of Q, K, V into both orders
            arm(CALLS[2])
            c(L.visual_attn_branches(P(qd), P(kd), P(vd), N, H, hd, P(perm), P(cu), M, P(gate),
                                     moga.ctypes.byref(gs), scale, P(o_acc), P(aws), aws.numel(), sp), "branches")
            disarm()
            mark(3)
            c(L.visual_attn_mean(P(o_acc), o_acc.numel(), P(out), sp), "mean")
            mark(len(CALLS) - 1)
            c(L.moga_balance_loss(P(counts), P(rws), N, M, wl.alpha, P(loss), sp), "loss")
            mark(len(CALLS))
            return
        arm(CALLS[2])
        c(L.moga_group_attn(P(qd), P(kd), P(vd), N, H, hd, P(perm), P(cu), M, P(gate), scale, P(o_acc), P(aws),
                            aws.numel(), sp), "moga")
        disarm()
        mark(3)
        arm(CALLS[3])
        if not args.fused_mean:
            c(L.stga_attn(P(qd), P(kd), P(vd), H, hd, moga.ctypes.byref(gs), scale, P(o_acc), P(aws), aws.numel(),
                          sp), "stga")
            disarm()
            mark(4)
            c(L.visual_attn_mean(P(o_acc), o_acc.numel(), P(out), sp), "mean")
        else:
            # the three-way mean taken inside the frame pass of STGA
            c(L.stga_attn_mean(P(qd), P(kd), P(vd), H, hd, moga.ctypes.byref(gs), scale, P(o_acc), P(out), P(aws),
                               aws.numel(), sp), "stga_mean")
            disarm()
        mark(len(CALLS) - 1)
        c(L.moga_balance_loss(P(counts), P(rws), N, M, wl.alpha, P(loss), sp), "loss")
        mark(len(CALLS))

    # route 2 (W_r^T copy + tensor-core router), permute 3, MoGA gather + attention 2,
    # STGA gather + window + frame 3, loss 1 (+ mean 1 and its tail when not fused)
    launches_per_step = 2 + 3 + 2 + 3 + 1
    if args.combined:   # one gather instead of two
        launches_per_step -= 1
    if not args.fused_mean:
        launches_per_step += 1 + (1 if (N * H * hd) % 8 else 0)

    for _ in range(args.warmup):
        flush.zero_()
        step(x, q, k, v)
    moga.device_status()

    # ---- device-timed region: K steps, L2 flushed between steps
    sampler = ClockSampler(local)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    call_ms = {name: [] for name in CALLS}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(args.steps):
        flush.zero_()
        t_index[0] = i
        evs[i][0].record(stream)
        step(x, q, k, v, timed=True)
        evs[i][1].record(stream)
        evl[-1].synchronize()
        for j, name in enumerate(CALLS):
            call_ms[name].append(evl[j].elapsed_time(evl[j + 1]))
    kern_ms = {name: [a.elapsed_time(b) for a, b in pairs] for name, pairs in kev.items()}
    moga_ms = call_ms[CALLS[2]]   # moga_group_attn, or the combined call
    moga_kern_ms = kern_ms[CALLS[2]]
    torch.cuda.synchronize()
    clocks = sampler.stop()
    moga.device_status()
    dev_ms = sum(a.elapsed_time(b) for a, b in evs)
    if world > 1:
        dist.barrier()
    job_ms = max_over_ranks(dev_ms, dev)
    value = job_throughput(world, N, args.steps, job_ms)

    # ---- end to end through the C ABI: pinned host inputs in, result out
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, world, dev, inp, step, out, loss, flush, stream, N)

    counts_h = counts.cpu().numpy()
    fl_moga = moga_flops(counts_h, H, hd)
    fl_stga = stga_flops(wl)
    pk, pk_kind = peaks()
    moga_avg_s = statistics.mean(moga_ms) / 1000.0
    kern_avg_s = statistics.mean(moga_kern_ms) / 1000.0
    # the combined call runs all three branches: its FLOPs are MoGA + STGA
    fl_call = fl_moga + fl_stga if args.combined else fl_moga
    achieved = fl_call / kern_avg_s / 1e12
    call_achieved = fl_call / moga_avg_s / 1e12
    # a kernel timed inside a timed region of seconds runs under the power
    # cap: the sustained peak applies; a short region gets the burst peak
    sustained = job_ms > 1000.0
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    if args.combined:
        traffic, traffic_src = None, "not captured for the combined call"
        call_traffic, call_traffic_src = None, traffic_src
    else:
        traffic, traffic_src = scaled_traffic(wl, KERNEL_TRAFFIC_BYTES, "attn_kernel<128> MoGA launch")
        call_traffic, call_traffic_src = scaled_traffic(wl, CALL_TRAFFIC_BYTES,
                                                        "gather3_kernel<0> + attn_kernel<128> MoGA launch")
    stga_tf = stga_call_tf = None
    if not args.combined:
        stga_tf = fl_stga / (statistics.median(kern_ms[CALLS[3]]) / 1000.0) / 1e12
        stga_call_tf = fl_stga / (statistics.median(call_ms[CALLS[3]]) / 1000.0) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": job_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator; no dataset)",
        "config": config_dict(wl),
        "roofline": {"bound": "tensor",
                     "kernel": ("attn_kernel<128>: the MoGA, window and frame launches of visual_attn_branches"
                                if args.combined else "attn_kernel<128>: the MoGA launch of moga_group_attn"),
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": "%s %s dense bf16" % (pk_kind, "sustained" if sustained else "burst"),
                     "frac_of_burst": achieved / pk["bf16_tflops"],
                     "traffic": traffic, "traffic_source": traffic_src,
                     "flops_per_launch": fl_call, "launch_ms": kern_avg_s * 1e3,
                     "timing": "CUDA events recorded by the library around the attention launch(es) of each "
                               "timed call, on the launching stream"},
        "attention_call_roofline": {
            "call": ("visual_attn_branches = gather_both_kernel + attn_kernel<128> x 3" if args.combined else
                     "moga_group_attn = gather3_kernel<0> (segment-order copy) + attn_kernel<128>"),
            "achieved": call_achieved, "frac": call_achieved / peak, "frac_of_burst": call_achieved / pk["bf16_tflops"],
            "call_ms": moga_avg_s * 1e3, "traffic": call_traffic, "traffic_source": call_traffic_src},
        "layer_tflops": (fl_moga + fl_stga) / (job_ms / args.steps / 1000.0) / 1e12,
        "breakdown_ms": {name: statistics.median(v) for name, v in call_ms.items()},
        "attention_kernels_ms": {name: statistics.median(v) for name, v in kern_ms.items()},
        "stga_tflops": stga_tf,
        "stga_frac": stga_tf / peak if stga_tf is not None else None,
        "stga_call_tflops": stga_call_tf,
        "attention_call": "visual_attn_branches (one gather)" if args.combined else "moga_group_attn + stga_attn",
        "group_sizes": {"min": int(counts_h.min()), "max": int(counts_h.max()), "sum_sq": float(np.sum(
            counts_h.astype(np.float64) ** 2))},
        "mean_fused_into_stga": bool(args.fused_mean),
        "route_permute_hbm": route_permute_hbm(wl, call_ms, pk),
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_val, det = oracle_sample(wl, inp)
        line["cpu_baseline"] = cpu_baseline_dict(wl, cpu_val, det)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    del keep
    return 0


def run_route(args):
    """The router alone on the workload's x and W_r (and the permute of its
    group ids): CUDA-event time per call with L2 flushed in between, GB/s and
    fraction of the measured HBM bandwidth.  Prints one JSON line (not the
    forward headline line)."""
    import torch
    import sparse_attention_long_moga_b200 as moga
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    wl = pick_workload(args, HEADLINE)
    redraw = W.redraw_map(wl)
    x_st = W.x_stored(wl, redraw)
    if x_st.dtype != np.uint16:
        raise SystemExit("--route times the bf16 router; %s has fp32 input" % wl.name)
    x = torch.from_numpy(x_st.view(np.int16)).to(dev).view(torch.bfloat16)
    w = torch.from_numpy(W.w_r_stored(wl).view(np.int16)).to(dev).view(torch.bfloat16)
    bias = None
    if wl.bias0 is not None:
        bias = torch.from_numpy(W.bias_f64(wl).astype(np.float32)).to(dev)
    del x_st
    N, d, M = wl.N, wl.d, wl.M
    L = moga._lib.lib()
    P = moga._ptr
    sp = moga._stream()
    stream = torch.cuda.current_stream()
    g = torch.empty(N, dtype=torch.int32, device=dev)
    gate = torch.empty(N, dtype=torch.float32, device=dev)
    rws = torch.empty(max(L.moga_route_ws_bytes(N, d, M), 16), dtype=torch.uint8, device=dev)
    pws = torch.empty(max(L.moga_permute_ws_bytes(N, M), 16), dtype=torch.uint8, device=dev)
    perm = torch.empty(N, dtype=torch.int32, device=dev)
    cu = torch.empty(M + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(M, dtype=torch.int32, device=dev)
    mx = torch.empty(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def route():
        moga.check(L.moga_route(P(x), P(w), moga.MOGA_BF16, P(bias) if bias is not None else None, N, d, M, P(g),
                                P(gate), P(rws), rws.numel(), sp), "route")

    def permute():
        moga.check(L.moga_permute(P(g), N, M, P(perm), P(cu), P(counts), P(mx), P(pws), pws.numel(), sp), "permute")

    for _ in range(args.warmup):
        route()
        permute()
    moga.device_status()
    ms = {"route": [], "permute": []}
    for _ in range(args.steps):
        for name, fn in (("route", route), ("permute", permute)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ms[name].append(a.elapsed_time(b))
    moga.device_status()
    pk, pk_kind = peaks()
    hbm = route_permute_hbm(wl, ms, pk)
    line = {"metric": "router and permute alone, GB/s (bf16 x)", "value": hbm["unit"]["gbs"], "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (seeded counter-based generator; no dataset)",
            "config": {"workload": wl.name, "tokens": N, "d": d, "M": M,
                       "l2": "flushed before every timed call (256 MiB write)"},
            "route_permute_hbm": hbm, "peak_kind": "%s HBM copy bandwidth" % pk_kind}
    print(json.dumps(line), flush=True)
    return 0


def run_train(args):
    """Training step on one GPU: the saving forward (route with probabilities, permute,
    MoGA and STGA with per-branch outputs and log-sum-exp, mean, loss) followed by the
    backward (attention branches, gate, router and loss), through the C ABI with
    persistent buffers.  Prints one JSON line (not the forward headline line)."""
    import torch

    import sparse_attention_long_moga_b200 as moga
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    wl = pick_workload(args, SECONDARY)
    inp = make_inputs(wl)
    geom = W.stga_shape(wl)

    def to_dev(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev).view(torch.bfloat16) if a.dtype == np.uint16 else t.to(dev)

    x, w_r, q, k, v = (to_dev(inp[n]) for n in ("x", "w_r", "q", "k", "v"))
    dout = torch.from_numpy(W.dout_bits(wl).view(np.int16)).to(dev).view(torch.bfloat16)
    N, M, H, hd, d = wl.N, wl.M, wl.H, wl.hd, wl.d
    L = moga._lib.lib()
    sp = moga._stream()
    P = moga._ptr
    stream = torch.cuda.current_stream()
    f32 = dict(dtype=torch.float32, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    g, perm, counts, mx, cu = (torch.empty(n, **i32) for n in (N, N, M, 1, M + 1))
    gate, dgate = torch.empty(N, **f32), torch.empty(N, **f32)
    probs = torch.empty((N, M), **f32)
    rws = torch.empty(max(L.moga_route_ws_bytes(N, d, M), 16), dtype=torch.uint8, device=dev)
    pws = torch.empty(max(L.moga_permute_ws_bytes(N, M), 16), dtype=torch.uint8, device=dev)
    aws = torch.empty(L.moga_attn_ws_bytes(N, H, hd), dtype=torch.uint8, device=dev)
    bws = torch.empty(L.moga_attn_bwd_ws_bytes(N, H, hd), dtype=torch.uint8, device=dev)
    rbws = torch.empty(L.moga_route_bwd_ws_bytes(N, d, M), dtype=torch.uint8, device=dev)
    o_moga, o_win, o_frame, dq, dk, dv = (torch.empty((N, H, hd), **f32) for _ in range(6))
    lse_moga, lse_win, lse_frame = (torch.empty((N, H), **f32) for _ in range(3))
    out = torch.empty((N, H, hd), dtype=torch.bfloat16, device=dev)
    loss = torch.empty(1, dtype=torch.float64, device=dev)
    dx, dw_r = torch.empty((N, d), **f32), torch.empty((d, M), **f32)
    gs, keep = moga.geom_struct(geom)
    scale = 1.0 / math.sqrt(hd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    CALLS = ("moga_route_train", "moga_permute", "moga_group_attn_train", "stga_attn_train", "visual_attn_mean3",
             "moga_balance_loss", "zero_grads", "moga_group_attn_bwd", "stga_attn_bwd", "moga_route_bwd")

    def step(evl=None):
        c = moga.check

        def mark(i):
            if evl is not None:
                evl[i].record(stream)
        mark(0)
        c(L.moga_route_train(P(x), P(w_r), moga.MOGA_BF16, None, N, d, M, P(g), P(gate), P(probs), P(rws),
                             rws.numel(), sp), "route")
        mark(1)
        c(L.moga_permute(P(g), N, M, P(perm), P(cu), P(counts), P(mx), P(pws), pws.numel(), sp), "permute")
        mark(2)
        c(L.moga_group_attn_train(P(q), P(k), P(v), N, H, hd, P(perm), P(cu), M, P(gate), scale, P(o_moga),
                                  P(lse_moga), P(aws), aws.numel(), sp), "moga")
        mark(3)
        c(L.stga_attn_train(P(q), P(k), P(v), H, hd, moga.ctypes.byref(gs), scale, P(o_win), P(lse_win),
                            P(o_frame), P(lse_frame), P(aws), aws.numel(), sp), "stga")
        mark(4)
        c(L.visual_attn_mean3(P(o_moga), P(o_win), P(o_frame), out.numel(), P(out), sp), "mean3")
        mark(5)
        c(L.moga_balance_loss(P(counts), P(rws), N, M, wl.alpha, P(loss), sp), "loss")
        mark(6)
        for t in (dq, dk, dv):
            t.zero_()
        mark(7)
        c(L.moga_group_attn_bwd(P(q), P(k), P(v), N, H, hd, P(perm), P(cu), M, P(gate), scale, P(o_moga),
                                P(lse_moga), P(dout), P(dq), P(dk), P(dv), P(dgate), P(bws), bws.numel(), sp),
          "moga bwd")
        mark(8)
        c(L.stga_attn_bwd(P(q), P(k), P(v), H, hd, moga.ctypes.byref(gs), scale, P(o_win), P(lse_win), P(o_frame),
                          P(lse_frame), P(dout), P(dq), P(dk), P(dv), P(bws), bws.numel(), sp), "stga bwd")
        mark(9)
        c(L.moga_route_bwd(P(x), P(w_r), moga.MOGA_BF16, N, d, M, P(g), P(probs), P(dgate), P(counts), wl.alpha, 1.0,
                           P(dx), P(dw_r), None, P(rbws), rbws.numel(), sp), "route bwd")
        mark(10)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    moga.device_status()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(CALLS) + 1)] for _ in range(args.steps)]
    sampler = ClockSampler(0)
    torch.cuda.synchronize()
    sampler.start()
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    moga.device_status()
    call_ms = {name: statistics.median(e[j].elapsed_time(e[j + 1]) for e in evs) for j, name in enumerate(CALLS)}
    step_ms = statistics.median(e[0].elapsed_time(e[-1]) for e in evs)
    fl_fwd_moga = moga_flops(counts.cpu().numpy(), H, hd)
    fl_fwd_stga = stga_flops(wl)
    pk, pk_kind = peaks()
    # attention backward FLOPs in the usual convention: 2.5 x forward (dV, dP, dQ, dK
    # and the recomputed S; the dQ pass recomputes S and dP once more on top of that)
    bwd_moga_tf = 2.5 * fl_fwd_moga / (call_ms["moga_group_attn_bwd"] * 1e-3) / 1e12
    bwd_stga_tf = 2.5 * fl_fwd_stga / (call_ms["stga_attn_bwd"] * 1e-3) / 1e12
    route_bwd_bytes = N * d * (2 + 4)
    line = {
        "metric": "visual-attn layer training step (fwd + bwd) tokens/s (bf16)", "value": N / (step_ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded counter-based generator; no dataset)",
        "config": config_dict(wl), "breakdown_ms": call_ms,
        "route_bwd_hbm": {"bytes": route_bwd_bytes, "gbs": route_bwd_bytes / (call_ms["moga_route_bwd"] * 1e-3) / 1e9,
                          "frac": route_bwd_bytes / (call_ms["moga_route_bwd"] * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "what": "x read (bf16) + dx written (fp32) over the moga_route_bwd call"},
        "attn_bwd_tflops": {"moga": bwd_moga_tf, "stga": bwd_stga_tf,
                            "moga_frac_of_peak": bwd_moga_tf / pk["bf16_tflops"],
                            "convention": "2.5 x forward FLOPs (4*H*hd*sum n_q*n_kv)"},
        "peak": {"bf16_tflops": pk["bf16_tflops"], "kind": pk_kind},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_batch(args):
    """Forward over a batch of B videos of the 5 s Wan-1.3B shape at M = 20 (the
    pages' MMDiT group count), per-video groups: route over the B*N tokens,
    batched permute (B*M segments), batched MoGA, batched STGA, mean and the
    batch loss, through the C ABI with persistent buffers.  One JSON line
    (not the headline line)."""
    import torch

    import sparse_attention_long_moga_b200 as moga
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    B = args.batch
    per = pick_workload(args, SECONDARY).with_(M=20)
    big = per.with_(name="%s_x%d" % (per.name, B), T=per.T * B, shots=tuple(per.shots) * B)
    inp = make_inputs(big)
    geom = W.stga_shape(per)

    def to_dev(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev).view(torch.bfloat16) if a.dtype == np.uint16 else t.to(dev)

    x, w_r, q, k, v = (to_dev(inp[n]) for n in ("x", "w_r", "q", "k", "v"))
    n, M, H, hd, d = per.N, per.M, per.H, per.hd, per.d
    N = B * n
    L = moga._lib.lib()
    sp = moga._stream()
    P = moga._ptr
    i32 = dict(dtype=torch.int32, device=dev)
    g, perm, counts, mx, cu = (torch.empty(c, **i32) for c in (N, N, B * M, 1, B * M + 1))
    gate = torch.empty(N, dtype=torch.float32, device=dev)
    rws = torch.empty(max(L.moga_route_ws_bytes(N, d, M), 16), dtype=torch.uint8, device=dev)
    pws = torch.empty(max(L.moga_permute_batched_ws_bytes(n, B, M), 16), dtype=torch.uint8, device=dev)
    aws = torch.empty(L.moga_attn_ws_bytes(N, H, hd), dtype=torch.uint8, device=dev)
    o = torch.empty((N, H, hd), dtype=torch.float32, device=dev)
    out = torch.empty((N, H, hd), dtype=torch.bfloat16, device=dev)
    loss = torch.empty(1, dtype=torch.float64, device=dev)
    gs, keep = moga.geom_struct(geom)
    scale = 1.0 / math.sqrt(hd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        c = moga.check
        c(L.moga_route(P(x), P(w_r), moga.MOGA_BF16, None, N, d, M, P(g), P(gate), P(rws), rws.numel(), sp), "route")
        c(L.moga_permute_batched(P(g), n, B, M, P(perm), P(cu), P(counts), P(mx), P(pws), pws.numel(), sp), "permute")
        c(L.moga_group_attn_batched(P(q), P(k), P(v), n, B, H, hd, P(perm), P(cu), M, P(gate), scale, P(o), None,
                                    P(aws), aws.numel(), sp), "moga")
        c(L.stga_attn_batched(P(q), P(k), P(v), B, H, hd, moga.ctypes.byref(gs), scale, P(o), P(aws), aws.numel(), sp),
          "stga")
        c(L.visual_attn_mean(P(o), o.numel(), P(out), sp), "mean")
        c(L.moga_balance_loss_batched(P(counts), B, P(rws), N, M, per.alpha, P(loss), sp), "loss")

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    moga.device_status()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(0)
    torch.cuda.synchronize()
    sampler.start()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    moga.device_status()
    step_ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    cnt = counts.cpu().numpy()
    flops = moga_flops(cnt, H, hd) + B * stga_flops(per)
    pk, pk_kind = peaks()
    cfg = config_dict(per)
    cfg.update({"workload": "%s, batch of %d videos, M=20" % (per.name, B), "batch": B, "tokens": N,
                "sequences_per_gpu": B, "parallelism": "per-video groups in one batch"})
    line = {
        "metric": "visual-attn layer fwd tokens/s, batch of videos (bf16)", "value": N / (step_ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded counter-based generator; no dataset)",
        "config": cfg, "layer_tflops": flops / (step_ms * 1e-3) / 1e12,
        "layer_frac_of_peak": flops / (step_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
        "peak": {"bf16_tflops": pk["bf16_tflops"], "kind": pk_kind}, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    del keep
    return 0


def run_sp(args):
    """Sequence-parallel forward: ONE 5 s Wan-1.3B video sharded over the N ranks
    (rank r holds tokens [r n, (r+1) n)), routing all-gathered, Q/K/V exchanged
    to head shards by all-to-all, the layer per head shard, the output
    exchanged back (sparse_attention_long_moga_b200.sp).  Strong scaling; the
    step time includes the collectives; max over ranks.  One JSON line."""
    import datetime

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if not dist.is_initialized():
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import sparse_attention_long_moga_b200 as moga
    from sparse_attention_long_moga_b200.sp import sp_visual_attention_forward
    wl = pick_workload(args, SECONDARY)
    if wl.H % world or wl.N % world:
        if rank == 0:
            print(json.dumps({"metric": "visual-attn layer fwd tokens/s, sequence-parallel (bf16)",
                              "unavailable": "%d ranks do not divide %d heads and %d tokens" % (world, wl.H, wl.N)}))
        dist.destroy_process_group()
        return 0
    inp = make_inputs(wl)
    geom = W.stga_shape(wl)
    n = wl.N // world
    sl = slice(rank * n, (rank + 1) * n)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a))
        return t.to(dev).view(torch.bfloat16) if a.dtype == np.uint16 else t.to(dev)

    x, q, k, v = (to_dev(inp[nm][sl]) for nm in ("x", "q", "k", "v"))
    w_r = to_dev(inp["w_r"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return sp_visual_attention_forward(x, w_r, None, q, k, v, wl.M, geom, wl.alpha)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    moga.device_status()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    moga.device_status()
    local_ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    step_ms = max_over_ranks(local_ms, device=dev)
    if rank == 0:
        cfg = config_dict(wl)
        cfg.update({"sequences_per_gpu": 1.0 / world, "parallelism": "sequence parallel over %d GPUs (routing "
                    "all-gather, Q/K/V all-to-all to head shards, output all-to-all back; NCCL)" % world})
        print(json.dumps({
            "metric": "visual-attn layer fwd tokens/s, sequence-parallel (bf16)", "value": wl.N / (step_ms * 1e-3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "strong", "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator; no dataset)", "config": cfg, "clocks": clocks}),
            flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_qkv(args):
    """The router fused into the Q/K/V projection on the 5 s Wan-1.3B workload (x
    [32760, 1536] bf16, W_qkv [4608, 1536]): moga_qkv_route timed against the unfused
    pair it replaces, a library GEMM (torch.matmul, cuBLAS) plus moga_route.  One JSON
    line (not the headline line)."""
    import torch

    import sparse_attention_long_moga_b200 as moga
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    wl = pick_workload(args, SECONDARY)
    inp = make_inputs(wl)
    x = torch.from_numpy(inp["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    w_r = torch.from_numpy(inp["w_r"].view(np.int16)).to(dev).view(torch.bfloat16)
    wq = np.ascontiguousarray(np.concatenate([W.proj_weight_bits(wl, c) for c in "qkv"], axis=1).T)
    w_qkv = torch.from_numpy(wq.view(np.int16)).to(dev).view(torch.bfloat16)
    N, d, H, hd, M = wl.N, wl.d, wl.H, wl.hd, wl.M
    L = moga._lib.lib()
    P = moga._ptr
    sp = moga._stream()
    q, k, v = (torch.empty((N, H, hd), dtype=torch.bfloat16, device=dev) for _ in range(3))
    y = torch.empty((N, 3 * H * hd), dtype=torch.bfloat16, device=dev)
    g = torch.empty(N, dtype=torch.int32, device=dev)
    gate = torch.empty(N, dtype=torch.float32, device=dev)
    ws = torch.empty(L.moga_qkv_route_ws_bytes(N, d, M), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def fused():
        moga.check(L.moga_qkv_route(P(x), P(w_qkv), P(w_r), None, N, d, H, hd, M, P(q), P(k), P(v), P(g), P(gate),
                                    P(ws), ws.numel(), sp), "qkv_route")

    def unfused():
        torch.matmul(x, w_qkv.t(), out=y)
        moga.check(L.moga_route(P(x), P(w_r), moga.MOGA_BF16, None, N, d, M, P(g), P(gate), P(ws), ws.numel(), sp),
                   "route")

    def timeit(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    sampler = ClockSampler(0)
    sampler.start()
    t_f = timeit(fused)
    t_u = timeit(unfused)
    clocks = sampler.stop()
    moga.device_status()
    flops = 2.0 * N * d * (3 * H * hd + M)
    pk, pk_kind = peaks()
    line = {"metric": "Q/K/V projection with the router fused in, tokens/s (bf16)", "value": N / (t_f * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_f,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded counter-based generator; no dataset)",
            "config": {"workload": wl.name + ", x [%d, %d] . W_qkv^T [%d, %d] + router M=%d" % (N, d, 3 * H * hd, d, M)},
            "fused_tflops": flops / (t_f * 1e-3) / 1e12,
            "fused_frac_of_peak": flops / (t_f * 1e-3) / 1e12 / pk["bf16_tflops"],
            "unfused_ms": t_u, "unfused_what": "torch.matmul (cuBLAS) + moga_route",
            "peak": {"bf16_tflops": pk["bf16_tflops"], "kind": pk_kind}, "clocks": clocks}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(W.SUITE), default=None,
                    help="suite workload (default: %s for the forward, %s for the other modes)"
                    % (HEADLINE.name, SECONDARY.name))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (host copies), e.g. for a profiler's launch list")
    ap.add_argument("--combined", action="store_true",
                    help="run the three attention branches as one visual_attn_branches call (one gather pass)")
    ap.add_argument("--fused-mean", action="store_true",
                    help="run stga_attn_mean (mean inside the STGA frame pass) instead of stga_attn + visual_attn_mean")
    ap.add_argument("--train", action="store_true",
                    help="time the training step (saving forward + backward) instead of the forward")
    ap.add_argument("--route", action="store_true",
                    help="time the router and the permute alone (L2 flushed before each call)")
    ap.add_argument("--qkv", action="store_true",
                    help="time the router fused into the Q/K/V projection against GEMM + route")
    ap.add_argument("--sp", action="store_true",
                    help="sequence-parallel forward of one video over the ranks (strong scaling)")
    ap.add_argument("--batch", type=int, default=0,
                    help="time the forward over a batch of this many videos (per-video groups, M=20)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.train:
        return run_train(args)
    if args.batch > 0:
        return run_batch(args)
    if args.sp:
        return run_sp(args)
    if args.qkv:
        return run_qkv(args)
    if args.route:
        return run_route(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
