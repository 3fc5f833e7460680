"""Builds libmoga.so (sm_100a) in-tree with nvcc.

Usage: python -m sparse_attention_long_moga_b200.build
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoga.so")
# the checking build: device-side index checks (-DMOGA_DEBUG), same ABI
DEBUG_LIB = os.path.join(PKG, "libmoga_debug.so")
SOURCES = ["moga_lib.cu"]
DEPS = ["tc_common.cuh", "route_tc.cu", "route_bwd.cu", "sp.cu", "qkv_route.cu", "attention_bwd.cu", "api_common.cu", "route.cu", "permute.cu", "permute_noalloc.cu", "mean_loss.cu", "attention.cu", "common.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False) -> list:
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(os.path.dirname(PKG), "include")]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    hdr = os.path.join(os.path.dirname(PKG), "include", "moga.h")
    srcs = [os.path.join(CSRC, s) for s in SOURCES + DEPS] + [hdr]
    return any(os.path.getmtime(s) > t for s in srcs if os.path.exists(s))


# The attention kernel launches at this many registers per thread and then
# splits them between its warpgroups with setmaxnreg (csrc/attention.cu:
# kLaunchRegs).  A different launch count would make the split unbalanced,
# so the build refuses to produce such a library.
ATTN_LAUNCH_REGS = 168


def check_register_split(ptxas_log: str) -> None:
    lines = ptxas_log.splitlines()
    found = 0
    for i, line in enumerate(lines):
        if "Compiling entry function" in line and "attn_kernel" in line:
            for nxt in lines[i + 1:i + 4]:
                m = re.search(r"Used (\d+) registers", nxt)
                if m:
                    found += 1
                    if int(m.group(1)) != ATTN_LAUNCH_REGS:
                        raise RuntimeError("attention kernel compiled to %s registers per thread, expected %d "
                                           "(the setmaxnreg split would not balance)" % (m.group(1), ATTN_LAUNCH_REGS))
                    break
    if found == 0:
        raise RuntimeError("could not find the attention kernel's register count in the ptxas report")


def _compile(lib: str, extra: list, verbose: bool) -> None:
    tmp = lib + ".tmp"
    cmd = [nvcc()] + flags(True) + extra + ["-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise subprocess.CalledProcessError(res.returncode, cmd, res.stdout, res.stderr)
    check_register_split(res.stdout + res.stderr)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds libmoga.so and (debug=True) the checking build libmoga_debug.so,
    each only when a source is newer (or force); returns the default library."""
    if force or stale(LIB):
        _compile(LIB, [], verbose)
    if debug and (force or stale(DEBUG_LIB)):
        _compile(DEBUG_LIB, ["-DMOGA_DEBUG"], verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
