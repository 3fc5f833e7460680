"""ctypes binding of libmoga.so: argument marshalling only.

Every function here checks shapes/dtypes/devices of torch tensors, passes raw
device pointers, sizes and the current CUDA stream to the C ABI declared in
include/moga.h, and raises MogaError on a non-zero status.  All arithmetic
runs in the library's CUDA kernels; there is no CPU fallback.  Importing this
module fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoga.so")
# the checking build (device-side index checks, same ABI); MOGA_DEBUG=1 in
# the environment makes lib() load it instead of the default build
DEBUG_LIB_PATH = os.path.join(PKG, "libmoga_debug.so")

STATUS = {0: "MOGA_OK", 1: "MOGA_ERR_INVALID_ARG", 2: "MOGA_ERR_UNSUPPORTED", 3: "MOGA_ERR_WORKSPACE",
          4: "MOGA_ERR_CUDA", 5: "MOGA_ERR_TIMEOUT", 6: "MOGA_ERR_BAD_INDEX"}
MOGA_F32, MOGA_BF16 = 0, 1

# exported symbol -> (restype, argtypes); the same list include/moga.h declares
_P, _I32, _I64, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "moga_route_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_route": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _I64, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "moga_permute_ws_bytes": (_SZ, [_I64, _I32]),
    "moga_permute": (ctypes.c_int, [_P, _I64, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "moga_permute_noalloc": (ctypes.c_int, [_P, _I64, _I32, _P, _P, _P, _P, _P]),
    "moga_attn_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_group_attn": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _I32, _P, _F32, _P, _P, _SZ, _P]),
    "stga_attn": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _F32, _P, _P, _SZ, _P]),
    "stga_attn_mean": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _F32, _P, _P, _P, _SZ, _P]),
    "visual_attn_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "visual_attn_branches": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _I32, _P, _P, _F32, _P, _P, _SZ,
                                            _P]),
    "visual_attn_mean": (ctypes.c_int, [_P, _I64, _P, _P]),
    "moga_balance_loss": (ctypes.c_int, [_P, _P, _I64, _I32, _F32, _P, _P]),
    "moga_permute_batched_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_permute_batched": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "moga_group_attn_batched": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _I32, _P, _P, _I32, _P, _F32, _P, _P,
                                               _P, _SZ, _P]),
    "stga_attn_batched": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _P, _F32, _P, _P, _SZ, _P]),
    "moga_balance_loss_batched": (ctypes.c_int, [_P, _I32, _P, _I64, _I32, _F32, _P, _P]),
    "moga_sp_pack_heads": (ctypes.c_int, [_P, _I64, _I32, _I32, _I32, _P, _P]),
    "moga_sp_unpack_heads": (ctypes.c_int, [_P, _I64, _I32, _I32, _I32, _P, _P]),
    "moga_balance_loss_part": (ctypes.c_int, [_P, _P, _I64, _I64, _I32, _F32, _P, _P]),
    "moga_qkv_route_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_qkv_route": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ,
                                      _P]),
    "moga_route_train": (ctypes.c_int, [_P, _P, ctypes.c_int, _P, _I64, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    "moga_group_attn_train": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _I32, _P, _F32, _P, _P, _P, _SZ,
                                             _P]),
    "stga_attn_train": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _F32, _P, _P, _P, _P, _P, _SZ, _P]),
    "visual_attn_mean3": (ctypes.c_int, [_P, _P, _P, _I64, _P, _P]),
    "moga_attn_bwd_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_group_attn_bwd": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _I32, _P, _F32, _P, _P, _P, _P, _P,
                                           _P, _P, _P, _SZ, _P]),
    "stga_attn_bwd": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _F32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moga_route_bwd_ws_bytes": (_SZ, [_I64, _I32, _I32]),
    "moga_route_bwd": (ctypes.c_int, [_P, _P, ctypes.c_int, _I64, _I32, _I32, _P, _P, _P, _P, _F32, _F32, _P, _P, _P,
                                      _P, _SZ, _P]),
    "moga_last_error": (ctypes.c_char_p, []),
    "moga_device_status": (ctypes.c_int, [_P]),
    "moga_version": (ctypes.c_char_p, []),
}


class MogaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), msg))
        self.status = status


class StgaGeom(ctypes.Structure):
    _fields_ = [("T", _I32), ("h", _I32), ("w", _I32), ("win_h", _I32), ("win_w", _I32),
                ("n_shots", _I32), ("shot_len", ctypes.POINTER(_I32)), ("tg_max", _I32),
                ("aug_frames", _I32)]


def load(path: str | None = None) -> ctypes.CDLL:
    if path is None:
        path = DEBUG_LIB_PATH if os.environ.get("MOGA_DEBUG", "") not in ("", "0") else LIB_PATH
    if not os.path.exists(path):
        raise ImportError("%s is not built (run sparse_attention_long_moga_b200.build); "
                          "there is no fallback path" % os.path.basename(path))
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise MogaError(status, where, lib().moga_last_error().decode())
