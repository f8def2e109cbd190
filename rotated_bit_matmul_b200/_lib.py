"""ctypes binding of libharp.so: the C ABI declared in include/harp.h, same names.

Only argument marshalling happens here (tensors -> device pointers, the current
CUDA stream, dtype codes); every step of the computation runs in the library's
sm_100a kernels. A missing or stale library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libharp.so")

HARP_OK, HARP_ERR_INVALID_ARG, HARP_ERR_UNSUPPORTED, HARP_ERR_CUDA, HARP_ERR_WORKSPACE, HARP_ERR_TIMEOUT, \
    HARP_ERR_DEVICE_CHECK = range(7)
HARP_F32, HARP_BF16, HARP_F16 = 0, 1, 2

STATUS_NAMES = {0: "HARP_OK", 1: "HARP_ERR_INVALID_ARG", 2: "HARP_ERR_UNSUPPORTED", 3: "HARP_ERR_CUDA",
                4: "HARP_ERR_WORKSPACE", 5: "HARP_ERR_TIMEOUT", 6: "HARP_ERR_DEVICE_CHECK"}

# name -> (restype, argtypes); mirrors include/harp.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "harp_last_error": (ctypes.c_char_p, []),
    "harp_device_status": (_I, [_P]),
    "harp_test_set_faults": (_I, [_I, _I, _I]),
    "harp_butterfly_fwd": (_I, [_I64, _I, _I, _P, _P, _P, _I, _P, _I, _P]),
    "harp_butterfly_inv": (_I, [_I64, _I, _I, _P, _P, _P, _I, _P, _I, _P]),
    "harp_quantize_weights": (_I, [_I64, _I64, _I, _I, _P, _P, _P, _P]),
    "harp_create_layer": (_I, [ctypes.POINTER(_P), _I64, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "harp_destroy_layer": (_I, [_P]),
    "harp_linear_workspace_size": (_I, [_P, _I, ctypes.POINTER(_SZ)]),
    "harp_linear_fwd": (_I, [_P, _I, _P, _I, _P, _I, _P, _SZ, _P]),
    "harp_linear_fwd_static": (_I, [_P, _I, _P, _I, _P, _I, _P]),
    "harp_stack_create": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, ctypes.c_float, ctypes.POINTER(_P), _P]),
    "harp_stack_destroy": (_I, [_P]),
    "harp_stack_workspace_size": (_I, [_P, _I, ctypes.POINTER(_SZ)]),
    "harp_stack_step": (_I, [_P, _I, _P, _I, _P, _I, _P, _SZ, _P]),
    "harp_stack_uses_fused_step": (_I, [_P, _I]),
    "harp_mr_plan_create": (_I, [ctypes.POINTER(_P), _I64, _I, ctypes.POINTER(ctypes.c_int), _P, _P, _P, _P]),
    "harp_mr_plan_destroy": (_I, [_P]),
    "harp_mr_butterfly_fwd": (_I, [_P, _I, _P, _I, _P, _I, _P]),
    "harp_mr_butterfly_inv": (_I, [_P, _I, _P, _I, _P, _I, _P]),
    "harp_quantize_angles": (_I, [_I, _I64, _P, _P, _P, _P]),
    "harp_create_layer_mr": (_I, [ctypes.POINTER(_P), _I64, _I64, _I, _I, _P, _P, _P, _P, _P]),
    "harp_create_layer_q8": (_I, [ctypes.POINTER(_P), _I64, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                  _P]),
    "harp_calib_workspace_size": (_I, [_I64, _I64, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "harp_calib_fit": (_I, [_I64, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, ctypes.c_double, _P, _P, _P, _P,
                            _SZ, _P]),
}


class HarpError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libharp.so (raises if it is missing or lacks a declared symbol)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m rotated_bit_matmul_b200.build_lib` "
                          "(the rotated low-bit kernels have no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != HARP_OK:
        msg = load().harp_last_error()
        raise HarpError(status, where, msg.decode() if msg else "")


def call(name: str, *args) -> None:
    """Calls the C entry point `name` and raises HarpError on a non-OK status."""
    check(getattr(load(), name)(*args), name)
