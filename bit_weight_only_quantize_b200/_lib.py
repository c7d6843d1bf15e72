"""ctypes binding of the C ABI in include/q4.h (argument marshalling only).

Every function here forwards raw pointers, sizes and the current CUDA stream to
``libq4b200.so``; all arithmetic happens in the library's kernels.  There is no
fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libq4b200.so")

Q4_OK = 0
STATUS_NAMES = {
    0: "Q4_OK", 1: "Q4_ERR_INVALID_ARG", 2: "Q4_ERR_SHAPE", 3: "Q4_ERR_ALIGN", 4: "Q4_ERR_DTYPE",
    5: "Q4_ERR_WORKSPACE", 6: "Q4_ERR_CUDA", 7: "Q4_ERR_UNSUPPORTED_DEVICE",
}
Q4_F32 = 0
Q4_BF16 = 1
FLAG_NONFINITE = 1
FLAG_SCALE_OVERFLOW = 2
GEMV_MAX_M = 16
MULTI_MAX = 4
WEIGHTS_STATIC = 1


class Weight(ctypes.Structure):
    """struct q4_weight of include/q4.h."""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("y", ctypes.c_void_p)]


class MixedWeight(ctypes.Structure):
    """struct q4_mixed_weight of include/q4.h."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("y", ctypes.c_void_p), ("bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]

# Every symbol include/q4.h declares, with (restype, argtypes).
_i64, _vp, _sz, _i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "q4_abi_version": (_i32, []),
    "q4_status_string": (ctypes.c_char_p, [_i32]),
    "q4_device_error": (_i32, [_vp, _i32]),
    "q4_set_consumer_wait_limit": (ctypes.c_uint64, [ctypes.c_uint64]),
    "q4_quantize": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "q4_gemv_workspace_size": (_sz, [_i64, _i64, _i64]),
    "q4_gemv": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "q4_gemv_noalloc": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp]),
    "q4_gemv_host": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, ctypes.c_uint32, _vp, _sz, _vp]),
    "q4_gemm": (_i32, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp]),
    "q4_gemv_multi_workspace_size": (_sz, [_i64, _i64, _vp, _i32]),
    "q4_gemv_multi": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, ctypes.c_uint32, _vp, _sz, _vp]),
    "q4_gemv_gate_up": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, ctypes.c_uint32, _vp]),
    "q4_f16_gemv": (_i32, [_vp, _i32, _i64, _i64, _vp, _i64, _vp, ctypes.c_uint32, _vp]),
    "q4_gemv_argmax_workspace_size": (_sz, []),
    "q4_gemv_argmax": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, ctypes.c_uint32, _vp, _sz,
                              _vp]),
    "q4_int8_quantize": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "q4_int8_gemv": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _vp, _vp]),
    "q4_gemv_mixed_workspace_size": (_sz, [_i64, _i64, _vp, _i32]),
    "q4_gemv_mixed": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, ctypes.c_uint32, _vp, _sz, _vp]),
    "q4_topk_merge": (_i32, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "q4_gemv_topk_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32]),
    "q4_gemv_topk": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, ctypes.c_uint32,
                            _vp, _sz, _vp]),
}


class Q4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load libq4b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"CUDA library {LIB_PATH} is missing; build it with "
                    "`python -m bit_weight_only_quantize_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def status_string(status: int) -> str:
    try:
        return load().q4_status_string(status).decode()
    except Exception:
        return STATUS_NAMES.get(status, f"status {status}")


def device_error(clear: bool = True) -> int:
    """The library's device error word for the current device (see q4_device_error)."""
    out = ctypes.c_uint32(0)
    check(load().q4_device_error(ctypes.byref(out), 1 if clear else 0), "q4_device_error")
    return int(out.value)


def check(status: int, where: str) -> None:
    if status != Q4_OK:
        raise Q4Error(status, where)
