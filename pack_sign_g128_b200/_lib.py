"""ctypes loader for libw1.so (the C ABI declared in include/w1.h).

The library is built in-tree by ``pack_sign_g128_b200.build``.  There is no
fallback: if the shared object is missing or does not load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw1.so")

W1_STATUS = {
    0: "W1_OK", 1: "W1_ERR_NULL", 2: "W1_ERR_SHAPE", 3: "W1_ERR_ALIGN", 4: "W1_ERR_NONFINITE",
    5: "W1_ERR_RANGE", 6: "W1_ERR_CUDA", 7: "W1_ERR_TIMEOUT", 8: "W1_ERR_WORKSPACE",
    9: "W1_ERR_UNSUPPORTED", 10: "W1_ERR_TOO_LARGE", 11: "W1_ERR_NOT_CONVERGED",
}
W1_OK, W1_ERR_NULL, W1_ERR_SHAPE, W1_ERR_ALIGN, W1_ERR_NONFINITE = 0, 1, 2, 3, 4
W1_ERR_RANGE, W1_ERR_CUDA, W1_ERR_TIMEOUT, W1_ERR_WORKSPACE, W1_ERR_UNSUPPORTED = 5, 6, 7, 8, 9
W1_ERR_TOO_LARGE = 10
W1_ERR_NOT_CONVERGED = 11

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_sz = ctypes.c_size_t

# name -> (restype, argtypes); must match include/w1.h
SIGNATURES = {
    "w1_status_string": (ctypes.c_char_p, [_int]),
    "w1_sync_status": (_int, [_p]),
    "w1_set_knob": (_int, [ctypes.c_char_p, ctypes.c_char_p]),
    "w1_pack": (_int, [_p, _i64, _i64, _p, _p, _p]),
    "w1_gemv": (_int, [_p, _p, _i64, _i64, _p, _i64, _p, _p]),
    "w1_gemv_ex": (_int, [_p, _p, _i64, _i64, _p, _i64, _p, ctypes.c_uint32, _p]),
    "w1_gemv_choice": (_int, [_i64, _i64, _i64, ctypes.c_uint32, ctypes.c_char_p, _sz]),
    "w1_gemv_set_choice": (_int, [_i64, _i64, _i64, ctypes.c_uint32, ctypes.c_char_p]),
    "w1_gemm": (_int, [_p, _p, _i64, _i64, _p, _i64, _p, _p, _sz, _p]),
    "w1_gemm_workspace_size": (_sz, [_i64, _i64]),
    "w1_moe_grouped": (_int, [_p, _p, _i64, _i64, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "w1_moe_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64]),
    "dbf_apply": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _i64, _p, _p, _sz, _p]),
    "dbf_workspace_size": (_sz, [_i64, _i64, _i64, _i64]),
    "dbf_apply_noalloc": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _i64, _p, _p]),
    "w1_okt_rotate": (_int, [_p, _i64, _p, _i64, _p, _i64, _p, _p]),
    "w1_measure_workspace_size": (_sz, [_i64, _i64]),
    "w1_residual": (_int, [_p, _i64, _i64, _p, _p, _p, _p, _p, _sz, _p]),
    "dbf_residual": (_int, [_p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _sz, _p]),
    "dbf_residual_workspace_size": (_sz, [_i64, _i64, _i64]),
    "w1_power_iteration": (_int, [_p, _i64, _i64, _p, _i64, _p, _p, _sz, _p]),
    "w1_stream_probe": (_int, [_p, _i64, _p, _i64, _i64, ctypes.c_uint32, _p, _p]),
    "dbf_reproject_mid_workspace_size": (_sz, [_i64, _i64, _i64]),
    "dbf_reproject_mid": (_int, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_double, _p, _p, _p, _p, _sz,
                                 _p]),
    "w1_okt_gemv": (_int, [_p, _p, _i64, _i64, _p, _i64, _p, _i64, _p, _i64, _p, _p, ctypes.c_uint32, _p]),
}

_lib = None


class W1Error(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {W1_STATUS.get(status, status)}")


def load() -> ctypes.CDLL:
    """Load libw1.so (once).  Raises if it is missing -- there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libw1.so not built ({LIB_PATH}); run python -m pack_sign_g128_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


_fns: dict = {}


def fn(name: str):
    """The ctypes function for `name` (looked up once)."""
    f = _fns.get(name)
    if f is None:
        f = getattr(load(), name)
        _fns[name] = f
    return f


def call(name: str, *args) -> int:
    return fn(name)(*args)


def check(status: int, where: str) -> None:
    if status != W1_OK:
        raise W1Error(status, where)
