"""ctypes loader for libmoe_fp8.so, the C ABI declared in include/moe_fp8.h.

The shared library is built in-tree (``python -m fine_grained_fp8_sigmoid_b200.build``
or ``__graft_entry__.build()``). There is no fallback: if the library is
missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_fp8.so")

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_z = ctypes.c_size_t

# name -> (restype, argtypes), in the order of include/moe_fp8.h
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_version": (_i, []),
    "moe_last_error_detail": (ctypes.c_char_p, []),
    "moe_get_error": (_i, [ctypes.POINTER(_i)]),
    "moe_quant_1x128": (_i, [_p, _i, _i, _p, _p, _p]),
    "moe_quant_128x128": (_i, [_p, _i, _i, _p, _p, _p]),
    "moe_route": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _p]),
    "moe_route_quant": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p]),
    "moe_permute_workspace": (_z, [_i, _i]),
    "moe_permute": (_i, [_p, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p, _p, _z, _p]),
    "moe_permute_noalloc": (_i, [_p, _i, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p, _p]),
    "moe_grouped_gemm_fp8_workspace": (_z, [_i, _i, _i, _i]),
    "moe_grouped_gemm_fp8_launches": (_i, [_i, _i]),
    "moe_grouped_gemm_fp8": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p,
                                  _i, _i, _p, _p, _p, _z, _p]),
    "moe_grouped_gemm_fp8_gather": (_i, [_p, _p, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p,
                                         _i, _i, _p, _p, _p, _z, _p]),
    "moe_grouped_gemm_fp8_rows_workspace": (_z, [_i, _i, _i, _i]),
    "moe_grouped_gemm_fp8_rows": (_i, [_p, _p, _p, _i, _i, _p, _p, _i, _p, _p, _p, _p, _p, _p,
                                       _i, _i, _p, _p, _p, _z, _p]),
    "moe_group_of_rows": (_i, [_p, _i, _i, _i, _p, _p]),
    "moe_gather_rows": (_i, [_p, _i, _p, _i, _i, _p, _p]),
    "moe_grouped_scaled_gemm_fp8_workspace": (_z, []),
    "moe_grouped_scaled_gemm_fp8": (_i, [_p, _p, _p, _i, _i, _i, _p, _p, _i, _i, _p, _p, _z, _p]),
    "moe_kgrouped_gemm_fp8_workspace": (_z, []),
    "moe_kgrouped_gemm_fp8": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _p, _z, _p]),
    "moe_swiglu_backward_quant": (_i, [_p, _p, _p, _i, _i, _p, _p, _p, _p]),
    "moe_quant_1x128_t": (_i, [_p, _i, _i, _i, _p, _p, _i, _i, _p, _p, _p]),
    "moe_quant_128x128_t": (_i, [_p, _p, _i, _i, _p, _p, _i, _i, _p, _p, _p]),
    "moe_transpose": (_i, [_p, _i, _i, _i, _i, _p, _i, _i, _p]),
    "moe_combine": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "moe_combine_fp32": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "moe_bias_update": (_i, [_p, _p, _i, _i, _i, _f, _p, _p]),
    "moe_debug_wait_timeout": (_i, [_i, _p]),
}

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_TIMEOUT = 4
MOE_ERR_NO_DEVICE = 5

_lock = threading.Lock()
_lib = None


class MoEError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        detail = load().moe_last_error_detail().decode(errors="replace")
        super().__init__(f"{call} failed: {status_string(status)} ({status}) [{detail}]")


def load() -> ctypes.CDLL:
    """Loads the library once; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m fine_grained_fp8_sigmoid_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def check(call: str, status: int) -> None:
    if status != MOE_OK:
        raise MoEError(call, status)
