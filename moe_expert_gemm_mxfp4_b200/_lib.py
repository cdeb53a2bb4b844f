"""ctypes binding of ``libmxfp4.so`` (the C ABI declared in ``include/mxfp4.h``).

Argument marshalling only: every step of every entry point runs in the CUDA
library.  torch tensors supply device memory and the current CUDA stream.
The library is loaded on first use; a missing or unloadable library raises
``Mxfp4LibraryMissing`` -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmxfp4.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "mxfp4.h")

# mxfp4_status values (include/mxfp4.h)
OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_MISALIGNED = 3
ERR_ARCH = 4
ERR_WORKSPACE = 5
ERR_CUDA = 6
ERR_TIMEOUT = 7

IN_BF16, IN_F32 = 0, 1
NOALLOC_SCRATCH_BYTES = 16 << 20   # MXFP4_NOALLOC_SCRATCH_BYTES in include/mxfp4.h
SCALE_FLOOR, SCALE_CEIL = 0, 1
W4A16, W4A4 = 0, 1


class Mxfp4LibraryMissing(RuntimeError):
    pass


class Mxfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int):
        self.status = status
        self.cuda_error = cuda_error
        name = _LIB.mxfp4_status_string(status).decode() if _LIB else str(status)
        super().__init__(f"{fn} failed: {name} (status {status}, cudaError {cuda_error})")


_LIB = None

_i64, _i32, _sz, _vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "mxfp4_quantize": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _vp, _vp, ctypes.c_int, _vp]),
    "mxfp4_dequantize": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp]),
    "mxfp4_gemm": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, ctypes.c_int, _vp, _sz, _vp]),
    "mxfp4_gemm_workspace_size": (_sz, [_i64, _i64, _i64, ctypes.c_int]),
    "mxfp4_token_tile_rows": (_i32, [_i64, _i64, ctypes.c_int]),
    "moe_mxfp4_route": (ctypes.c_int, [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_mxfp4_route_workspace_size": (_sz, [_i64, _i64, _i32]),
    "moe_mxfp4_route_project": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _sz, _vp]),
    "moe_mxfp4_mlp": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _vp, _i64, _vp, _vp, _vp,
                                     ctypes.c_int, _vp, _sz, _vp]),
    "moe_mxfp4_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32, ctypes.c_int]),
    "moe_mxfp4_mlp_noalloc": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _vp, _i64, _vp, _vp, _vp,
                                             ctypes.c_int, _vp]),
    "mxfp4_gather_rows": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _vp]),
    "moe_mxfp4_experts": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp,
                                         ctypes.c_int, _vp, _sz, _vp]),
    "moe_mxfp4_experts_workspace_size": (_sz, [_i64, _i64, _i64, _i64, ctypes.c_int]),
    "moe_mxfp4_combine": (ctypes.c_int, [_vp, _vp, _i64, _i32, _i64, _vp, _vp]),
    "moe_bf16_mlp": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _i64, _vp, _vp, _vp, _sz, _vp]),
    "moe_bf16_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i32]),
    "mxfp4_get_device_status": (ctypes.c_int, [_vp]),
    "mxfp4_selftest_wait_timeout": (ctypes.c_int, [_vp]),
    "mxfp4_selftest_mma_rate": (ctypes.c_int, [_i32, _i32, ctypes.POINTER(ctypes.c_double), _vp]),
    "mxfp4_set_trace_events": (None, [_vp, ctypes.c_int]),
    "mxfp4_last_cuda_error": (ctypes.c_int, []),
    "mxfp4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}


def header_symbols(path: str = HEADER) -> list[str]:
    """Names of the functions the public header declares (MXFP4_API prefix)."""
    with open(path) as f:
        text = f.read()
    return re.findall(r"MXFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def load(path: str = LIB_PATH):
    """Load the library (once).  Raises Mxfp4LibraryMissing if it is absent."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise Mxfp4LibraryMissing(
            f"{path} not found: build it with `python -m moe_expert_gemm_mxfp4_b200.build`")
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:
        raise Mxfp4LibraryMissing(f"cannot load {path}: {e}") from e
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def check(fn_name: str, status: int):
    if status != OK:
        raise Mxfp4Error(fn_name, status, _LIB.mxfp4_last_cuda_error())
