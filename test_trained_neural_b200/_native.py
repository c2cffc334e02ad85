"""ctypes declarations of libtitansmem's C ABI (include/titansmem.h).

Argument marshalling only: every step of the memory's write-and-read runs in
the library's CUDA kernels. Importing this module without the built library
raises at once; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtitansmem.so")

TM_OK, TM_ERR_INVALID_ARG, TM_ERR_UNSUPPORTED, TM_ERR_CUDA, TM_ERR_OOM, TM_ERR_TIMEOUT, \
    TM_ERR_DEVICE = range(7)
TM_ACT_SILU = 0
TM_F32, TM_BF16 = 0, 1
TM_PATH_AUTO, TM_PATH_SIMT, TM_PATH_TC, TM_PATH_TC_LAYERED, TM_PATH_TC_PHASED, TM_PATH_TC_GLOBAL = 0, 1, 2, 3, 4, 5

# name -> (restype, argtypes); mirrors include/titansmem.h
_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "tm_create": (_I, [_I, _I, _I, _I, ctypes.POINTER(_P)]),
    "tm_destroy": (_I, [_P]),
    "tm_param_count": (_SZ, [_P]),
    "tm_set_path": (_I, [_P, _I]),
    "tm_query_path": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
    "tm_launch_count": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_longlong)]),
    "tm_workspace_size": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "tm_run": (_I, [_P, _I, _I, _I, _I, _I] + [_P] * 11 + [_P, _SZ, _P]),
    "tm_run_noalloc": (_I, [_P, _I, _I, _I, _I, _I] + [_P] * 11 + [_P]),
    "tm_host_workspace_size": (_I, [_P, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)]),
    "tm_run_host": (_I, [_P, _I, _I, _I, _I, _I] + [_P] * 11 + [_I, _P, _SZ, _P]),
    "tm_sync": (_I, [_P, _P, _P]),
    "tm_set_debug": (_I, [_I, ctypes.c_ulonglong]),
    "tm_prologue": (_I, [_I, _I, _I, _I, _I, _I] + [_P] * 12 + [_P]),
    "tm_decode_step": (_I, [_P, _I, _I, _I] + [_P] * 9 + [_P]),
    "tm_backward_workspace_size": (_I, [_P, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "tm_backward": (_I, [_P, _I, _I, _I, _I, _I] + [_P] * 20 + [ctypes.c_size_t, _P]),
    "tm_status_string": (ctypes.c_char_p, [_I]),
    "tm_version": (_I, []),
}

_lib = None


class TitansMemError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtitansmem.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().tm_status_string(int(code)).decode()


def check(code: int, where: str) -> None:
    if code != TM_OK:
        raise TitansMemError(code, where)
