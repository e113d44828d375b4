"""ctypes binding of libhalo.so (argument marshalling only).

Every entry point of ``include/halo.h`` is declared here with the same name.
Loading fails loudly when the library has not been built: there is no other
implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhalo.so")

HALO_F32 = 0
HALO_BF16 = 1

HALO_OK = 0
HALO_ERR_NULL = -1
HALO_ERR_DIMS = -2
HALO_ERR_DIVISIBILITY = -3
HALO_ERR_STRIDE = -4
HALO_ERR_ALIGN = -5
HALO_ERR_UNSUPPORTED = -6
HALO_ERR_CUDA = -7
HALO_ERR_TIMEOUT = -8
HALO_ERR_DTYPE = -9
HALO_ERR_ALIAS = -10
HALO_ERR_DEVICE = -11
HALO_ERR_KERNEL = -12
HALO_ERR_WORKSPACE = -13
HALO_ERR_SCRATCH_LIMIT = -14

HALO_KERNEL_NONE = 0
HALO_KERNEL_SIMT_F32 = 1
HALO_KERNEL_TC_BF16 = 2

_vp = ctypes.c_void_p
_i = ctypes.c_int

# name -> (restype, argtypes); mirrors include/halo.h
SIGNATURES = {
    "halo_attn": (_i, [_vp] * 6 + [_i] * 9 + [_vp]),
    "halo_attn_host": (_i, [_vp] * 12 + [_i] * 9 + [_vp]),
    "halo_attn_masked": (_i, [_vp] * 6 + [_i] * 10 + [_vp]),
    "halo_attn_fused": (_i, [_vp] * 6 + [_i] * 10 + [_vp]),
    "halo_attn_bwd": (_i, [_vp] * 13 + [ctypes.c_size_t] + [_i] * 10 + [_vp]),
    "halo_attn_bwd_workspace_size": (_i, [_i] * 10 + [ctypes.POINTER(ctypes.c_size_t)]),
    "halo_attn_bwd_noalloc": (_i, [_vp] * 12 + [_i] * 10 + [_vp]),
    "halo_kernel_for": (_i, [_i] * 9),
    "halo_kernel_name": (ctypes.c_char_p, [_i] * 9),
    "halo_masked_kernel_name": (ctypes.c_char_p, [_i] * 10),
    "halo_fused_kernel_name": (ctypes.c_char_p, [_i] * 10),
    "halo_bwd_kernel_name": (ctypes.c_char_p, [_i] * 10),
    "halo_strerror": (ctypes.c_char_p, [_i]),
    "halo_get_last_error": (_i, []),
    "halo_debug_wait_timeout": (_i, [_i, _vp]),
    "halo_version": (_i, []),
}

_lib = None


class HaloError(RuntimeError):
    def __init__(self, code: int, where: str = "halo_attn"):
        self.code = code
        super().__init__(f"{where} failed: {code} ({strerror(code)})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m blocked_local_self_b200.build` "
                "(nvcc, sm_100a); this package has no non-CUDA implementation")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def strerror(code: int) -> str:
    return lib().halo_strerror(int(code)).decode()
