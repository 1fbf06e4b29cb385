"""ctypes binding of libmxattn.so (the C ABI of include/mxattn.h), argument marshalling only.

The raw entry points keep their C names (``mxattn_quantize``, ``mxattn_forward`` ...). Loading
fails loudly when the library has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libmxattn.so")

_c_int, _c_i64, _c_size, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
_u8p = ctypes.c_void_p

# name -> (restype, argtypes), mirroring include/mxattn.h
SIGNATURES = {
    "mxattn_quantize": (_c_int, [_vp, _c_i64, _c_i64, _c_i64, _c_int, _c_int, _u8p, _u8p, _vp]),
    "mxattn_forward_workspace_size": (_c_size, [_c_int] * 5),
    "mxattn_forward": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 9 + [_vp, _c_size, _vp]),
    "mxattn_forward_prepare": (_c_int, [_vp, _vp, _vp] + [_c_int] * 6 + [_vp, _c_size, _vp]),
    "mxattn_forward_attend": (_c_int, [_vp] + [_c_int] * 9 + [_vp, _c_size, _vp]),
    "mxattn_forward_debug": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 9 + [_vp, _c_size, _vp]
                             + [_c_int] * 3 + [_u8p, _u8p]),
    "mxattn_forward_noalloc": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 9 + [_vp]),
    "mxattn_forward_host_workspace_size": (_c_size, [_c_int] * 6),
    "mxattn_forward_host": (_c_int, [_vp, _vp, _vp, _vp] + [_c_int] * 9 + [_vp, _c_size, _vp]),
    "mxattn_forward_quantized": (_c_int, [_u8p] * 6 + [_vp] + [_c_int] * 9 + [_vp, _c_size, _vp]),
    "mxattn_gemm_workspace_size": (_c_size, [_c_i64] * 3),
    "mxattn_gemm": (_c_int, [_u8p] * 4 + [_vp] + [_c_i64] * 3 + [_c_int, _vp, _c_size, _vp]),
    "mxattn_selftest_wait_timeout": (_c_int, [_vp, _vp]),
    "mxattn_quantize_nvfp4": (_c_int, [_vp, _c_i64, _c_i64, _u8p, _u8p, _vp]),
    "mxattn_gemm_nvfp4_workspace_size": (_c_size, [_c_i64] * 3),
    "mxattn_gemm_nvfp4": (_c_int, [_u8p] * 4 + [_vp] + [_c_i64] * 3 + [_c_int, _vp, _c_size, _vp]),
    "mxattn_check_status": (_c_int, [_vp, _vp, ctypes.POINTER(ctypes.c_uint)]),
    "mxattn_check_status_noalloc": (_c_int, [_vp, ctypes.POINTER(ctypes.c_uint)]),
    "mxattn_status_string": (ctypes.c_char_p, [_c_int]),
    "mxattn_version": (_c_int, []),
}

STATUS = {0: "MXATTN_OK", 1: "MXATTN_ERR_INVALID_ARG", 2: "MXATTN_ERR_UNSUPPORTED",
          3: "MXATTN_ERR_WORKSPACE", 4: "MXATTN_ERR_CUDA", 5: "MXATTN_ERR_TIMEOUT"}


class MxattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmxattn.so once and attach the C signatures. Raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"libmxattn.so not built at {path}; run "
                           "`python -m mxfp4_microscaled_bit_quantize_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def check(status: int, where: str) -> None:
    if status != 0:
        raise MxattnError(status, where)
