"""ctypes binding of libwq.so: the same entry points as include/wq.h.

Argument marshalling only.  Tensors are passed as raw device pointers
(``tensor.data_ptr()``); every computation happens in the library's CUDA
kernels.  There is no fallback: if libwq.so is missing or cannot be loaded,
importing a symbol raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwq.so")

WQ_OK = 0
WQ_ERR_ARG = -1
WQ_ERR_ALIGN = -2
WQ_ERR_LAYOUT = -3
WQ_ERR_CUDA = -4
WQ_ERR_DEVICE = -5
WQ_ERR_TIMEOUT = -6
WQ_ERR_UNSUPPORTED = -7
WQ_LAYOUT_CANONICAL = 0
WQ_LAYOUT_B200_V1 = 1

_ERRNAMES = {v: k for k, v in dict(globals()).items() if k.startswith("WQ_ERR_")}

# name -> (restype, argtypes); mirrors include/wq.h
_vp, _i, _sz, _cp = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_char_p
SIGNATURES = {
    "gemv_int4_blockwise": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "gemv_q4k": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "gemv_q4k_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "gemv_q4k_dsc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "gemv_bf16": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "gemv_mxfp4": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "gemv_int4_swiglu": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "wq_repack_int4_gate_up": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "wq_int4_gate_up_packed_bytes": (_sz, [_i, _i, _i, _i]),
    "dequant_int4_blockwise": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "dequant_q4k": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "dequant_mxfp4": (_i, [_vp, _vp, _vp, _i, _i, _vp]),
    "quantize_q8": (_i, [_vp, _vp, _vp, _i, _i, _vp]),
    "wq_tp_rows": (_i, [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "gemv_int4_tp": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_void_p), _i, _i, _i, _i, _i, _i, _i, _vp]),
    "wq_ipc_handle": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_ulonglong)]),
    "wq_ipc_open": (_i, [_vp, ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_void_p)]),
    "wq_ipc_close": (_i, [_vp, ctypes.c_ulonglong]),
    "gemm_q4k_q8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "wq_q8_bytes": (_sz, [_i, _i]),
    "wq_q8_scale_bytes": (_sz, [_i, _i]),
    "wq_int4_bytes": (_sz, [_i, _i, _i, _i]),
    "wq_int4_codes_bytes": (_sz, [_i, _i, _i]),
    "wq_repack_int4": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "wq_int4_packed_bytes": (_sz, [_i, _i, _i, _i]),
    "wq_q4k_bytes": (_sz, [_i, _i]),
    "wq_q4k_dsc_bytes": (_sz, [_i, _i]),
    "wq_q4k_packed_bytes": (_sz, [_i, _i, _i]),
    "wq_repack_q4k": (_i, [_vp, _vp, _i, _i, _i, _vp]),
    "wq_build_q4k_dsc": (_i, [_vp, _i, _i, _vp]),
    "wq_build_q4k_dsc_device": (_i, [_vp, _vp, _i, _i, _vp]),
    "wq_last_error": (_cp, []),
    "wq_last_kernel": (_cp, []),
    "wq_layout_version": (_i, []),
    "wq_build_info": (_cp, []),
    "wq_device_status": (_i, []),
    "wq_test_expire_wait": (_i, [ctypes.c_ulonglong, _vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libwq.so (once).  Raises if it is absent: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwq.so not built at {LIB_PATH}; run `python -m weight_only_quantized_q4_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class WQError(RuntimeError):
    def __init__(self, code: int, fn: str, msg: str):
        super().__init__(f"{fn} failed: {_ERRNAMES.get(code, code)}: {msg}")
        self.code = code


def last_error() -> str:
    return lib().wq_last_error().decode()


def last_kernel() -> str:
    return lib().wq_last_kernel().decode()


def _check(rc: int, fn: str) -> None:
    if rc != WQ_OK:
        raise WQError(rc, fn, last_error())
