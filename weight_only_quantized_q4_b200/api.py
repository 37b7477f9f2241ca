"""Python face of the C ABI: the same names, tensors in, status checked.

Each function takes torch CUDA tensors (or raw integer device pointers),
passes their addresses and sizes to libwq.so on the current torch stream (or
an explicit ``stream``), and raises WQError on a negative status.  Nothing
here touches the data.
"""
from __future__ import annotations

import ctypes

import numpy as np

from ._lib import (WQ_ERR_ARG, WQ_ERR_TIMEOUT, WQ_ERR_UNSUPPORTED, WQ_LAYOUT_B200_V1, WQ_LAYOUT_CANONICAL, WQError,  # noqa: F401
                   _check, last_error, last_kernel, lib)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def gemv_int4_blockwise(x, w_packed, scales, zeros, y, M, N, K, block_size, layout=WQ_LAYOUT_CANONICAL,
                        stream=None):
    _check(lib().gemv_int4_blockwise(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(zeros), _ptr(y), M, N, K,
                                     block_size, layout, _stream(stream)), "gemv_int4_blockwise")


def gemv_q4k(x, w_q4k, y, M, N, K, layout=WQ_LAYOUT_CANONICAL, stream=None):
    _check(lib().gemv_q4k(_ptr(x), _ptr(w_q4k), _ptr(y), M, N, K, layout, _stream(stream)), "gemv_q4k")


def gemv_q4k_noalloc(x, w_q4k, y, M, N, K, layout=WQ_LAYOUT_B200_V1, stream=None):
    """gemv_q4k over the B200_V1 stream that never allocates device memory.

    For callers that own all device memory (their own pool, a fixed budget) or
    must not let a library call block the device the way cudaMalloc can.  Its
    scratch is one fixed array in the library's device memory (about 272 KB
    per GPU, held until exit) shared by every call: calls that overlap on the
    GPU race.  The first call on a device looks up that array's address, so
    make it before any stream capture.  N is limited to 65536 rows."""
    _check(lib().gemv_q4k_noalloc(_ptr(x), _ptr(w_q4k), _ptr(y), M, N, K, layout, _stream(stream)), "gemv_q4k_noalloc")


def gemv_q4k_dsc(x, w_q4k, w_dsc, y, M, N, K, layout=WQ_LAYOUT_CANONICAL, stream=None):
    _check(lib().gemv_q4k_dsc(_ptr(x), _ptr(w_q4k), _ptr(w_dsc), _ptr(y), M, N, K, layout, _stream(stream)),
           "gemv_q4k_dsc")


def gemv_bf16(x, w, y, M, N, K, stream=None):
    _check(lib().gemv_bf16(_ptr(x), _ptr(w), _ptr(y), M, N, K, _stream(stream)), "gemv_bf16")


def gemv_int4_swiglu(x, w_gate_up, y, M, N, K, block_size, layout=WQ_LAYOUT_B200_V1, stream=None):
    _check(lib().gemv_int4_swiglu(_ptr(x), _ptr(w_gate_up), _ptr(y), M, N, K, block_size, layout, _stream(stream)),
           "gemv_int4_swiglu")


def wq_int4_gate_up_packed_bytes(N, K, block_size, layout=WQ_LAYOUT_B200_V1) -> int:
    return int(lib().wq_int4_gate_up_packed_bytes(N, K, block_size, layout))


def wq_repack_int4_gate_up(w_gate, scales_gate, zeros_gate, w_up, scales_up, zeros_up, w_out, N, K, block_size,
                           to_layout=WQ_LAYOUT_B200_V1, stream=None):
    _check(lib().wq_repack_int4_gate_up(_ptr(w_gate), _ptr(scales_gate), _ptr(zeros_gate), _ptr(w_up),
                                        _ptr(scales_up), _ptr(zeros_up), _ptr(w_out), N, K, block_size, to_layout,
                                        _stream(stream)), "wq_repack_int4_gate_up")


def dequant_int4_blockwise(w_packed, scales, zeros, w_out, N, K, block_size, layout=WQ_LAYOUT_CANONICAL,
                           stream=None):
    _check(lib().dequant_int4_blockwise(_ptr(w_packed), _ptr(scales), _ptr(zeros), _ptr(w_out), N, K, block_size,
                                        layout, _stream(stream)), "dequant_int4_blockwise")


def gemv_mxfp4(x, w_packed, scales, y, M, N, K, stream=None):
    _check(lib().gemv_mxfp4(_ptr(x), _ptr(w_packed), _ptr(scales), _ptr(y), M, N, K, _stream(stream)), "gemv_mxfp4")


def dequant_mxfp4(w_packed, scales, w_out, N, K, stream=None):
    _check(lib().dequant_mxfp4(_ptr(w_packed), _ptr(scales), _ptr(w_out), N, K, _stream(stream)), "dequant_mxfp4")


def quantize_q8(x, qa8, sda, M, K, stream=None):
    _check(lib().quantize_q8(_ptr(x), _ptr(qa8), _ptr(sda), M, K, _stream(stream)), "quantize_q8")


def gemm_q4k_q8(qa8, sda, w_q4k, w_dsc, y, M, N, K, stream=None):
    _check(lib().gemm_q4k_q8(_ptr(qa8), _ptr(sda), _ptr(w_q4k), _ptr(w_dsc), _ptr(y), M, N, K, _stream(stream)),
           "gemm_q4k_q8")


def wq_q8_bytes(M, K) -> int:
    return int(lib().wq_q8_bytes(M, K))


def wq_q8_scale_bytes(M, K) -> int:
    return int(lib().wq_q8_scale_bytes(M, K))


def dequant_q4k(w_q4k, w_dsc, w_out, N, K, layout=WQ_LAYOUT_CANONICAL, stream=None):
    _check(lib().dequant_q4k(_ptr(w_q4k), _ptr(w_dsc), _ptr(w_out), N, K, layout, _stream(stream)), "dequant_q4k")


def wq_int4_bytes(N, K, block_size, layout=WQ_LAYOUT_CANONICAL) -> int:
    return int(lib().wq_int4_bytes(N, K, block_size, layout))


def wq_int4_codes_bytes(N, K, layout=WQ_LAYOUT_CANONICAL) -> int:
    return int(lib().wq_int4_codes_bytes(N, K, layout))


def wq_int4_packed_bytes(N, K, block_size, layout=WQ_LAYOUT_B200_V1) -> int:
    return int(lib().wq_int4_packed_bytes(N, K, block_size, layout))


def wq_repack_int4(w_canonical, scales, zeros, w_out, N, K, block_size, to_layout=WQ_LAYOUT_B200_V1, stream=None):
    _check(lib().wq_repack_int4(_ptr(w_canonical), _ptr(scales), _ptr(zeros), _ptr(w_out), N, K, block_size,
                                to_layout, _stream(stream)), "wq_repack_int4")


def wq_q4k_bytes(N, K) -> int:
    return int(lib().wq_q4k_bytes(N, K))


def wq_q4k_dsc_bytes(N, K) -> int:
    return int(lib().wq_q4k_dsc_bytes(N, K))


def wq_q4k_packed_bytes(N, K, layout=WQ_LAYOUT_B200_V1) -> int:
    return int(lib().wq_q4k_packed_bytes(N, K, layout))


def wq_repack_q4k(w_q4k, w_out, N, K, to_layout=WQ_LAYOUT_B200_V1, stream=None):
    _check(lib().wq_repack_q4k(_ptr(w_q4k), _ptr(w_out), N, K, to_layout, _stream(stream)), "wq_repack_q4k")


def wq_build_q4k_dsc(w_q4k_host: np.ndarray, N: int, K: int) -> np.ndarray:
    """Host plane builder: returns float32 [K/32, N, 2] built by libwq's C++ packer."""
    src = np.ascontiguousarray(w_q4k_host, dtype=np.uint8)
    out = np.empty((K // 32, N, 2), dtype=np.float32)
    _check(lib().wq_build_q4k_dsc(src.ctypes.data_as(ctypes.c_void_p), N, K, out.ctypes.data_as(ctypes.c_void_p)),
           "wq_build_q4k_dsc")
    return out


def wq_build_q4k_dsc_device(w_q4k, out, N, K, stream=None):
    _check(lib().wq_build_q4k_dsc_device(_ptr(w_q4k), _ptr(out), N, K, _stream(stream)), "wq_build_q4k_dsc_device")


def wq_layout_version() -> int:
    return int(lib().wq_layout_version())


def wq_device_status() -> None:
    _check(lib().wq_device_status(), "wq_device_status")


def wq_test_expire_wait(limit_ns: int, stream=None) -> None:
    _check(lib().wq_test_expire_wait(int(limit_ns), _stream(stream)), "wq_test_expire_wait")


def wq_tp_rows(N, world, rank, align=16):
    """Rows (n0, n1) of rank `rank` in a row split of N rows over `world` GPUs."""
    n0, n1 = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().wq_tp_rows(N, world, rank, align, ctypes.byref(n0), ctypes.byref(n1)), "wq_tp_rows")
    return n0.value, n1.value


def gemv_int4_tp(x, w_shard, y_dsts, M, N_shard, K, block_size, N_total, n_offset, stream=None):
    ptrs = (ctypes.c_void_p * len(y_dsts))(*[_ptr(t) for t in y_dsts])
    _check(lib().gemv_int4_tp(_ptr(x), _ptr(w_shard), ptrs, len(y_dsts), M, N_shard, K, block_size, N_total, n_offset,
                              _stream(stream)), "gemv_int4_tp")


def wq_ipc_handle(t):
    """(64-byte handle, byte offset) of the device allocation holding t."""
    buf = ctypes.create_string_buffer(64)
    off = ctypes.c_ulonglong(0)
    _check(lib().wq_ipc_handle(_ptr(t), buf, ctypes.byref(off)), "wq_ipc_handle")
    return buf.raw, off.value


def wq_ipc_open(handle: bytes, offset: int) -> int:
    p = ctypes.c_void_p(0)
    _check(lib().wq_ipc_open(ctypes.create_string_buffer(handle, 64), offset, ctypes.byref(p)), "wq_ipc_open")
    return int(p.value)


def wq_ipc_close(ptr: int, offset: int) -> None:
    _check(lib().wq_ipc_close(ptr, offset), "wq_ipc_close")
