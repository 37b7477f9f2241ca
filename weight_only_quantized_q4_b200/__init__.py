"""weight_only_quantized_q4_b200 — B200 (sm_100a) weight-only quantized decode linear layer.

y = x·Wᵀ with W dequantized on the fly, for int4 MatMulNBits-style blocks,
q4_K super-blocks (optionally with the pre-decoded W_dsc plane) and bf16.
The kernels live in libwq.so (C ABI in include/wq.h); this package is a thin
ctypes binding with the same entry-point names.
"""
from .api import (  # noqa: F401
    WQ_ERR_ARG,
    WQ_ERR_TIMEOUT,
    WQ_ERR_UNSUPPORTED,
    WQ_LAYOUT_B200_V1,
    WQ_LAYOUT_CANONICAL,
    WQError,
    dequant_int4_blockwise,
    dequant_mxfp4,
    dequant_q4k,
    gemv_bf16,
    gemv_int4_blockwise,
    gemv_int4_swiglu,
    gemv_mxfp4,
    gemv_q4k,
    gemv_q4k_dsc,
    gemv_q4k_noalloc,
    last_error,
    last_kernel,
    wq_build_q4k_dsc,
    wq_build_q4k_dsc_device,
    wq_device_status,
    wq_int4_bytes,
    wq_int4_codes_bytes,
    wq_int4_gate_up_packed_bytes,
    wq_int4_packed_bytes,
    wq_repack_int4,
    wq_repack_int4_gate_up,
    wq_layout_version,
    wq_q4k_bytes,
    wq_q4k_dsc_bytes,
    wq_q4k_packed_bytes,
    wq_repack_q4k,
    wq_test_expire_wait,
)
