"""CPU oracle for the weight-only quantized decode linear layer y = x·Wᵀ.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA path (its own unpackers, its own plane builder);
the only thing the two sides share is the seeded input generator module,
which holds none of the method's arithmetic.

Everything is computed in float64 from the stored bytes, with plain numpy
array operations; each function cites the passage it follows.  For every
format in scope the dequantized weight is an exact real that is also exactly
representable in fp32 (checked by ``exact_in_f32``), so fp32 RN(W) is the
bit-exact target for any device dequantization.

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py`` (hand-worked golden fixtures, closed forms,
invariants, brute force on tiny inputs); none is "parity unpinned".
"""
from .q4 import (  # noqa: F401
    QK_K,
    Q4K_BLOCK_BYTES,
    accept,
    bound,
    dequant_bf16,
    dequant_int4,
    dequant_mxfp4,
    e2m1_value,
    e8m0_value,
    MXFP4_BLOCK,
    dequant_q4k,
    dequant_q4k_from_plane,
    dequant_q8,
    exact_in_f32,
    f16_bits_to_f64,
    gemv,
    get_scale_min_k4,
    int4_codes,
    int4_zero_points,
    mmq_q4k,
    Q8_CHUNK,
    q4k_codes,
    q4k_fields,
    q4k_plane,
    q4k_scales_mins,
    quantize_q8,
    SILU_MAX_SLOPE,
    silu,
    swiglu_gemv,
    swiglu_tolerance,
    violations,
)
