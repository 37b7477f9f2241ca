"""Seeded synthetic inputs for the decode linear layer y = x·Wᵀ.

This module draws raw canonical bytes and activation values straight from a
seeded PRNG.  It holds none of the method's arithmetic: no unpacking, no
dequantisation, no products.  Both the CPU oracle (in tests) and the CUDA path
consume what it returns, so it is the only code the two sides share.

Value distributions follow the decode workloads the pages measure (glm/qwen
int4 MatMulNBits decode, 7B q4_K_M GGUF weights, Qwen-class bf16 linears),
with synthetic stand-ins because no model files are available:

* x ~ N(0, 1), rounded to fp16 (int4, q4_K) or bf16 (bf16 path).
* int4: nibbles uniform 0..15 (uniform random bytes), fp16 scales uniform in
  a per-workload range, uint4 zero-points uniform 0..15 or absent (z = 8).
* q4_K: d, dmin fp16 uniform in [1e-3, 4e-3]; the 12 packed scale bytes and
  the 128 qs bytes uniform random (uniform bytes give uniform 6-bit scales
  and mins because the 12-byte packing is a bijection on 96 bits).
* bf16: W ~ N(0, 0.02).

Seeds: seed = 1000·workload + tensor id (x=0, W/qs=1, scales/d=2,
zero-points/dmin=3, packed 6-bit scale bytes=4).
"""
from __future__ import annotations

import numpy as np

# q4_K super-block geometry (llama.cpp block_q4_K): 256 weights in 144 bytes.
QK_K = 256
Q4K_BLOCK_BYTES = 144

TENSOR_X, TENSOR_W, TENSOR_SCALE, TENSOR_ZERO, TENSOR_SC6 = 0, 1, 2, 3, 4


def _rng(workload: int, tensor: int) -> np.random.Generator:
    return np.random.default_rng(1000 * workload + tensor)


def _to_bf16_bits(values: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (round-to-nearest-even) and return the uint16 bit patterns.

    Uses torch's own conversion so no rounding code lives here.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations_f16(M: int, K: int, workload: int = 1) -> np.ndarray:
    """x [M, K] as float16, drawn N(0,1) and rounded by numpy's float16 cast (RNE)."""
    return _rng(workload, TENSOR_X).standard_normal((M, K)).astype(np.float16)


def activations_bf16_bits(M: int, K: int, workload: int = 2) -> np.ndarray:
    """x [M, K] as bf16 bit patterns (uint16), drawn N(0,1)."""
    return _to_bf16_bits(_rng(workload, TENSOR_X).standard_normal((M, K)))


def int4_weights(N: int, K: int, block_size: int, *, scale_lo: float, scale_hi: float,
                 with_zeros: bool, workload: int) -> dict:
    """Canonical int4 MatMulNBits-style tensors as raw arrays.

    Returns a dict with
      w_packed [N, K/2] uint8   (two codes per byte, low nibble = even k)
      scales   [N, nb] float16, nb = ceil(K/block) (the last block may be shorter)
      zeros    [N, ceil(nb/2)] uint8 or None (None means z = 8)
    """
    if K % 2:
        raise ValueError("K must be even (two codes per byte)")
    nb = -(-K // block_size)
    w = _rng(workload, TENSOR_W).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = _rng(workload, TENSOR_SCALE).uniform(scale_lo, scale_hi, size=(N, nb)).astype(np.float16)
    z = None
    if with_zeros:
        z = _rng(workload, TENSOR_ZERO).integers(0, 256, size=(N, (nb + 1) // 2), dtype=np.uint8)
        if nb % 2:  # the unused high nibble of the last byte stays zero
            z[:, -1] &= 0x0F
    return {"w_packed": w, "scales": s, "zeros": z}


def q4k_weights(N: int, K: int, *, workload: int = 4,
                d_lo: float = 1e-3, d_hi: float = 4e-3) -> np.ndarray:
    """Canonical q4_K super-blocks: uint8 [N, K/256, 144].

    Bytes 0-1 fp16 d, 2-3 fp16 dmin (little-endian), 4-15 packed 6-bit
    scales/mins, 16-143 the 4-bit codes.
    """
    if K % QK_K:
        raise ValueError("K must be a multiple of 256 for q4_K")
    nsb = K // QK_K
    raw = np.empty((N, nsb, Q4K_BLOCK_BYTES), dtype=np.uint8)
    d = _rng(workload, TENSOR_SCALE).uniform(d_lo, d_hi, size=(N, nsb)).astype(np.float16)
    dmin = _rng(workload, TENSOR_ZERO).uniform(d_lo, d_hi, size=(N, nsb)).astype(np.float16)
    raw[:, :, 0:2] = d.view(np.uint8).reshape(N, nsb, 2)
    raw[:, :, 2:4] = dmin.view(np.uint8).reshape(N, nsb, 2)
    raw[:, :, 4:16] = _rng(workload, TENSOR_SC6).integers(0, 256, size=(N, nsb, 12), dtype=np.uint8)
    raw[:, :, 16:144] = _rng(workload, TENSOR_W).integers(0, 256, size=(N, nsb, 128), dtype=np.uint8)
    return raw


def bf16_weights_bits(N: int, K: int, workload: int = 2, std: float = 0.02) -> np.ndarray:
    """W [N, K] as bf16 bit patterns (uint16), drawn N(0, std)."""
    return _to_bf16_bits(_rng(workload, TENSOR_W).normal(0.0, std, size=(N, K)))


def with_element_offset(a: np.ndarray, offset: int) -> tuple[np.ndarray, np.ndarray]:
    """Place a 2-byte-element array at `offset` elements into a larger flat buffer.

    Returns (buffer, view) where view is a contiguous view of `a`'s values that
    starts `offset` elements after buffer[0].  Used for the unaligned-storage
    workloads (2-byte offsets).
    """
    flat = np.ascontiguousarray(a).reshape(-1)
    buf = np.zeros(flat.size + offset + 8, dtype=flat.dtype)
    buf[offset:offset + flat.size] = flat
    return buf, buf[offset:offset + flat.size].reshape(a.shape)


def mxfp4_weights(N: int, K: int, *, workload: int = 6, e_lo: int = 121, e_hi: int = 129) -> dict:
    """mxfp4 blockwise weights: codes uint8 [N, K/2] (uniform bytes: every E2M1
    code, both signs), E8M0 scale bytes uint8 [N, K/32] uniform in [e_lo, e_hi]
    (2^-6 .. 2^2 with the defaults)."""
    if K % 32:
        raise ValueError("mxfp4 needs K % 32 == 0")
    w = _rng(workload, TENSOR_W).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = _rng(workload, TENSOR_SCALE).integers(e_lo, e_hi + 1, size=(N, K // 32), dtype=np.uint8)
    return {"w_packed": w, "scales": s}
