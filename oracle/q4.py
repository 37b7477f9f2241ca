"""fp64 definitions: unpack, dequantize, contract, bound.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Sources, by page:

* onnx-genai PR #1000 (cp.async re-test of the int4 MatMulNBits M=1 decode
  GEMV), section "What it does": the int4 blockwise format with fp16 scales
  and per-column fp32 accumulation.  The byte layout is not printed there; the
  reading taken is the plain row-major MatMulNBits one (codes [N][K/2], two
  per byte, low nibble = even k; scales [N][K/bs] fp16; zero-points packed
  two per byte, low nibble = even block; no zero-point array means z = 8) and
  w = (q - z)·s.
* minfer doc 62 "r59 — q4_K W_dsc plane", §2.1 (the per-chunk coefficients
  d·sc and -dmin·m), §2.2 (the chunk-major float2 plane and its size), §2.3
  (bit-identity rules), §3.2 (super-block byte offsets and the 6-bit
  scale/min unpacking rule).
* the same page, §3.2 (the MMQ dispatch arm: an int8 prepass over the
  activations feeding an integer GEMM rescaled per (chunk, row) pair as in
  §2.1): ``quantize_q8`` and ``mmq_q4k``; the prepass format is a reading.
* AstrAI commit log (astrai/extension/backend), the uint4-anchoring bullet:
  the bf16 GEMV is defined for any K >= 1 and any 2-byte storage offset.

Readings where the pages are silent are listed in the design notes; the one
that matters for values is the order of the 128 q4_K code bytes (``q4k_codes``).
"""
from __future__ import annotations

import numpy as np

QK_K = 256            # weights per q4_K super-block
Q4K_BLOCK_BYTES = 144  # 2 (d) + 2 (dmin) + 12 (scales/mins) + 128 (codes)
Q4K_CHUNK = 32        # weights sharing one (scale, min) pair


# --------------------------------------------------------------------------
# shared little helpers (value conversions only)
# --------------------------------------------------------------------------

def f16_bits_to_f64(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (exact widening)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: bf16 is the top half of a binary32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def exact_in_f32(w: np.ndarray) -> bool:
    """True when every float64 value survives a round trip through float32."""
    w = np.asarray(w, dtype=np.float64)
    return bool(np.all(w.astype(np.float32).astype(np.float64) == w))


# --------------------------------------------------------------------------
# int4 MatMulNBits-style blockwise (onnx-genai PR #1000, "What it does")
# --------------------------------------------------------------------------

def int4_codes(w_packed, N: int, K: int) -> np.ndarray:
    """Unpack the 4-bit codes q[n, k] in 0..15 from [N][K/2] bytes, low nibble first."""
    if K % 2:
        raise ValueError("int4 K must be even")
    b = np.asarray(w_packed, dtype=np.uint8).reshape(N, K // 2)
    q = np.empty((N, K), dtype=np.int64)
    q[:, 0::2] = b & 0x0F
    q[:, 1::2] = b >> 4
    return q


def int4_zero_points(zeros, N: int, n_blocks: int) -> np.ndarray:
    """Zero-points z[n, b]: uint4 packed two per byte (low nibble = even block); None means 8."""
    if zeros is None:
        return np.full((N, n_blocks), 8, dtype=np.int64)
    per_row = (n_blocks + 1) // 2
    b = np.asarray(zeros, dtype=np.uint8).reshape(N, per_row)
    z = np.empty((N, 2 * per_row), dtype=np.int64)
    z[:, 0::2] = b & 0x0F
    z[:, 1::2] = b >> 4
    return z[:, :n_blocks]


def dequant_int4(w_packed, scales, zeros, N: int, K: int, block_size: int) -> np.ndarray:
    """W[n, k] = (q[n,k] - z[n, k//bs]) · s[n, k//bs] in float64 (exact).

    A row has nb = ceil(K/bs) blocks; when bs does not divide K the last one
    covers the remaining K - (nb-1)·bs codes (ragged last block; the code
    array keeps K/2 bytes per row, no padding)."""
    if block_size <= 0:
        raise ValueError("block_size must be positive")
    nb = -(-K // block_size)
    q = int4_codes(w_packed, N, K)
    s = f16_bits_to_f64(np.asarray(scales).view(np.uint16).reshape(N, nb))
    z = int4_zero_points(zeros, N, nb)
    blk = np.arange(K) // block_size
    return (q - z[:, blk]).astype(np.float64) * s[:, blk]


# --------------------------------------------------------------------------
# q4_K super-blocks (minfer doc 62, §2.1, §2.2, §3.2)
# --------------------------------------------------------------------------

def q4k_fields(raw, N: int, K: int):
    """Split [N][K/256][144] bytes into (d, dmin, sc12, qs) with d, dmin as float64.

    Byte offsets per super-block (§3.2): fp16 d at 0..1, fp16 dmin at 2..3
    (little-endian), 12 packed scale/min bytes at 4..15, 128 code bytes at 16..143.
    """
    if K % QK_K:
        raise ValueError("q4_K needs K % 256 == 0")
    blk = np.asarray(raw, dtype=np.uint8).reshape(N, K // QK_K, Q4K_BLOCK_BYTES)
    d_bits = blk[..., 0].astype(np.uint16) | (blk[..., 1].astype(np.uint16) << 8)
    m_bits = blk[..., 2].astype(np.uint16) | (blk[..., 3].astype(np.uint16) << 8)
    return f16_bits_to_f64(d_bits), f16_bits_to_f64(m_bits), blk[..., 4:16], blk[..., 16:144]


def get_scale_min_k4(j: int, sc12) -> tuple:
    """6-bit (scale, min) of chunk j (0..7) from the 12 packed bytes (§2.1, §3.2).

    Chunks 0..3 keep their scale in the low 6 bits of byte j and their min in
    the low 6 bits of byte j+4.  Chunks 4..7 combine a low nibble of byte j+4
    (scale) or its high nibble (min) with the two top bits of byte j-4
    (scale) or byte j (min) as bits 4..5.  Works elementwise on arrays whose
    last axis holds the 12 bytes.
    """
    b = np.asarray(sc12).astype(np.int64)
    if j < 4:
        return b[..., j] & 63, b[..., j + 4] & 63
    scale = (b[..., j + 4] & 0x0F) | ((b[..., j - 4] >> 6) << 4)
    mn = (b[..., j + 4] >> 4) | ((b[..., j] >> 6) << 4)
    return scale, mn


def q4k_scales_mins(sc12):
    """All eight (scale, min) pairs: two int arrays with a trailing axis of 8."""
    pairs = [get_scale_min_k4(j, sc12) for j in range(8)]
    return (np.stack([p[0] for p in pairs], axis=-1), np.stack([p[1] for p in pairs], axis=-1))


def q4k_codes(qs) -> np.ndarray:
    """Codes q[..., e] for the 256 elements of a super-block from its 128 code bytes.

    Reading (the pages only say "128 B of 4-bit q" in 32-element chunks): the
    llama.cpp grouping.  Code bytes come in four runs of 32; run p holds chunk
    2p in its low nibbles and chunk 2p+1 in its high nibbles, element i of
    each chunk in byte i of the run.
    """
    b = np.asarray(qs, dtype=np.uint8).astype(np.int64)
    out = np.empty(b.shape[:-1] + (QK_K,), dtype=np.int64)
    for p in range(4):
        run = b[..., 32 * p:32 * p + 32]
        out[..., 64 * p:64 * p + 32] = run & 0x0F
        out[..., 64 * p + 32:64 * p + 64] = run >> 4
    return out


def dequant_q4k(raw, N: int, K: int) -> np.ndarray:
    """W[n, k] = d·sc_c·q − dmin·m_c in float64, c = the 32-element chunk of k (§2.1)."""
    d, dmin, sc12, qs = q4k_fields(raw, N, K)
    sc, mn = q4k_scales_mins(sc12)                     # [N, nsb, 8]
    q = q4k_codes(qs)                                  # [N, nsb, 256]
    chunk = np.arange(QK_K) // Q4K_CHUNK               # chunk of each element
    scale = d[..., None] * sc[..., chunk]              # d·sc   (exact in fp64)
    offset = dmin[..., None] * mn[..., chunk]          # dmin·m (exact in fp64)
    w = scale * q - offset
    return w.reshape(N, K)


def q4k_plane(raw, N: int, K: int) -> np.ndarray:
    """The chunk-major W_dsc plane as float32 [K/32, N, 2] (§2.2, §2.3).

    Entry (c, n) = (fp32(d)·fp32(sc), −(fp32(dmin)·fp32(m))) for global chunk
    c = 8·superblock + j of row n: one IEEE binary32 multiply each (numpy
    float32 multiply, no contraction) and an exact negation.  Flattened, entry
    (c, n) sits at byte offset (c·N + n)·8, so the plane is N·K/4 bytes.
    """
    d, dmin, sc12, _ = q4k_fields(raw, N, K)
    sc, mn = q4k_scales_mins(sc12)                     # [N, nsb, 8]
    d32 = d.astype(np.float32)
    m32 = dmin.astype(np.float32)
    px = d32[..., None] * sc.astype(np.float32)        # [N, nsb, 8]
    py = -(m32[..., None] * mn.astype(np.float32))
    plane = np.empty((K // Q4K_CHUNK, N, 2), dtype=np.float32)
    plane[:, :, 0] = px.reshape(N, K // Q4K_CHUNK).T
    plane[:, :, 1] = py.reshape(N, K // Q4K_CHUNK).T
    return plane


def dequant_q4k_from_plane(raw, plane, N: int, K: int) -> np.ndarray:
    """W[n, k] = P.x·q + P.y with P the plane entry of k's chunk, in float64."""
    _, _, _, qs = q4k_fields(raw, N, K)
    q = q4k_codes(qs).reshape(N, K).astype(np.float64)
    P = np.asarray(plane, dtype=np.float32).reshape(K // Q4K_CHUNK, N, 2).astype(np.float64)
    chunk = np.arange(K) // Q4K_CHUNK
    return P[chunk, :, 0].T * q + P[chunk, :, 1].T


# --------------------------------------------------------------------------
# mxfp4 blockwise (named by the block_quantized_matmul / _moe mxfp4 rows of the
# CPU criterion bench block in onnx-genai PR #1000; the page does not print
# the format, so the reading taken is the OCP microscaling FP4 definition:
# blocks of 32 along K share one E8M0 scale 2^(E - 127), elements are E2M1)
# --------------------------------------------------------------------------

MXFP4_BLOCK = 32


def e2m1_value(code) -> np.ndarray:
    """Value of a 4-bit E2M1 code: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.

    Exponent field 0 is the subnormal range (0 or 0.5); otherwise the value is
    2^(e - 1)·(1 + m/2).
    """
    c = np.asarray(code).astype(np.int64)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.ldexp(1.0, np.maximum(e - 1, 0)))
    return sign * mag


def e8m0_value(byte) -> np.ndarray:
    """2^(E - 127) for an E8M0 scale byte (255 is NaN)."""
    b = np.asarray(byte).astype(np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


def dequant_mxfp4(w_packed, scales, N: int, K: int) -> np.ndarray:
    """W[n, k] = 2^(E[n, k // 32] - 127) · e2m1(q[n, k]) in float64 (exact).

    Codes [N][K/2] bytes, two per byte, low nibble = even k (the int4 reading);
    scales [N][K/32] E8M0 bytes.
    """
    if K % MXFP4_BLOCK:
        raise ValueError("mxfp4 needs K % 32 == 0")
    q = int4_codes(w_packed, N, K)
    E = np.asarray(scales, dtype=np.uint8).reshape(N, K // MXFP4_BLOCK)
    blk = np.arange(K) // MXFP4_BLOCK
    return e8m0_value(E)[:, blk] * e2m1_value(q)


# --------------------------------------------------------------------------
# bf16 (AstrAI commit log, uint4-anchoring bullet: any K, any 2-byte offset)
# --------------------------------------------------------------------------

def dequant_bf16(w_bits, N: int, K: int, offset: int = 0) -> np.ndarray:
    """W[n, k] from bf16 bits stored row-major with row stride K, `offset` elements in."""
    flat = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    return bf16_bits_to_f64(flat[offset:offset + N * K]).reshape(N, K)


# --------------------------------------------------------------------------
# contraction, bound and acceptance
# --------------------------------------------------------------------------

def gemv(W, x) -> np.ndarray:
    """y[m, n] = Σ_k W[n, k]·x[m, k] in float64 (x given as its stored values)."""
    W = np.asarray(W, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    return x @ W.T


def bound(W, x) -> np.ndarray:
    """B[m, n] = Σ_k |W[n, k]·x[m, k]|, the scale of the acceptance test."""
    return np.abs(np.asarray(x, dtype=np.float64)) @ np.abs(np.asarray(W, dtype=np.float64)).T


def violations(y, y_ref, B, rel: float = 2e-3, abs_: float = 1e-3) -> np.ndarray:
    """Boolean mask of elements with |y − y_ref| > rel·B + abs_."""
    y = np.asarray(y, dtype=np.float64)
    return ~(np.abs(y - y_ref) <= rel * B + abs_)


def accept(y, y_ref, B, rel: float = 2e-3, abs_: float = 1e-3) -> bool:
    """True iff every element satisfies |y − y_ref| ≤ rel·B + abs_ (NaN fails)."""
    return not bool(np.any(violations(y, y_ref, B, rel, abs_)))


# --------------------------------------------------------------------------
# fused gate / up projection with the SiLU·mul epilogue (the "swiglu" launch
# that minfer doc 62 "r59 — q4_K W_dsc plane", §3.3 riders, prewarms; the page
# names the fused launch but not its formula: the reading taken is the usual
# SwiGLU feed-forward half, silu(x·Wgᵀ) ⊙ (x·Wuᵀ), with silu(a) = a·σ(a))
# --------------------------------------------------------------------------

SILU_MAX_SLOPE = 1.0999  # an upper bound of |d silu / da| over the reals (1.09984 near a = 2.4)


def silu(a) -> np.ndarray:
    """silu(a) = a·σ(a) = a / (1 + e^(−a)) in float64."""
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu_gemv(Wg, Wu, x) -> np.ndarray:
    """y[m, n] = silu(Σ_k Wg[n,k]·x[m,k]) · Σ_k Wu[n,k]·x[m,k] in float64."""
    return silu(gemv(Wg, x)) * gemv(Wu, x)


def swiglu_tolerance(a, b, Ba, Bb, rel: float = 2e-3, abs_: float = 1e-3) -> np.ndarray:
    """Acceptance bound for y = silu(a)·b when each projection is computed to
    the GEMV bound |Δa| ≤ ea = rel·Ba + abs_, |Δb| ≤ eb = rel·Bb + abs_ (Ba,
    Bb the Σ|w·x| of each), and y is rounded once to fp16 at the end:

      |Δy| ≤ S·ea·(|b| + eb) + |silu(a)|·eb + 2^-10·(|silu(a)·b| + S·ea·(|b| + eb) + |silu(a)|·eb) + abs_,

    S the largest slope of silu (mean value theorem on silu(a + Δa)), 2^-10 a
    generous bound on the relative rounding of the fp16 result and of the
    fp32 evaluation of silu."""
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    ea = rel * np.asarray(Ba, dtype=np.float64) + abs_
    eb = rel * np.asarray(Bb, dtype=np.float64) + abs_
    prop = SILU_MAX_SLOPE * ea * (np.abs(b) + eb) + np.abs(silu(a)) * eb
    return prop + 2.0 ** -10 * (np.abs(silu(a) * b) + prop) + abs_


# --------------------------------------------------------------------------
# int8-activation batched q4_K (minfer doc 62 "r59 — q4_K W_dsc plane": §2.1
# the rank-1 rescale of each (chunk, row) pair by (d·sc, −dmin·m); §3.2 the
# MMQ dispatch arm, which quantizes the activations to int8 in a prepass and
# hands the GEMM the int8 values and their scales)
# --------------------------------------------------------------------------

Q8_CHUNK = 32  # activations sharing one int8 scale (one q4_K chunk)


def quantize_q8(x, M: int, K: int):
    """The q8 prepass over fp16 activations x [M, K].

    The pages name the prepass but print no format; the reading taken: per
    row m and 32-element chunk c (the q4_K chunk), in IEEE binary32 with each
    operation rounded once (numpy float32 arithmetic, no contraction):
      amax = max |x|            (exact: fp16 values widen exactly),
      d    = amax / 127,
      q    = x / d rounded to the nearest integer, ties to even (0 when d = 0),
      s    = d · Σ q            (Σ q is an exact integer).
    Returns qa int8 [M, K], d float32 [M, K/32], s float32 [M, K/32].
    """
    if K % Q8_CHUNK:
        raise ValueError("the q8 prepass needs K % 32 == 0")
    x32 = np.asarray(x, dtype=np.float16).reshape(M, K // Q8_CHUNK, Q8_CHUNK).astype(np.float32)
    amax = np.max(np.abs(x32), axis=2)
    d = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(d > 0, d, np.float32(1.0)).astype(np.float32)
    q = np.rint((x32 / safe[..., None]).astype(np.float32))
    q = np.where(d[..., None] > 0, q, 0.0).astype(np.int64)
    s = (d * q.sum(axis=2).astype(np.float32)).astype(np.float32)
    return q.reshape(M, K).astype(np.int8), d, s


def dequant_q8(qa, d, M: int, K: int) -> np.ndarray:
    """The activations the int8 path multiplies by: d[m, c]·q[m, k] in float64 (exact)."""
    q = np.asarray(qa, dtype=np.int8).astype(np.float64).reshape(M, K // Q8_CHUNK, Q8_CHUNK)
    return (q * np.asarray(d, dtype=np.float32).astype(np.float64)[..., None]).reshape(M, K)


def mmq_q4k(raw, qa, d, s, M: int, N: int, K: int) -> np.ndarray:
    """y[m, n] = Σ_c (d·sc)[n,c]·d[m,c]·I[m,n,c] + (−dmin·m)[n,c]·s[m,c] in float64.

    I[m, n, c] = Σ_{k in chunk c} q[n, k]·qa[m, k] is the exact integer dot
    product of the chunk's 4-bit weight codes and int8 activations; the two
    coefficients of each (chunk, row) pair are the W_dsc plane entries (§2.2:
    one fp32 multiply each), and (d, s) are the prepass's per-chunk activation
    scale and scaled code sum.  Since w = (d·sc)·q − dmin·m on every element
    of a chunk, this is Σ_k w[n,k]·d[m,c]·qa[m,k] up to the rounding of s.
    """
    C = K // Q8_CHUNK
    P = q4k_plane(raw, N, K).astype(np.float64)                # [C, N, 2]
    _, _, _, qs = q4k_fields(raw, N, K)
    q = q4k_codes(qs).reshape(N, C, Q8_CHUNK)                   # int64 codes 0..15
    a = np.asarray(qa, dtype=np.int8).astype(np.int64).reshape(M, C, Q8_CHUNK)
    isum = np.einsum("ncj,mcj->mnc", q, a)                      # exact int64
    dd = np.asarray(d, dtype=np.float32).astype(np.float64).reshape(M, C)
    ss = np.asarray(s, dtype=np.float32).astype(np.float64).reshape(M, C)
    scale_term = np.einsum("cn,mc,mnc->mn", P[:, :, 0], dd, isum.astype(np.float64))
    min_term = np.einsum("cn,mc->mn", P[:, :, 1], ss)
    return scale_term + min_term
