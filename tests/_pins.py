"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes a namespace ``o`` holding the oracle's functions, so the same
pins run against the real oracle (tests/test_oracle_pins.py) and against
deliberately broken copies of it (tests/test_oracle_mutants.py), which shows
that a plausible mistake in the oracle fails at least one pin.

Sources of truth used here: hand-worked golden fixtures under tests/golden/
(each citing the page passage it follows), closed forms, the bijection of
the 12-byte 6-bit packing, brute-force pure-Python loops on tiny inputs, and
math.fsum for exact sums.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from weight_only_quantized_q4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f16_bytes(v):
    return list(np.array([v], dtype=np.float16).view(np.uint8))


# ---------------------------------------------------------------- q4_K pins

def pin_scale_min_golden(o):
    """Hand-worked examples of the two-case 6-bit unpacking rule."""
    for case in _golden("q4k_scale_min_k4.json")["cases"]:
        sc12 = np.array(case["sc12"], dtype=np.uint8)
        for j in range(8):
            s, m = o.get_scale_min_k4(j, sc12)
            assert int(s) == case["scales"][j], (j, int(s), case["scales"][j])
            assert int(m) == case["mins"][j], (j, int(m), case["mins"][j])


def _pack_scale_min(s, m):
    """Inverse of the 6-bit rule, written from the bit positions it names.

    scales 0..3 -> low 6 bits of bytes 0..3, their top 2 bits unused by them;
    mins 0..3 -> low 6 bits of bytes 4..7;
    scales 4..7 -> low nibble of bytes 8..11 and the top 2 bits of bytes 0..3;
    mins 4..7 -> high nibble of bytes 8..11 and the top 2 bits of bytes 4..7.
    """
    b = [0] * 12
    for j in range(4):
        b[j] = (s[j] & 63) | ((s[j + 4] >> 4) << 6)
        b[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        b[j + 8] = (s[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    return b


def pin_scale_min_bijection(o):
    """The 12 bytes carry exactly 8 six-bit scales + 8 six-bit mins (96 bits, each once)."""
    rng = np.random.default_rng(7)
    for _ in range(300):
        s = [int(v) for v in rng.integers(0, 64, 8)]
        m = [int(v) for v in rng.integers(0, 64, 8)]
        b = np.array(_pack_scale_min(s, m), dtype=np.uint8)
        got = [o.get_scale_min_k4(j, b) for j in range(8)]
        assert [int(g[0]) for g in got] == s
        assert [int(g[1]) for g in got] == m
    for _ in range(300):
        b = [int(v) for v in rng.integers(0, 256, 12)]
        got = [o.get_scale_min_k4(j, np.array(b, dtype=np.uint8)) for j in range(8)]
        assert _pack_scale_min([int(g[0]) for g in got], [int(g[1]) for g in got]) == b


def _hand_superblock():
    g = _golden("q4k_superblock_hand.json")
    blk = np.zeros(144, dtype=np.uint8)
    blk[0:2] = np.array([g["d_f16_bits"]], dtype=np.uint16).view(np.uint8)
    blk[2:4] = np.array([g["dmin_f16_bits"]], dtype=np.uint16).view(np.uint8)
    blk[4:16] = g["sc12"]
    for k, v in g["qs_nonzero"].items():
        blk[16 + int(k)] = v
    return g, blk


def pin_q4k_hand_superblock(o):
    """A hand-built super-block with hand-worked dequantized values."""
    g, blk = _hand_superblock()
    W = o.dequant_q4k(blk.reshape(1, 1, 144), 1, 256)
    for e, v in g["expect"].items():
        assert W[0, int(e)] == v, (e, W[0, int(e)], v)


def _brute_q4k(raw, N, K):
    """Element-by-element q4_K dequantization in pure Python (tiny inputs only)."""
    raw = np.asarray(raw, dtype=np.uint8).reshape(N, K // 256, 144)
    out = np.zeros((N, K))
    for n in range(N):
        for sb in range(K // 256):
            blk = [int(v) for v in raw[n, sb]]
            d = float(np.array([blk[0] | (blk[1] << 8)], dtype=np.uint16).view(np.float16)[0])
            dmin = float(np.array([blk[2] | (blk[3] << 8)], dtype=np.uint16).view(np.float16)[0])
            sc = blk[4:16]
            for e in range(256):
                c = e // 32
                if c < 4:
                    s, m = sc[c] & 63, sc[c + 4] & 63
                else:
                    s = (sc[c + 4] & 15) | ((sc[c - 4] >> 6) << 4)
                    m = (sc[c + 4] >> 4) | ((sc[c] >> 6) << 4)
                run, i = divmod(e, 64)
                byte = blk[16 + 32 * run + (i % 32)]
                q = (byte & 15) if i < 32 else (byte >> 4)
                out[n, 256 * sb + e] = d * s * q - dmin * m
    return out


def pin_q4k_brute(o):
    """q4_K value = d·sc·q − dmin·m, element by element, on a 3×512 tensor."""
    raw = synth.q4k_weights(3, 512, workload=901)
    W = o.dequant_q4k(raw, 3, 512)
    assert np.array_equal(W, _brute_q4k(raw, 3, 512))


def pin_q4k_sc_zero(o):
    """With all scales 0 every weight of a chunk is the constant −dmin·m."""
    raw = synth.q4k_weights(2, 256, workload=902).copy()
    s = [0] * 8
    m = [1, 7, 13, 63, 2, 40, 5, 33]
    raw[:, :, 4:16] = np.array(_pack_scale_min(s, m), dtype=np.uint8)
    W = o.dequant_q4k(raw, 2, 256)
    for n in range(2):
        dmin = float(raw[n, 0, 2:4].view(np.float16)[0])
        for c in range(8):
            assert np.all(W[n, 32 * c:32 * c + 32] == -dmin * m[c])


def pin_q4k_plane(o):
    """Plane entries reproduce the products: P.x == d·sc, P.y == −dmin·m (exact),
    P.x·q + P.y == W bitwise in fp32 and exactly in fp64, the plane is
    chunk-major (entry (c, n) at flat index c·N + n) and N·K/4 bytes."""
    N, K = 5, 768
    raw = synth.q4k_weights(N, K, workload=903)
    P = np.asarray(o.q4k_plane(raw, N, K))
    assert P.dtype == np.float32 and P.nbytes == N * K // 4
    flat = P.reshape(-1, 2)
    for n in range(N):
        for sb in range(K // 256):
            blk = raw.reshape(N, K // 256, 144)[n, sb]
            d = float(blk[0:2].view(np.float16)[0])
            dmin = float(blk[2:4].view(np.float16)[0])
            sc = [int(v) for v in blk[4:16]]
            for j in range(8):
                if j < 4:
                    s, m = sc[j] & 63, sc[j + 4] & 63
                else:
                    s = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4)
                    m = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4)
                c = 8 * sb + j
                assert float(flat[c * N + n, 0]) == d * s
                assert float(flat[c * N + n, 1]) == -(dmin * m)
    W = o.dequant_q4k(raw, N, K)
    Wp = o.dequant_q4k_from_plane(raw, P, N, K)
    assert np.array_equal(W, Wp)
    assert np.array_equal(W.astype(np.float32), Wp.astype(np.float32))


def pin_q4k_codes_layout(o):
    """Code-byte order: a byte whose low nibble is l and high nibble h in run p
    at position i gives element 64p+i = l and element 64p+32+i = h."""
    qs = np.zeros(128, dtype=np.uint8)
    rng = np.random.default_rng(11)
    qs[:] = rng.integers(0, 256, 128)
    q = o.q4k_codes(qs)
    for p in range(4):
        for i in range(32):
            b = int(qs[32 * p + i])
            assert q[64 * p + i] == (b & 15)
            assert q[64 * p + 32 + i] == (b >> 4)


# ---------------------------------------------------------------- int4 pins

def _hand_int4(with_zeros):
    g = _golden("int4_hand.json")
    w = np.zeros((1, 16), dtype=np.uint8)
    for k, v in g["w_bytes_nonzero"].items():
        w[0, int(k)] = v
    s = np.array([g["scales_f16"]], dtype=np.float16)
    z = np.array([[g["zeros_byte"]]], dtype=np.uint8) if with_zeros else None
    return g, w, s, z


def pin_int4_hand(o):
    """Hand-worked (q − z)·s values, with and without a zero-point array."""
    for with_zeros, key in ((True, "expect_with_zeros"), (False, "expect_without_zeros")):
        g, w, s, z = _hand_int4(with_zeros)
        W = o.dequant_int4(w, s, z, 1, 32, 16)
        for k, v in g[key].items():
            assert W[0, int(k)] == v, (key, k, W[0, int(k)], v)


def _brute_int4(w, s, z, N, K, bs):
    out = np.zeros((N, K))
    nb = (K + bs - 1) // bs  # a shorter last block when bs does not divide K
    for n in range(N):
        for k in range(K):
            byte = int(w[n, k // 2])
            q = (byte & 15) if k % 2 == 0 else (byte >> 4)
            b = k // bs
            if z is None:
                zz = 8
            else:
                zb = int(z[n, b // 2])
                zz = (zb & 15) if b % 2 == 0 else (zb >> 4)
            out[n, k] = (q - zz) * float(s[n, b])
    assert nb == s.shape[1]
    return out


def pin_int4_brute(o):
    """(q − z)·s element by element, odd block count included (3 blocks of 32)."""
    for with_zeros in (True, False):
        t = synth.int4_weights(3, 96, 32, scale_lo=0.005, scale_hi=0.02,
                               with_zeros=with_zeros, workload=904)
        W = o.dequant_int4(t["w_packed"], t["scales"], t["zeros"], 3, 96, 32)
        assert np.array_equal(W, _brute_int4(t["w_packed"], t["scales"], t["zeros"], 3, 96, 32))


def pin_int4_ragged_brute(o):
    """A ragged last block (K not a multiple of the block): element by element,
    odd and even block counts (80 = 32+32+16, 48 = 32+16, 144 = 128+16)."""
    for N, K, bs in ((3, 80, 32), (2, 48, 32), (2, 144, 128)):
        for with_zeros in (True, False):
            t = synth.int4_weights(N, K, bs, scale_lo=0.005, scale_hi=0.02,
                                   with_zeros=with_zeros, workload=907)
            assert t["scales"].shape == (N, -(-K // bs))
            W = o.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs)
            assert np.array_equal(W, _brute_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs))


def pin_int4_ragged_is_a_prefix(o):
    """Cutting K to a ragged length keeps the first K columns of the full-block
    matrix: same scales and zero-points, each row's first K/2 code bytes."""
    N, bs = 3, 64
    Kf = 4 * bs
    t = synth.int4_weights(N, Kf, bs, scale_lo=0.005, scale_hi=0.02, with_zeros=True, workload=908)
    Wf = o.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, Kf, bs)
    for K in (Kf - 16, Kf - bs + 2, 3 * bs + 32):
        w = np.ascontiguousarray(t["w_packed"][:, :K // 2])
        W = o.dequant_int4(w, t["scales"], t["zeros"], N, K, bs)
        assert np.array_equal(W, Wf[:, :K])


def pin_int4_zero_equals_code(o):
    """z = q everywhere (every code equal to its block's zero-point) gives W ≡ 0, y ≡ 0."""
    N, K, bs = 4, 64, 16
    codes = np.random.default_rng(3).integers(0, 16, (N, K // bs))
    w = np.zeros((N, K // 2), dtype=np.uint8)
    z = np.zeros((N, K // bs // 2), dtype=np.uint8)
    for n in range(N):
        for b in range(K // bs):
            c = int(codes[n, b])
            for k in range(b * bs, (b + 1) * bs, 2):
                w[n, k // 2] = c | (c << 4)
            z[n, b // 2] |= c << (4 * (b % 2))
    s = np.random.default_rng(4).uniform(0.01, 1.0, (N, K // bs)).astype(np.float16)
    W = o.dequant_int4(w, s, z, N, K, bs)
    assert np.all(W == 0)
    x = synth.activations_f16(3, K, workload=905)
    assert np.all(o.gemv(W, x) == 0)


# ---------------------------------------------------------------- bf16 pins

def pin_bf16_offsets_and_odd_k(o):
    """bf16 for K ∈ {7, 12, 100, 1534} at offsets 0 and +1 element (2 bytes):
    identical values, and y equal to a brute-force fsum loop."""
    for K in (7, 12, 100, 1534):
        N, M = 3, 2
        wb = synth.bf16_weights_bits(N, K, workload=906)
        xb = synth.activations_bf16_bits(M, K, workload=906)
        ref = None
        for off in (0, 1):
            buf, _ = synth.with_element_offset(wb, off)
            W = o.dequant_bf16(buf, N, K, offset=off)
            if ref is None:
                ref = W
            assert np.array_equal(W, ref)
        x = o.dequant_bf16(xb, M, K)
        y = o.gemv(ref, x)
        for m in range(M):
            for n in range(N):
                w_row = [float(np.array([int(wb[n, k]) << 16], dtype=np.uint32).view(np.float32)[0])
                         for k in range(K)]
                x_row = [float(np.array([int(xb[m, k]) << 16], dtype=np.uint32).view(np.float32)[0])
                         for k in range(K)]
                exact = math.fsum(a * b for a, b in zip(w_row, x_row))
                assert abs(y[m, n] - exact) <= 1e-12 * math.fsum(abs(a * b) for a, b in zip(w_row, x_row)) + 1e-300


# ------------------------------------------------------- contraction pins

def pin_gemv_one_hot(o):
    """x = e_k picks column k of W exactly."""
    t = synth.int4_weights(6, 64, 32, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=907)
    W = o.dequant_int4(t["w_packed"], t["scales"], t["zeros"], 6, 64, 32)
    for k in (0, 1, 31, 63):
        x = np.zeros((1, 64))
        x[0, k] = 1.0
        assert np.array_equal(o.gemv(W, x)[0], W[:, k])


def pin_gemv_constant(o):
    """x ≡ 1 with a constant W gives y = K·w."""
    K = 40
    W = np.full((3, K), -1.375)
    x = np.ones((2, K))
    assert np.all(o.gemv(W, x) == K * -1.375)


def pin_gemv_fsum(o):
    """y equals a brute-force fsum of the products (to fp64 rounding) and the
    bound equals the fsum of absolute products; x and W not transposed."""
    rng = np.random.default_rng(12)
    W = rng.standard_normal((4, 9))
    x = rng.standard_normal((3, 9))
    y = o.gemv(W, x)
    B = o.bound(W, x)
    assert y.shape == (3, 4) and B.shape == (3, 4)
    for m in range(3):
        for n in range(4):
            exact = math.fsum(W[n, k] * x[m, k] for k in range(9))
            absum = math.fsum(abs(W[n, k] * x[m, k]) for k in range(9))
            assert abs(y[m, n] - exact) <= 1e-13 * absum
            assert abs(B[m, n] - absum) <= 1e-13 * absum


def pin_accept_threshold(o):
    """The acceptance test passes at 0.99× the tolerance and fails at 1.01× and on NaN."""
    for y0, b in ((1.0, 10.0), (-2.0, 3.0), (0.0, 0.0), (5.0, 1000.0)):
        y_ref = np.array([[y0]])
        B = np.array([[b]])
        tol = 2e-3 * b + 1e-3
        assert o.accept(y_ref + 0.99 * tol, y_ref, B)
        assert o.accept(y_ref - 0.99 * tol, y_ref, B)
        assert not o.accept(y_ref + 1.01 * tol, y_ref, B)
        assert not o.accept(y_ref - 1.01 * tol, y_ref, B)
    assert not o.accept(np.array([[np.nan]]), np.array([[0.0]]), np.array([[1.0]]))


def pin_exact_in_f32(o):
    """Dequantized weights of every workload distribution are exact fp32 values."""
    t = synth.int4_weights(64, 1024, 32, scale_lo=0.005, scale_hi=0.02, with_zeros=False, workload=1)
    assert o.exact_in_f32(o.dequant_int4(t["w_packed"], t["scales"], None, 64, 1024, 32))
    t = synth.int4_weights(64, 1024, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=3)
    assert o.exact_in_f32(o.dequant_int4(t["w_packed"], t["scales"], t["zeros"], 64, 1024, 128))
    raw = synth.q4k_weights(64, 1024, workload=4)
    assert o.exact_in_f32(o.dequant_q4k(raw, 64, 1024))
    assert not o.exact_in_f32(np.array([1.0 + 2.0 ** -30]))


# ---------------------------------------------------------------- mxfp4 pins

# The sixteen E2M1 values in code order (sign bit 3, exponent bits 2..1,
# mantissa bit 0): the format's value table, typed out, not computed.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def pin_e2m1_table(o):
    got = o.e2m1_value(np.arange(16))
    assert [float(v) for v in got] == E2M1_TABLE
    assert all(math.copysign(1.0, float(g)) == math.copysign(1.0, t) for g, t in zip(got, E2M1_TABLE))


def pin_e8m0_scales(o):
    """E8M0 byte E is 2^(E - 127); 255 is NaN."""
    cases = {127: 1.0, 128: 2.0, 126: 0.5, 0: 2.0 ** -127, 254: 2.0 ** 127, 120: 1.0 / 128}
    for b, v in cases.items():
        assert float(o.e8m0_value(b)) == v, b
    assert math.isnan(float(o.e8m0_value(255)))


def pin_mxfp4_hand(o):
    """Two blocks of one row: block 0 scale byte 128 (x2) with first codes 1, 2
    (0.5, 1.0 -> 1.0, 2.0); block 1 scale byte 125 (x1/4) with first codes
    15, 8 (-6, -0 -> -1.5, -0); every other code 0."""
    w = np.zeros((1, 32), dtype=np.uint8)
    w[0, 0] = 0x21                   # k0 = code 1, k1 = code 2
    w[0, 16] = 0x8F                  # k32 = code 15, k33 = code 8
    sc = np.array([[128, 125]], dtype=np.uint8)
    W = o.dequant_mxfp4(w, sc, 1, 64)
    assert W[0, 0] == 1.0 and W[0, 1] == 2.0 and W[0, 32] == -1.5 and W[0, 33] == 0.0
    assert np.count_nonzero(W) == 3


def pin_mxfp4_brute(o):
    """Element by element through the typed value table on a small random tensor."""
    rng = np.random.default_rng(91)
    N, K = 3, 96
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sc = rng.integers(110, 140, (N, K // 32), dtype=np.uint8)
    W = o.dequant_mxfp4(w, sc, N, K)
    for n in range(N):
        for k in range(K):
            byte = int(w[n, k // 2])
            code = byte & 15 if k % 2 == 0 else byte >> 4
            want = E2M1_TABLE[code] * 2.0 ** (int(sc[n, k // 32]) - 127)
            assert W[n, k] == want, (n, k)
    assert o.exact_in_f32(W)


# ---------------------------------------------------------------- SwiGLU pins

def pin_silu_closed_forms(o):
    """silu(a) = a·σ(a) where the logistic function has closed forms:
    σ(0) = 1/2, σ(ln 3) = 3/4, σ(−ln 3) = 1/4, σ(1) = e/(e + 1); and its limits."""
    ln3 = math.log(3.0)
    assert float(o.silu(0.0)) == 0.0
    assert abs(float(o.silu(ln3)) - 0.75 * ln3) <= 1e-15
    assert abs(float(o.silu(-ln3)) + 0.25 * ln3) <= 1e-15
    assert abs(float(o.silu(1.0)) - math.e / (math.e + 1.0)) <= 1e-15
    assert float(o.silu(40.0)) == 40.0
    assert abs(float(o.silu(-40.0))) <= 1e-15 and float(o.silu(-1e4)) == 0.0


def pin_silu_reflection_and_slope(o):
    """silu(a) − silu(−a) = a (σ(a) + σ(−a) = 1), and the slope bound the
    tolerance uses is attained: the steepest finite-difference slope on a
    fine grid lies just below it."""
    a = np.random.default_rng(71).uniform(-30.0, 30.0, 2000)
    assert np.allclose(o.silu(a) - o.silu(-a), a, rtol=1e-12, atol=1e-12)
    g = np.linspace(-12.0, 12.0, 240001)
    h = 1e-6
    slope = np.abs((o.silu(g + h) - o.silu(g - h)) / (2 * h))
    assert slope.max() <= o.SILU_MAX_SLOPE and slope.max() >= o.SILU_MAX_SLOPE - 1e-3


def pin_swiglu_hand(o):
    """Hand example: gate row (0.5, 0.5) and x = (1, 1) give a = 1, up row
    (2, 0) gives b = 2, so y = 2·silu(1) = 2e/(e + 1); a gate row of zeros
    gives y = 0 whatever b is; a = −30 gives |y| ≤ 30·e^-30·|b|."""
    Wg = np.array([[0.5, 0.5], [0.0, 0.0]])
    Wu = np.array([[2.0, 0.0], [1.0, 3.0]])
    y = o.swiglu_gemv(Wg, Wu, np.array([[1.0, 1.0]]))
    assert abs(y[0, 0] - 2.0 * math.e / (math.e + 1.0)) <= 1e-15 and y[0, 1] == 0.0
    y2 = o.swiglu_gemv(Wg, Wu, np.array([[-60.0, 0.0]]))
    assert abs(y2[0, 0]) <= 30.0 * math.exp(-30.0) * 120.0 * 1.0001 and y2[0, 1] == 0.0


def pin_swiglu_tolerance_covers_worst_case(o):
    """The acceptance bound of the fused projection covers every combination
    of a and b each off by its full GEMV bound, plus fp16 rounding of y."""
    rng = np.random.default_rng(72)
    a = rng.uniform(-8, 8, 4000)
    b = rng.uniform(-8, 8, 4000) * rng.choice([1.0, 1e-3], 4000)
    Ba = np.abs(a) * rng.uniform(1, 50, 4000)
    Bb = np.abs(b) * rng.uniform(1, 50, 4000)
    tol = o.swiglu_tolerance(a, b, Ba, Bb)
    ea, eb = 2e-3 * Ba + 1e-3, 2e-3 * Bb + 1e-3
    y = a / (1 + np.exp(-a)) * b  # the unperturbed value, for the property only
    for sa in (-1, 1):
        for sb in (-1, 1):
            a2, b2 = a + sa * ea, b + sb * eb
            yp = a2 / (1 + np.exp(-a2)) * b2
            for r in (1 - 2.0 ** -11, 1 + 2.0 ** -11):
                assert np.all(np.abs(yp * r - y) <= tol)


# ---------------------------------------------------------------- q8 prepass and int8-activation q4_K

def _golden_q8():
    g = _golden("q8_prepass_hand.json")
    x = np.zeros((1, 32 * len(g["x_chunks"])), dtype=np.float16)
    q = np.zeros(x.shape, dtype=np.int64)
    for c, (xs, qs) in enumerate(zip(g["x_chunks"], g["q_chunks"])):
        x[0, 32 * c:32 * c + len(xs)] = xs
        q[0, 32 * c:32 * c + len(qs)] = qs
    bits = lambda v: np.array([int(b, 16) for b in v], dtype=np.uint32).view(np.float32)  # noqa: E731
    return x, q, bits(g["d_bits"]), bits(g["s_bits"])


def pin_q8_golden(o):
    """Hand-worked chunks: exact scales, ties to even, zero chunk, a scale that rounds."""
    x, q, d, s = _golden_q8()
    qa, dd, ss = o.quantize_q8(x, 1, x.shape[1])
    assert qa.dtype == np.int8 and np.array_equal(qa.astype(np.int64), q)
    assert np.array_equal(dd.reshape(-1).view(np.uint32), d.view(np.uint32))
    assert np.array_equal(ss.reshape(-1).view(np.uint32), s.view(np.uint32))


def pin_q8_properties(o):
    """On random fp16 rows (plus a tiny-valued and a large-valued row): |q| <= 127,
    the largest |q| of every non-zero chunk is 127, |x - d·q| <= d·(1/2 + 2^-16)
    (one rounding of the quotient), and s is d·Σq rounded once."""
    M, K = 5, 1024
    x = synth.activations_f16(M, K, workload=910)
    x[3] = (x[3].astype(np.float64) * 1e-6).astype(np.float16)    # fp16 subnormal range
    x[4] = (x[4].astype(np.float64) * 1.5e4).astype(np.float16)
    x[2, 64:96] = 0
    qa, d, s = o.quantize_q8(x, M, K)
    q = qa.astype(np.int64).reshape(M, K // 32, 32)
    xc = x.astype(np.float64).reshape(M, K // 32, 32)
    dd = d.astype(np.float64)[..., None]
    assert np.all(np.abs(q) <= 127)
    nz = np.max(np.abs(xc), axis=2) > 0
    assert np.all(np.max(np.abs(q), axis=2)[nz] == 127) and np.all(q[~nz] == 0) and np.all(d[~nz] == 0)
    assert np.all(np.abs(xc - dd * q) <= dd * (0.5 + 2.0 ** -16))
    exact = d.astype(np.float64) * q.sum(axis=2)
    assert np.all(np.abs(s.astype(np.float64) - exact) <= 2.0 ** -24 * np.abs(exact))


def _brute_mmq(raw, qa, d, s, M, N, K):
    """y by the definition, in pure Python: per chunk, the exact integer dot
    product of the nibble codes and the int8 values, times d·sc and the
    activation scale, plus −dmin·m times s (d·sc and dmin·m are exact: an fp16
    times a 6-bit integer)."""
    raw = np.asarray(raw, dtype=np.uint8).reshape(N, K // 256, 144)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            terms = []
            for sb in range(K // 256):
                blk = [int(v) for v in raw[n, sb]]
                dw = float(np.array([blk[0] | (blk[1] << 8)], dtype=np.uint16).view(np.float16)[0])
                dmin = float(np.array([blk[2] | (blk[3] << 8)], dtype=np.uint16).view(np.float16)[0])
                sc = blk[4:16]
                for c in range(8):
                    if c < 4:
                        sv, mv = sc[c] & 63, sc[c + 4] & 63
                    else:
                        sv = (sc[c + 4] & 15) | ((sc[c - 4] >> 6) << 4)
                        mv = (sc[c + 4] >> 4) | ((sc[c] >> 6) << 4)
                    isum = 0
                    for i in range(32):
                        byte = blk[16 + 32 * (c // 2) + i]
                        code = (byte & 15) if c % 2 == 0 else (byte >> 4)
                        isum += code * int(qa[m, 256 * sb + 32 * c + i])
                    gc = 8 * sb + c
                    terms.append(dw * sv * float(d[m, gc]) * isum)
                    terms.append(-(dmin * mv) * float(s[m, gc]))
            y[m, n] = math.fsum(terms)
    return y


def pin_mmq_brute(o):
    """The int8-activation q4_K product equals the definition evaluated term by term."""
    M, N, K = 2, 3, 512
    raw = synth.q4k_weights(N, K, workload=911)
    qa, d, s = o.quantize_q8(synth.activations_f16(M, K, workload=911), M, K)
    y = o.mmq_q4k(raw, qa, d, s, M, N, K)
    yb = _brute_mmq(raw, qa, d, s, M, N, K)
    assert np.all(np.abs(y - yb) <= 1e-12 * (1 + np.abs(yb))), np.abs(y - yb).max()


def pin_mmq_is_the_gemv_of_the_quantized_activations(o):
    """Since w = d·sc·q − dmin·m on every element of a chunk, the factored
    product equals W·(d·qa) except for the one rounding of s: the difference
    is at most Σ_c |dmin·m|·|s − d·Σqa| (plus fp64 noise)."""
    M, N, K = 3, 40, 1024
    raw = synth.q4k_weights(N, K, workload=912)
    x = synth.activations_f16(M, K, workload=912)
    qa, d, s = o.quantize_q8(x, M, K)
    y = o.mmq_q4k(raw, qa, d, s, M, N, K)
    W = _brute_q4k(raw, N, K)
    xd = qa.astype(np.float64) * np.repeat(d.astype(np.float64), 32, axis=1)
    y2 = xd @ W.T
    P = o.q4k_plane(raw, N, K).astype(np.float64)                       # [C, N, 2]
    ds = np.abs(s.astype(np.float64) - d.astype(np.float64) * qa.astype(np.int64).reshape(M, -1, 32).sum(axis=2))
    slack = ds @ np.abs(P[:, :, 1]) + 1e-12 * (np.abs(xd) @ np.abs(W).T)
    assert np.all(np.abs(y - y2) <= slack)
    assert np.array_equal(o.dequant_q8(qa, d, M, K), xd)


ALL_PINS = [
    pin_scale_min_golden,
    pin_scale_min_bijection,
    pin_q4k_hand_superblock,
    pin_q4k_brute,
    pin_q4k_sc_zero,
    pin_q4k_plane,
    pin_q4k_codes_layout,
    pin_int4_hand,
    pin_int4_brute,
    pin_int4_ragged_brute,
    pin_int4_ragged_is_a_prefix,
    pin_int4_zero_equals_code,
    pin_bf16_offsets_and_odd_k,
    pin_gemv_one_hot,
    pin_gemv_constant,
    pin_gemv_fsum,
    pin_accept_threshold,
    pin_exact_in_f32,
    pin_e2m1_table,
    pin_e8m0_scales,
    pin_mxfp4_hand,
    pin_mxfp4_brute,
    pin_silu_closed_forms,
    pin_silu_reflection_and_slope,
    pin_swiglu_hand,
    pin_swiglu_tolerance_covers_worst_case,
    pin_q8_golden,
    pin_q8_properties,
    pin_mmq_brute,
    pin_mmq_is_the_gemv_of_the_quantized_activations,
]
