"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutant is a small, realistic slip: a swapped nibble order, a wrong
byte index in the 6-bit unpacking, a dropped or sign-flipped min term, a
row-major plane, an operand read backwards, a missing absolute value.
"""
import numpy as np
import pytest

import oracle.q4 as oq
from _pins import ALL_PINS

_orig = {name: getattr(oq, name) for name in dir(oq) if not name.startswith("__")}


def _int4_codes_high_first(w_packed, N, K):
    b = np.asarray(w_packed, dtype=np.uint8).reshape(N, K // 2)
    q = np.empty((N, K), dtype=np.int64)
    q[:, 0::2] = b >> 4
    q[:, 1::2] = b & 0x0F
    return q


def _zero_points_default_zero(zeros, N, n_blocks):
    if zeros is None:
        return np.zeros((N, n_blocks), dtype=np.int64)
    return _orig["int4_zero_points"](zeros, N, n_blocks)


def _scale_min_wrong_byte(j, sc12):
    b = np.asarray(sc12).astype(np.int64)
    if j < 4:
        return b[..., j] & 63, b[..., j + 4] & 63
    return ((b[..., j + 4] & 0x0F) | ((b[..., j - 4] >> 6) << 4),
            (b[..., j + 4] >> 4) | ((b[..., j - 4] >> 6) << 4))  # min takes byte j-4


def _scale_min_nibbles_swapped(j, sc12):
    b = np.asarray(sc12).astype(np.int64)
    if j < 4:
        return b[..., j] & 63, b[..., j + 4] & 63
    return ((b[..., j + 4] >> 4) | ((b[..., j - 4] >> 6) << 4),
            (b[..., j + 4] & 0x0F) | ((b[..., j] >> 6) << 4))


def _codes_sequential(qs):
    b = np.asarray(qs, dtype=np.uint8).astype(np.int64)
    out = np.empty(b.shape[:-1] + (256,), dtype=np.int64)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


def _dequant_q4k_no_min(raw, N, K):
    d, dmin, sc12, qs = oq.q4k_fields(raw, N, K)
    sc, mn = oq.q4k_scales_mins(sc12)
    q = oq.q4k_codes(qs)
    chunk = np.arange(256) // 32
    return (d[..., None] * sc[..., chunk] * q).reshape(N, K)


def _dequant_q4k_plus_min(raw, N, K):
    d, dmin, sc12, qs = oq.q4k_fields(raw, N, K)
    sc, mn = oq.q4k_scales_mins(sc12)
    q = oq.q4k_codes(qs)
    chunk = np.arange(256) // 32
    return (d[..., None] * sc[..., chunk] * q + dmin[..., None] * mn[..., chunk]).reshape(N, K)


def _fields_d_dmin_swapped(raw, N, K):
    d, dmin, sc12, qs = _orig["q4k_fields"](raw, N, K)
    return dmin, d, sc12, qs


def _plane_row_major(raw, N, K):
    P = _orig["q4k_plane"](raw, N, K)                 # [K/32, N, 2]
    return np.ascontiguousarray(P.transpose(1, 0, 2)).reshape(K // 32, N, 2)


def _gemv_k_reversed(W, x):
    return np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64)[:, ::-1].T


def _bound_no_abs(W, x):
    return np.asarray(x, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def _accept_loose(y, y_ref, B, rel=2e-3, abs_=1e-3):
    return _orig["accept"](y, y_ref, B, rel * 2, abs_)


def _dequant_bf16_ignores_offset(w_bits, N, K, offset=0):
    return _orig["dequant_bf16"](w_bits, N, K, 0)


def _dequant_int4_block_off_by_one(w_packed, scales, zeros, N, K, block_size):
    nb = K // block_size
    q = oq.int4_codes(w_packed, N, K)
    s = oq.f16_bits_to_f64(np.asarray(scales).view(np.uint16).reshape(N, nb))
    z = oq.int4_zero_points(zeros, N, nb)
    blk = np.minimum((np.arange(K) + 1) // block_size, nb - 1)
    return (q - z[:, blk]).astype(np.float64) * s[:, blk]


def _dequant_int4_ragged_tail_in_last_full_block(w_packed, scales, zeros, N, K, block_size):
    nb = -(-K // block_size)
    q = oq.int4_codes(w_packed, N, K)
    s = oq.f16_bits_to_f64(np.asarray(scales).view(np.uint16).reshape(N, nb))
    z = oq.int4_zero_points(zeros, N, nb)
    blk = np.minimum(np.arange(K) // block_size, max(K // block_size - 1, 0))
    return (q - z[:, blk]).astype(np.float64) * s[:, blk]


def _silu_without_a(a):
    a = np.asarray(a, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-a))


def _silu_reflected(a):
    a = np.asarray(a, dtype=np.float64)
    return a / (1.0 + np.exp(a))


def _swiglu_gate_up_swapped(Wg, Wu, x):
    return oq.silu(oq.gemv(Wu, x)) * oq.gemv(Wg, x)


def _swiglu_tolerance_no_up_term(a, b, Ba, Bb, rel=2e-3, abs_=1e-3):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    ea = rel * np.asarray(Ba, dtype=np.float64) + abs_
    prop = oq.SILU_MAX_SLOPE * ea * np.abs(b)
    return prop + 2.0 ** -10 * (np.abs(oq.silu(a) * b) + prop) + abs_


def _e2m1_exponent_unbiased(code):
    c = np.asarray(code).astype(np.int64)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    return sign * np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.ldexp(1.0, e))


def _e2m1_unsigned(code):
    return np.abs(_orig["e2m1_value"](code))


def _e8m0_bias_128(byte):
    b = np.asarray(byte).astype(np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 128))


def _mxfp4_block_16(w_packed, scales, N, K):
    q = oq.int4_codes(w_packed, N, K)
    E = np.asarray(scales, dtype=np.uint8).reshape(N, K // 32)
    blk = np.minimum(np.arange(K) // 16, K // 32 - 1)
    return oq.e8m0_value(E)[:, blk] * oq.e2m1_value(q)


def _q8_variant(x, M, K, *, half_away=False, div=127.0, s_without_d=False):
    x32 = np.asarray(x, dtype=np.float16).reshape(M, K // 32, 32).astype(np.float32)
    amax = np.max(np.abs(x32), axis=2)
    d = (amax / np.float32(div)).astype(np.float32)
    safe = np.where(d > 0, d, np.float32(1.0)).astype(np.float32)
    v = (x32 / safe[..., None]).astype(np.float32)
    q = np.sign(v) * np.floor(np.abs(v) + 0.5) if half_away else np.rint(v)
    q = np.clip(np.where(d[..., None] > 0, q, 0.0), -127, 127).astype(np.int64)
    qs = q.sum(axis=2).astype(np.float32)
    s = qs if s_without_d else (d * qs).astype(np.float32)
    return q.reshape(M, K).astype(np.int8), d, s


def _mmq_variant(raw, qa, d, s, M, N, K, *, min_sign=-1.0, shift_qa=0, shift_d=0):
    C = K // 32
    P = oq.q4k_plane(raw, N, K).astype(np.float64)
    _, _, _, qs = oq.q4k_fields(raw, N, K)
    q = oq.q4k_codes(qs).reshape(N, C, 32)
    a = np.roll(np.asarray(qa, dtype=np.int8).astype(np.int64), shift_qa, axis=1).reshape(M, C, 32)
    isum = np.einsum("ncj,mcj->mnc", q, a)
    dd = np.roll(np.asarray(d, dtype=np.float32).astype(np.float64).reshape(M, C), shift_d, axis=1)
    ss = np.asarray(s, dtype=np.float32).astype(np.float64).reshape(M, C)
    return (np.einsum("cn,mc,mnc->mn", P[:, :, 0], dd, isum.astype(np.float64))
            - min_sign * np.einsum("cn,mc->mn", P[:, :, 1], ss))


MUTANTS = {
    "int4 nibbles high-first": ("int4_codes", _int4_codes_high_first),
    "int4 default zero-point 0": ("int4_zero_points", _zero_points_default_zero),
    "int4 block index off by one": ("dequant_int4", _dequant_int4_block_off_by_one),
    "int4 ragged tail read with the last full block": ("dequant_int4", _dequant_int4_ragged_tail_in_last_full_block),
    "6-bit min from byte j-4": ("get_scale_min_k4", _scale_min_wrong_byte),
    "6-bit nibbles swapped": ("get_scale_min_k4", _scale_min_nibbles_swapped),
    "q4_K codes sequential": ("q4k_codes", _codes_sequential),
    "q4_K min term dropped": ("dequant_q4k", _dequant_q4k_no_min),
    "q4_K min term sign": ("dequant_q4k", _dequant_q4k_plus_min),
    "q4_K d/dmin swapped": ("q4k_fields", _fields_d_dmin_swapped),
    "plane row-major": ("q4k_plane", _plane_row_major),
    "gemv k reversed": ("gemv", _gemv_k_reversed),
    "bound without abs": ("bound", _bound_no_abs),
    "acceptance twice as loose": ("accept", _accept_loose),
    "bf16 offset ignored": ("dequant_bf16", _dequant_bf16_ignores_offset),
    "e2m1 exponent without its bias": ("e2m1_value", _e2m1_exponent_unbiased),
    "e2m1 sign dropped": ("e2m1_value", _e2m1_unsigned),
    "e8m0 bias 128": ("e8m0_value", _e8m0_bias_128),
    "mxfp4 blocks of 16": ("dequant_mxfp4", _mxfp4_block_16),
    "silu without the a factor": ("silu", _silu_without_a),
    "silu reflected": ("silu", _silu_reflected),
    "swiglu gate and up swapped": ("swiglu_gemv", _swiglu_gate_up_swapped),
    "swiglu tolerance without the up error": ("swiglu_tolerance", _swiglu_tolerance_no_up_term),
    "q8 ties away from zero": ("quantize_q8", lambda x, M, K: _q8_variant(x, M, K, half_away=True)),
    "q8 scale amax/128": ("quantize_q8", lambda x, M, K: _q8_variant(x, M, K, div=128.0)),
    "q8 code sum without the scale": ("quantize_q8", lambda x, M, K: _q8_variant(x, M, K, s_without_d=True)),
    "mmq min term sign": ("mmq_q4k", lambda *a: _mmq_variant(*a, min_sign=1.0)),
    "mmq activations one k late": ("mmq_q4k", lambda *a: _mmq_variant(*a, shift_qa=1)),
    "mmq activation scale of the next chunk": ("mmq_q4k", lambda *a: _mmq_variant(*a, shift_d=-1)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oq, attr, fn)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(oq)
        except Exception:  # noqa: BLE001 - any failure of a pin counts as caught
            failed.append(pin.__name__)
    assert failed, f"mutant {name!r} passed every pin"
