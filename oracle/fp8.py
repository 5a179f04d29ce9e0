"""FP8 E4M3 (the "e4m3fn" variant: no infinities, max finite 448) encode and
decode, written from the format definition.  TEST INFRASTRUCTURE.

Used for the FP8 KV pool write: zigzag.py, ``materialize_full_kv`` hands
``layer.k_scale`` / ``layer.v_scale`` to ``set_kv_buffer``.  Reading (the page
shows only the call): the pool holds ``e4m3(x / scale)`` with the division in
fp32, rounding to nearest even, and finite overflow saturating to +-448.

Format: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent 0
holds subnormals m/8 * 2^-6; codes S.1111.111 are NaN; the largest finite
magnitude is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import numpy as np

MAX_FINITE = 448.0


def decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _round_half_even(x):
    return np.round(x)      # numpy rounds halves to even


def encode(x) -> np.ndarray:
    """float32 values -> E4M3 codes (round to nearest even, saturate finite overflow)."""
    x = np.asarray(x, dtype=np.float64)       # exact widening of the fp32 inputs
    sign = (np.signbit(x)).astype(np.int64) << 7
    a = np.abs(x)
    out = np.zeros(a.shape, dtype=np.int64)
    nan = np.isnan(a)
    # exponent of the leading bit, clamped to the subnormal range
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    e = np.maximum(e, -6)
    # quantum at that exponent: 2^(e-3); round the magnitude to a multiple of it
    q = np.ldexp(1.0, e - 3)
    r = _round_half_even(a / q) * q
    # rounding may carry into the next binade; recompute the fields from r
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(r > 0, r, 1.0))).astype(np.int64)
    er = np.maximum(er, -6)
    sub = r < 2.0 ** -6
    mant_sub = np.round(r / 2.0 ** -9).astype(np.int64)                  # r = m * 2^-9
    mant_norm = np.round((r / np.ldexp(1.0, er) - 1.0) * 8).astype(np.int64)
    code_norm = ((er + 7) << 3) | mant_norm
    code = np.where(sub, mant_sub, code_norm)
    code = np.where(r > MAX_FINITE, 0x7E, code)       # saturate: 1.1111.110 = 448
    code = np.where(nan, 0x7F, code)
    out = (code | np.where(nan, 0, sign)).astype(np.uint8)
    return out


def scale_encode(x_bf16_as_f32, scale: float) -> np.ndarray:
    """The pool value: e4m3(fp32(x) / fp32(scale)), division rounded in fp32."""
    q = (np.asarray(x_bf16_as_f32, dtype=np.float32) / np.float32(scale)).astype(np.float32)
    return encode(q)
