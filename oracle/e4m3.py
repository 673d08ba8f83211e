"""FP8 E4M3 codec written from the OCP 8-bit floating point definition (test infrastructure).

Format (OCP "E4M3", the ``fn`` flavour): 1 sign bit, 4 exponent bits with bias
7, 3 mantissa bits. Exponent field 0 holds subnormals ``m/8 * 2^-6``; exponent
fields 1..15 hold normals ``(1 + m/8) * 2^(e-7)``, except that ``S.1111.111``
is NaN. There are no infinities; the largest finite magnitude is
``1.75 * 2^8 = 448`` and the smallest subnormal is ``2^-9``.

The vLLM pages list an "FP8 KV Cache" among the added quantisation features
("vLLM 前世今生" sections 5.2 and 7.3) without fixing the encoding, so the
reading used here is the one the cache kernel implements: round the float32
value to nearest, ties to even, and saturate magnitudes beyond 448 to 448
("satfinite"); NaN stays NaN.
"""
from __future__ import annotations

import numpy as np

MAX_FINITE = 448.0
_MIN_NORMAL_EXP = -6  # smallest normal is 2^-6
_SUBNORMAL_QUANTUM = 2.0 ** -9


def decode(codes) -> np.ndarray:
    """uint8 codes -> float64 values (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sub = m * _SUBNORMAL_QUANTUM
    norm = (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int32))
    val = np.where(e == 0, sub, norm)
    val = np.where((e == 0xF) & (c & 0x7 == 0x7), np.nan, val)
    return sign * val


def encode(x) -> np.ndarray:
    """float values (taken exactly, as float64) -> uint8 codes, RNE with saturation.

    Every float32 input is exact in float64, and every step below (frexp,
    scaling by powers of two, ``rint``) is exact, so the rounding decision is
    taken on the exact input value.
    """
    v = np.asarray(x, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.uint8)
    sign_bit = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    nan = np.isnan(v)
    a = np.where(nan, 0.0, a)

    # Exponent of the leading bit: a = f * 2^k with f in [0.5, 1) -> leading bit 2^(k-1).
    _, k = np.frexp(a)
    lead = k.astype(np.int64) - 1
    lead = np.maximum(lead, _MIN_NORMAL_EXP)  # below 2^-6 the quantum stays 2^-9
    quantum_exp = lead - 3  # 3 mantissa bits
    q = np.rint(np.ldexp(a, (-quantum_exp).astype(np.int32)))  # ties to even
    # q counts quanta of 2^quantum_exp; q == 16 means the mantissa carried into the next binade.
    carry = q >= 16
    q = np.where(carry, q / 2, q)
    lead = np.where(carry, lead + 1, lead)
    # Subnormal region: lead == -6 and q < 8 (no implicit bit).
    is_sub = (lead == _MIN_NORMAL_EXP) & (q < 8)
    e_field = np.where(is_sub, 0, lead + 7)
    m_field = np.where(is_sub, q, q - 8)
    # Saturate: largest finite is e_field 15, m_field 6.
    over = (e_field > 15) | ((e_field == 15) & (m_field > 6)) | np.isinf(a)
    e_field = np.where(over, 15, e_field)
    m_field = np.where(over, 6, m_field)
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(a == 0.0, 0, code)
    out = (code.astype(np.uint8) | sign_bit)
    out = np.where(nan, np.uint8(0x7F) | sign_bit, out).astype(np.uint8)
    return out


def quantize(x, scale: float) -> np.ndarray:
    """Cache-side quantisation: code = encode(float32(x) * float32(1 / scale)).

    ``1/scale`` is formed once in float32 (IEEE division), and the product is
    one float32 multiply rounded to nearest, as a float32 device multiply does.
    """
    inv = np.float32(1.0) / np.float32(scale)
    prod = np.asarray(x, dtype=np.float32) * inv
    return encode(prod.astype(np.float32))


def dequantize(codes, scale: float) -> np.ndarray:
    """value = decode(code) * scale, in float64 (the scale taken as its float32 value)."""
    return decode(codes) * np.float64(np.float32(scale))
