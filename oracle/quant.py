"""8-bit floating-point (E4M3) cache values (oracle, test infrastructure).

"What is paged attention in vLLM, and why does it matter?", "Trade-offs and
edge cases" (fourth point): narrower cache values shrink every block. The
pages name 16-bit formats; this restates the 8-bit E4M3 format used for an
fp8 KV cache with a scale per KV head:

  stored code c = encode(x / scale)    (x / scale computed in float32)
  cache value   = decode(c) * scale

E4M3 (from its definition: 1 sign bit, 4 exponent bits with bias 7, 3
mantissa bits, no infinities): normal values (1 + m/8) * 2^(e-7) for
e = 1..15 (e = 15 with m = 7 is NaN, so the largest finite value is
1.75 * 2^8 = 448); subnormals (m/8) * 2^-6 = m * 2^-9. Encoding rounds to the
nearest representable value, ties to even, and saturates finite values beyond
448 to +-448.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_encode(x) -> np.ndarray:
    """uint8 codes of float32 values: round to nearest even, saturate at +-448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)  # exact widening
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    # subnormal range |x| < 2^-6: steps of 2^-9; the code is the step count
    # (a count of 8 rounds up into code 0x08, the smallest normal 2^-6)
    sub = _round_half_even(np.where(a < 2.0 ** -6, a, 0.0) / 2.0 ** -9)
    # normal range: |x| = (1 + f) * 2^e with f in [0, 1); code (e + 7) << 3 | round(8 f)
    normal_range = (a >= 2.0 ** -6) & (a < E4M3_MAX)
    an = np.where(normal_range, a, 1.0)
    _, e2 = np.frexp(an)                        # an = r * 2^e2 with r in [0.5, 1)
    e = e2 - 1
    m = _round_half_even((np.ldexp(an, -e) - 1.0) * 8.0)
    e = np.where(m == 8, e + 1, e)              # rounding carried into the exponent
    m = np.where(m == 8, 0, m)
    normal = ((e + 7) << 3) | m.astype(np.int64)
    code = np.where(a < 2.0 ** -6, sub.astype(np.int64), normal)
    code = np.where(a >= E4M3_MAX, 0x7E, code)  # saturate (448 itself is 0x7E)
    code = np.where(np.isnan(a), 0x7F, code)
    return code.astype(np.uint8) | sign


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of uint8 E4M3 codes (exact)."""
    c = np.asarray(codes, dtype=np.uint8)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    value = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7))
    value = np.where((c & 0x7F) == 0x7F, np.nan, value)
    return sign * value


def quantize(x, scale) -> np.ndarray:
    """Codes of x / scale, the division done in float32 (as stored by the cache)."""
    q = np.asarray(x, dtype=np.float32) / np.asarray(scale, dtype=np.float32)
    return e4m3_encode(q.astype(np.float32))


def dequantize(codes, scale) -> np.ndarray:
    """float64 cache values decode(c) * scale."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)


def _round_half_even(v):
    """Nearest integer, ties to even (numpy's rint)."""
    return np.rint(v)
