"""Plain CPU statement of the FP8 latent cache: how a 576-dim bf16 row is
encoded into FP8 E4M3 codes with one per-token scale, and what row the decode
then attends to.

TEST INFRASTRUCTURE ONLY: the tests are its only callers.  It shares no code
with the CUDA path and imports nothing from it.

The pages name FP8 support as the next step to cut the cache's memory ("FlashMLA:
Revolutionizing Efficient Decoding...", section 9 "Future Directions") and give
no format.  The reading taken here:
  - E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; subnormals;
    largest finite value 448; codes 0x7F and 0xFF are NaN and never written);
  - one scale per cached token, a power of two 2^k, so that code * 2^k is
    exactly the value the decode uses (no rounding when it is widened back);
  - k is the smallest integer with max_c |x_c| <= 448 * 2^k (k = 0 for an
    all-zero row), so the largest magnitude lands in (224, 448];
  - code_c = x_c / 2^k rounded to the nearest E4M3 value, ties to the even
    code (x_c / 2^k is exact, so this is the only rounding); the sign is kept,
    so a negative value that rounds to zero is coded -0 (0x80), as an IEEE
    conversion does.
The decode over an FP8 cache is then the plain definition of the decode over
the dequantised rows code * 2^k (oracle.decode on those rows).
"""
from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """The real number an E4M3 code stands for (NaN for 0x7F / 0xFF)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * m * 2.0 ** -9          # subnormal: m/8 * 2^(1-7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


# every finite non-negative code with its value, in increasing value order
_POS_CODES = np.array([c for c in range(0x7F)], dtype=np.int64)
_POS_VALUES = np.array([e4m3_value(c) for c in _POS_CODES], dtype=np.float64)
assert np.all(np.diff(_POS_VALUES) > 0)


def e4m3_round(y) -> np.ndarray:
    """Codes of the E4M3 values nearest to y (|y| <= 448), ties to the even code."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    if np.any(a > E4M3_MAX) or np.any(np.isnan(a)):
        raise ValueError("value outside the E4M3 range")
    hi = np.searchsorted(_POS_VALUES, a, side="left")       # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(a == _POS_VALUES[hi], _POS_CODES[hi], code)
    # the sign is kept, zero included (a negative value that rounds to zero is -0)
    return (code | np.where(np.signbit(y), 0x80, 0)).astype(np.uint8)


def e4m3_round_grid(y) -> np.ndarray:
    """e4m3_round computed on the value grid instead of by table search (faster,
    the same result): |y| in [2^E, 2^(E+1)) is a multiple of 2^(E-3) away from
    an E4M3 value (E >= -6; below 2^-6 the grid is 2^-9), so the nearest value
    is rint(|y| / 2^(E-3)) steps, rint rounding halves to even."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    if np.any(a > E4M3_MAX) or np.any(np.isnan(a)):
        raise ValueError("value outside the E4M3 range")
    _, e = np.frexp(a)
    E = np.maximum(e - 1, -6)
    m = np.rint(np.ldexp(a, 3 - E)).astype(np.int64)   # steps of 2^(E-3)
    carry = m == 16                                     # rounded up into the next binade
    E = np.where(carry, E + 1, E)
    m = np.where(carry, 8, m)
    normal = m >= 8
    code = np.where(normal, ((E + 7) << 3) | (m - 8), m)
    return (code | np.where(np.signbit(y), 0x80, 0)).astype(np.uint8)


def decode_codes(codes) -> np.ndarray:
    """Values of an array of codes (float64)."""
    table = np.array([e4m3_value(c) for c in range(256)])
    return table[np.asarray(codes, dtype=np.int64)]


def scale_exponent(amax: float) -> int:
    """Smallest integer k with amax <= 448 * 2^k (0 when amax is 0)."""
    if amax == 0.0:
        return 0
    k = math.ceil(math.log2(amax / E4M3_MAX))
    # guard the floating-point log against an off-by-one either way
    while amax > E4M3_MAX * 2.0 ** k:
        k += 1
    while amax <= E4M3_MAX * 2.0 ** (k - 1):
        k -= 1
    return k


def encode_row(x):
    """(codes uint8 [576], scale float) for one row of real values."""
    x = np.asarray(x, dtype=np.float64)
    k = scale_exponent(float(np.max(np.abs(x))) if x.size else 0.0)
    return e4m3_round(np.ldexp(x, -k)), math.ldexp(1.0, k)


def encode_rows(rows, chunk: int = 4096):
    """rows [..., 576] float -> (codes [..., 576] uint8, scales [...] float64).

    The same rule as encode_row, applied to `chunk` rows at a time."""
    rows = np.asarray(rows, dtype=np.float64)
    flat = rows.reshape(-1, rows.shape[-1])
    codes = np.zeros(flat.shape, dtype=np.uint8)
    scales = np.zeros(flat.shape[0], dtype=np.float64)
    for n0 in range(0, flat.shape[0], chunk):
        block = flat[n0:n0 + chunk]
        # scale_exponent for every row at once: amax = f * 2^e with f in [0.5, 1)
        # and 448 = 0.875 * 2^9, so k = e - 9 when f <= 0.875, else e - 8
        f, e = np.frexp(np.max(np.abs(block), axis=1))
        k = np.where(f == 0, 0, np.where(f <= 0.875, e - 9, e - 8)).astype(np.int64)
        codes[n0:n0 + chunk] = e4m3_round_grid(np.ldexp(block, -k[:, None]))
        scales[n0:n0 + chunk] = np.ldexp(1.0, k)
    return codes.reshape(rows.shape), scales.reshape(rows.shape[:-1])


def dequantize(codes, scales) -> np.ndarray:
    """codes [..., 576] with scales [...] -> values [..., 576] float64 (exact)."""
    return decode_codes(codes) * np.asarray(scales, dtype=np.float64)[..., None]
