"""Exact narrow-float codecs used by the oracle (TEST INFRASTRUCTURE ONLY).

E2M1 and E4M3 are the element and block-scale formats of NVFP4 ([P1]
"Optimizing FLUX 3 Image Klein inference on NVIDIA Blackwell GPUs", §How it
works, names NVFP4 weights and activations; the encoding itself is the
standard one: E2M1 elements, unsigned E4M3 block scales).  E4M3 is also the
FP8 format of the quantised Q/K/V attention ([P1] §How it works: the
quantised attention keeps Q, K and V in FP8).  bf16 is the activation storage
format.

Every encoder here is written as "pick the nearest representable value, ties
to the even code, saturate to the largest finite value", evaluated exactly in
fp64 over the explicit table of representable values.  That is the definition
of round-to-nearest-even with saturation; there is no bit trick to check.
"""

import numpy as np

# ---------------------------------------------------------------------------
# E2M1: 1 sign bit, 2 exponent bits, 1 mantissa bit; codes 0..7 are the
# magnitudes below, bit 3 is the sign.
# ---------------------------------------------------------------------------
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(codes):
    """Decode 4-bit E2M1 codes (uint8 in 0..15) to float64 values."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def _nearest_even(mag, table):
    """Index of the nearest table entry to each |value|, ties to the even index.

    ``table`` is sorted ascending and starts at 0; values above the last entry
    saturate to the last index.  All comparisons are exact in fp64 for the
    magnitudes that matter (values beyond the table saturate).
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(table, mag, side="left")          # table[hi] >= mag
    hi = np.minimum(hi, len(table) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - table[lo]
    d_hi = table[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= table[-1], len(table) - 1, idx)  # satfinite
    return idx.astype(np.uint8)


def e2m1_encode(values):
    """Round float values to E2M1 codes: nearest, ties to even, saturate at 6.

    The sign bit is the sign bit of the input, so a negative value whose
    magnitude rounds to zero encodes as 0x8 ("negative zero").  NaN input is
    rejected.
    """
    v = np.asarray(values, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("e2m1_encode: NaN input has no E2M1 code")
    code = _nearest_even(np.abs(v), E2M1_MAGNITUDES)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (code | sign).astype(np.uint8)


# ---------------------------------------------------------------------------
# E4M3 (the "fn" variant: bias 7, no infinities, S.1111.111 is NaN, largest
# finite 448).
# ---------------------------------------------------------------------------
def _e4m3_table():
    vals = np.empty(128, dtype=np.float64)
    for code in range(128):
        e, m = code >> 3, code & 7
        if e == 0:
            vals[code] = m * 2.0 ** -9                      # subnormal
        else:
            vals[code] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    vals[127] = np.nan
    return vals


E4M3_VALUES = _e4m3_table()           # index = code & 0x7f
E4M3_FINITE = E4M3_VALUES[:127]       # codes 0..126, ascending
E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Decode E4M3 bytes to float64 (0x7f / 0xff decode to NaN)."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E4M3_VALUES[codes & 0x7F]
    return np.where(codes & 0x80, -mag, mag)


def e4m3_encode(values):
    """Round float values to E4M3 bytes: nearest, ties to even, saturate to +-448.

    Infinities saturate to +-448; NaN encodes as 0x7f (sign kept).
    """
    v = np.asarray(values, dtype=np.float64)
    nan = np.isnan(v)
    mag = np.where(nan, 0.0, np.abs(v))
    code = _nearest_even(mag, E4M3_FINITE)
    code = np.where(nan, 0x7F, code).astype(np.uint8)
    sign = np.signbit(v).astype(np.uint8) << 7
    return (code | sign).astype(np.uint8)


def e4m3_round(values):
    """Value of ``values`` after rounding to E4M3 (as float64)."""
    return e4m3_decode(e4m3_encode(values))


# ---------------------------------------------------------------------------
# bf16: 8 significant bits, fp32 exponent range.
# ---------------------------------------------------------------------------
_BF16_MAX = float(np.float32(3.3895313892515355e38))


def bf16_round(values):
    """Round float64 (or fp32) values to the nearest bf16, ties to even.

    One rounding straight from the input precision: the value is split as
    m * 2**e with 0.5 <= |m| < 1, and m * 2**8 is rounded to an integer with
    round-half-even (``np.rint``), except in the subnormal range where the
    quantum is fixed at 2**-133.  Returns float32 (every bf16 is an fp32).
    """
    x = np.asarray(values, dtype=np.float64)
    _, e = np.frexp(x)
    q_exp = np.maximum(e - 8, -133)
    q = np.ldexp(1.0, q_exp)
    r = np.rint(x / q) * q                      # x / q is exact (power of 2)
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, x), r)
    r = np.where(np.isfinite(x), r, x)
    return r.astype(np.float32)


def bf16_bits(values):
    """uint16 bit patterns of bf16 values given as exact float32."""
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("bf16_bits: input is not exactly representable in bf16")
    return (bits >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    """float32 values of uint16 bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)
