"""FP8 formats E4M3 and E5M2: decode table and saturating RNE encoder.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages name the two formats ("AstrAI commits, branch main, tests/extension",
quantize split commit: "validate the fmt enum"; the te-style commit uses E4M3
for x/w and E5M2 for gradients) but do not define them.  The definitions
below are the OCP OFP8 ones:

* E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.  No infinities;
  S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
  Exponent field 0 is subnormal: m/8 * 2^-6.
* E5M2: 1 sign, 5 exponent bits (bias 15), 2 mantissa bits, IEEE-like:
  S.11111.00 is infinity, S.11111.{01,10,11} are NaN, largest finite
  1.75 * 2^15 = 57344.  Exponent field 0 is subnormal: m/4 * 2^-14.

Encoding of a float64/float32 value v (the method's "saturating
round-to-nearest-even"):
  * NaN -> 0x7F with v's sign bit (reading; parity unpinned, no workload
    holds NaN).
  * |v| >= FP8_MAX (infinity included) -> FP8_MAX with v's sign.
  * otherwise the representable magnitude nearest to |v|; on an exact tie
    the code whose last mantissa bit is 0 (the even code).
"""

import numpy as np

E4M3 = 0
E5M2 = 1

_LAYOUT = {E4M3: (4, 3, 7), E5M2: (5, 2, 15)}  # exponent bits, mantissa bits, bias


def decode_code(code, fmt):
    """Value of one 8-bit code as a Python float (exact), from the OFP8 fields."""
    ebits, mbits, bias = _LAYOUT[fmt]
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    emax_field = (1 << ebits) - 1
    if fmt == E4M3 and e == emax_field and m == (1 << mbits) - 1:
        return float("nan")
    if fmt == E5M2 and e == emax_field:
        return sign * float("inf") if m == 0 else float("nan")
    if e == 0:  # subnormal: 0.m * 2^(1-bias)
        return sign * (m / (1 << mbits)) * 2.0 ** (1 - bias)
    return sign * (1.0 + m / (1 << mbits)) * 2.0 ** (e - bias)


def decode_table(fmt):
    """float64[256]: value of every code (NaN/inf where the format says so)."""
    return np.array([decode_code(c, fmt) for c in range(256)], dtype=np.float64)


def fp8_max(fmt):
    """Largest finite magnitude of the format: 448 (E4M3) or 57344 (E5M2)."""
    t = decode_table(fmt)
    return float(np.max(np.abs(t[np.isfinite(t)])))


def _positive_ladder(fmt):
    """Codes 0x00.. of non-negative finite values in increasing order, and those values."""
    t = decode_table(fmt)
    codes = [c for c in range(0x80) if np.isfinite(t[c])]
    vals = t[codes]
    assert np.all(np.diff(vals) > 0), "sign-magnitude codes must be monotone"
    return np.array(codes, dtype=np.uint8), vals


def encode(v, fmt):
    """Saturating round-to-nearest-even of each element of ``v`` to an FP8 code.

    ``v`` is any float array (float32 values are exact in float64).  Returns
    uint8 codes of the same shape.
    """
    v = np.asarray(v, dtype=np.float64)
    codes, vals = _positive_ladder(fmt)
    vmax = vals[-1]
    a = np.abs(v)
    sign = np.signbit(v).astype(np.uint8) << 7

    # Index of the largest ladder value <= a (a >= 0 here; NaN handled below).
    a_clip = np.where(np.isnan(a), 0.0, np.minimum(a, vmax))
    lo = np.searchsorted(vals, a_clip, side="right") - 1
    hi = np.minimum(lo + 1, len(vals) - 1)
    lo_v = vals[lo]
    hi_v = vals[hi]
    # Midpoint of two adjacent FP8 values has at most a few significant bits,
    # so it is exact in float64 and the comparison below is exact.
    mid = (lo_v + hi_v) / 2.0
    lo_c = codes[lo]
    hi_c = codes[hi]
    even_c = np.where((lo_c & 1) == 0, lo_c, hi_c)
    pick = np.where(a_clip < mid, lo_c, np.where(a_clip > mid, hi_c, even_c))
    pick = np.where(a_clip == lo_v, lo_c, pick)
    pick = np.where(a >= vmax, codes[-1], pick)  # saturation (inf included)
    out = (pick.astype(np.uint8) | sign).astype(np.uint8)
    out = np.where(np.isnan(v), np.uint8(0x7F) | sign, out).astype(np.uint8)
    return out


def decode(codes, fmt):
    """float64 values of an array of uint8 codes."""
    return decode_table(fmt)[np.asarray(codes, dtype=np.uint8)]
