"""The oracle's FP8 encoder against an independent bit-level encoder.

``oracle.fp8_formats.encode`` rounds through a searchsorted ladder of the
decoded codes.  The reference here shares nothing with it: it works on the
float32 bit pattern with integer arithmetic (quanta of the target binade,
round-half-to-even on the remainder, carry into the exponent, saturation to
the largest finite code).  By default every 251st of the 2^32 float32
patterns is compared (about 17M values, every exponent and every high
mantissa bit pattern); with FP8DS_EXHAUSTIVE=1 all 2^32 are.  NaN patterns
are left out (their code is a reading the pages do not fix).
"""

import os

import numpy as np
import pytest

from oracle import fp8_formats as F

# exponent bits, mantissa bits, bias, largest finite code magnitude
FMT = {F.E4M3: (4, 3, 7, 0x7E), F.E5M2: (5, 2, 15, 0x7B)}


def encode_bits(u, fmt):
    """Saturating RNE of float32 bit patterns ``u`` (uint32, no NaN) to FP8 codes."""
    E, M, bias, maxc = FMT[fmt]
    u = np.asarray(u, dtype=np.uint64)
    sign = (u >> np.uint64(31)).astype(np.int64)
    mag = (u & np.uint64(0x7FFFFFFF)).astype(np.int64)
    e32 = (mag >> 23) - 127                       # unbiased exponent of normal float32
    s = (mag & 0x7FFFFF) | (1 << 23)              # 24-bit significand: value = s * 2^(e32 - 23)
    emin = 1 - bias                               # FP8 smallest normal exponent
    te = np.maximum(e32, emin)                    # binade whose quantum 2^(te - M) applies
    sh = np.clip(23 - M + te - e32, 0, 62)        # value / quantum = s >> sh (+ remainder)
    n = s >> sh
    r = s - (n << sh)
    half = np.where(sh > 0, np.int64(1) << np.maximum(sh - 1, 0), 0)
    up = (sh > 0) & ((r > half) | ((r == half) & ((n & 1) == 1)))
    n = n + up.astype(np.int64)
    code = n + ((te + bias - 1) << M)             # carries into the exponent field by itself
    code = np.minimum(code, maxc)                 # saturation (infinity included)
    code = np.where(mag < (1 << 23), 0, code)     # float32 zero and subnormals: below half the FP8 quantum
    return (code | (sign << 7)).astype(np.uint8)


def _compare(lo, hi, step, fmt):
    u = np.arange(lo, hi, step, dtype=np.uint64).astype(np.uint32)
    x = u.view(np.float32)
    keep = ~np.isnan(x)
    u, x = u[keep], x[keep]
    got = F.encode(x, fmt)
    ref = encode_bits(u, fmt)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (f"{bad.size} mismatches; first input 0x{int(u[bad[0]]):08x}: "
                           f"oracle 0x{int(got[bad[0]]):02x}, bits 0x{int(ref[bad[0]]):02x}")


def test_bit_encoder_hand_values():
    """The reference itself on values worked by hand (OFP8 tables)."""
    vals = np.array([0.0, -0.0, 1.0, -2.0, 0.5, 480.0, 448.0, 464.0, 2.0 ** -9, 2.0 ** -10, 1.5 * 2.0 ** -10,
                     57344.0, 61440.0, np.inf, 0.875], dtype=np.float32)
    u = vals.view(np.uint32)
    e4 = encode_bits(u, F.E4M3)
    assert list(e4[:8]) == [0x00, 0x80, 0x38, 0xC0, 0x30, 0x7E, 0x7E, 0x7E]
    assert list(e4[8:11]) == [0x01, 0x00, 0x01]   # min subnormal; half of it ties to 0; 0.75 of it rounds up
    assert e4[-1] == 0x36 and e4[-2] == 0x7E
    e5 = encode_bits(u, F.E5M2)
    assert e5[11] == 0x7B and e5[12] == 0x7B and e5[13] == 0x7B  # 57344 exact; above saturates


@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_oracle_encode_equals_bit_encoder_strided(fmt):
    step = 251
    chunk = step << 22
    for lo in range(0, 1 << 32, chunk):
        _compare(lo, min(lo + chunk, 1 << 32), step, fmt)


@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_oracle_encode_equals_bit_encoder_at_rounding_boundaries(fmt):
    """Every sign, exponent and top-12 mantissa pattern with the low 11 bits at
    0, 1, 0x400 or 0x7FF: every tie between FP8 neighbours (normal and
    subnormal), one float32 ulp either side of it, and every exact code."""
    hi = np.arange(1 << 21, dtype=np.uint32) << np.uint32(11)   # sign, exponent, top 12 mantissa bits
    for low in (0, 1, 0x400, 0x7FF):
        u = hi | np.uint32(low)
        x = u.view(np.float32)
        keep = ~np.isnan(x)
        got = F.encode(x[keep], fmt)
        ref = encode_bits(u[keep], fmt)
        assert np.array_equal(got, ref), f"low bits 0x{low:x}: {int(np.count_nonzero(got != ref))} mismatches"


@pytest.mark.skipif(os.environ.get("FP8DS_EXHAUSTIVE") != "1", reason="all 2^32 patterns: set FP8DS_EXHAUSTIVE=1")
@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_oracle_encode_equals_bit_encoder_all_patterns(fmt):
    chunk = 1 << 26
    for lo in range(0, 1 << 32, chunk):
        _compare(lo, lo + chunk, 1, fmt)
