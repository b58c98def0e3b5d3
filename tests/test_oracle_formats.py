"""Pins for oracle/fp8_formats.py: the OFP8 definitions, a library cast and brute force.

None of these checks re-types the oracle's formula: decoded values are pinned
to closed forms and to torch's float8 dtypes (a library decoder); encoding is
pinned to torch's float8 cast inside the finite range (a library encoder with
round-to-nearest-even), to exact rational brute force, and to hand-picked ties.
"""

import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp8_formats as F


def test_decode_closed_forms_e4m3():
    t = F.decode_table(F.E4M3)
    assert t[0x00] == 0.0 and not np.signbit(t[0x00])
    assert t[0x80] == 0.0 and np.signbit(t[0x80])
    assert t[0x01] == 2.0 ** -9          # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert t[0x08] == 2.0 ** -6          # smallest normal
    assert t[0x38] == 1.0
    assert t[0x39] == 1.125
    assert t[0x7E] == 448.0
    assert t[0xFE] == -448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2 and np.sum(np.isinf(t)) == 0
    assert F.fp8_max(F.E4M3) == 448.0


def test_decode_closed_forms_e5m2():
    t = F.decode_table(F.E5M2)
    assert t[0x01] == 2.0 ** -16
    assert t[0x04] == 2.0 ** -14
    assert t[0x3C] == 1.0
    assert t[0x7B] == 57344.0
    assert t[0x7C] == np.inf and t[0xFC] == -np.inf
    assert all(np.isnan(t[c]) for c in (0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF))
    assert np.sum(np.isnan(t)) == 6 and np.sum(np.isinf(t)) == 2
    assert F.fp8_max(F.E5M2) == 57344.0


@pytest.mark.parametrize("fmt,tdt", [(F.E4M3, torch.float8_e4m3fn), (F.E5M2, torch.float8_e5m2)])
def test_decode_matches_torch_float8(fmt, tdt):
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(tdt).to(torch.float64).numpy()
    ours = F.decode_table(fmt)
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(lib[~nan], ours[~nan])
    assert np.array_equal(np.signbit(lib[~nan]), np.signbit(ours[~nan]))


@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_roundtrip_every_code(fmt):
    t = F.decode_table(fmt)
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], dtype=np.uint8)
    assert np.array_equal(F.encode(t[codes], fmt), codes)


def _structured_fp32():
    """fp32 patterns: every sign, exponent and top-8 mantissa bits, with 6 low-bit tails.

    The round and sticky positions of both formats (normal and subnormal) lie in
    the top 8 mantissa bits, so ties and just-above / just-below cases all occur.
    """
    s = np.arange(2, dtype=np.uint32)[:, None, None, None] << 31
    e = np.arange(256, dtype=np.uint32)[None, :, None, None] << 23
    m = np.arange(256, dtype=np.uint32)[None, None, :, None] << 15
    low = np.array([0, 1, 0x3FFF, 0x4000, 0x4001, 0x7FFF], dtype=np.uint32)[None, None, None, :]
    bits = (s | e | m | low).ravel()
    return bits.view(np.float32)


@pytest.mark.parametrize("fmt,tdt", [(F.E4M3, torch.float8_e4m3fn), (F.E5M2, torch.float8_e5m2)])
def test_encode_matches_torch_cast_in_range(fmt, tdt):
    v = _structured_fp32()
    v = v[np.isfinite(v) & (np.abs(v) <= F.fp8_max(fmt))]
    lib = torch.from_numpy(v.copy()).to(tdt).view(torch.uint8).numpy()
    ours = F.encode(v, fmt)
    bad = np.nonzero(lib != ours)[0]
    assert bad.size == 0, (v[bad[:5]], lib[bad[:5]], ours[bad[:5]])


def _f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def _brute_nearest(v, fmt):
    """Exact rational nearest finite code, ties to the even code, saturating."""
    t = F.decode_table(fmt)
    fin = [c for c in range(0x80) if np.isfinite(t[c])]
    vmax = max(t[c] for c in fin)
    sign = 0x80 if np.signbit(v) else 0
    if np.isinf(v):
        return max(fin, key=lambda c: t[c]) | sign
    a = abs(Fraction(v))
    if a >= Fraction(vmax):
        return max(fin, key=lambda c: t[c]) | sign
    best = min(fin, key=lambda c: (abs(Fraction(t[c]) - a), c & 1))
    return best | sign


@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_encode_matches_rational_brute_force(fmt):
    rng = np.random.default_rng(7)
    t = F.decode_table(fmt)
    fin = np.array([t[c] for c in range(0x80) if np.isfinite(t[c])])
    mids = (fin[:-1] + fin[1:]) / 2.0
    samples = list(mids) + list(-mids[::7])
    samples += list(np.float32(rng.standard_normal(300) * 10.0 ** rng.integers(-6, 6, 300)))
    samples += [fin[-1] * 1.01, 1e30, -np.inf, np.inf, 0.0, -0.0]
    samples = np.array(samples, dtype=np.float32)
    ours = F.encode(samples, fmt)
    for v, got in zip(samples, ours):
        assert got == _brute_nearest(float(v), fmt), (float(v), hex(got))


def test_ties_go_to_even_code():
    # 1.0625 lies halfway between 1.0 (0x38) and 1.125 (0x39): even code 0x38.
    assert F.encode([1.0625], F.E4M3)[0] == 0x38
    # 1.1875 lies halfway between 1.125 (0x39) and 1.25 (0x3A): even code 0x3A.
    assert F.encode([1.1875], F.E4M3)[0] == 0x3A
    # Half the smallest subnormal rounds to zero; three halves to code 2.
    assert F.encode([2.0 ** -10], F.E4M3)[0] == 0x00
    assert F.encode([3 * 2.0 ** -10], F.E4M3)[0] == 0x02
    assert F.encode([-(2.0 ** -17)], F.E5M2)[0] == 0x80
    # In the top binade the E4M3 step is 32: 400 is halfway between 384 (0x7C)
    # and 416 (0x7D), so it takes the even code 0x7C.
    assert F.encode([400.0], F.E4M3)[0] == 0x7C


def test_saturation():
    assert list(F.encode([448.0, 449.0, 464.0, 1e6, np.inf], F.E4M3)) == [0x7E] * 5
    assert list(F.encode([-480.0, -np.inf], F.E4M3)) == [0xFE, 0xFE]
    assert list(F.encode([57344.0, 61440.0, 1e9, np.inf], F.E5M2)) == [0x7B] * 4
    assert F.encode([-1e9], F.E5M2)[0] == 0xFB


def test_fp32_bit_boundaries_near_max():
    # Largest fp32 below 448 must round to 448 or 416 by distance; 432 is the midpoint.
    below_mid = _f32(0x43D7FFFF)  # just under 432
    above_mid = _f32(0x43D80001)
    assert F.encode([below_mid], F.E4M3)[0] == 0x7D  # 416
    assert F.encode([above_mid], F.E4M3)[0] == 0x7E  # 448
    assert F.encode([432.0], F.E4M3)[0] == 0x7E      # tie -> even code 0x7E
